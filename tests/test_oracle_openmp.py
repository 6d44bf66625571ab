"""The OpenMP build of the oracle (blocks and elements spread over threads)
gives the single-threaded build's results bit for bit: window rows, codes,
delta/Delta and parameters (fp32 and bf16), on flat and per-tensor cuts, over
several steps with a full window."""
import numpy as np
import pytest

import oracle
from compressed_state_optimizer_b200 import workloads


@pytest.mark.parametrize("d,Bd,kb,m,steps,segs,bf16", [
    (20 * 2048 + 777, 2048, 21, 4, 7, None, False),
    (6 * 4096 + 8, 4096, 41, 3, 5, [4096 * 2 + 8, 1000, 4096 * 3 + 3096], False),
    (9 * 1024 + 6, 1024, 11, 5, 7, None, True),
])
def test_openmp_build_bit_identical(oracle_lib, d, Bd, kb, m, steps, segs, bf16):
    if segs is not None:
        assert sum(segs) == d
    oracle.set_threads(4)
    w = workloads.Workload("omp", d, Bd, kb, m, "t3", steps, seed=5)
    p0 = workloads.make_params(d, seed=3).numpy()
    if bf16:
        p0 = workloads.bf16_bits(workloads.make_params(d, seed=3).to(__import__("torch").bfloat16))
    a, b = (oracle.new_state(d, Bd, kb, m, segments=segs) for _ in range(2))
    pa, pb = p0.copy(), p0.copy()
    hyper = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.01, seed=17)
    for t in range(1, steps + 1):
        g = workloads.bf16_bits(workloads.make_grads(w, t))
        sa = oracle.step(a, pa, g, t=t, want_stats=True, **hyper)
        sb = oracle.step(b, pb, g, t=t, want_stats=True, openmp=True, **hyper)
        for x, y in ((a.codes, b.codes), (a.scal, b.scal), (a.G_idx, b.G_idx),
                     (a.G_val, b.G_val), (pa, pb), *zip(sa, sb)):
            assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), t
