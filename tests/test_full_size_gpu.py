"""Full-size parity on the benchmark workloads, in the launch configuration
bench.py times, on outputs the oracle can compute one block at a time.

Step 1 starts from the zero state, so every block is independent of the others
except through delta_2 / Delta_2:
  * sampled blocks: the window row and the parameter update equal the oracle
    run on that block alone (bit for bit / 1e-5);
  * delta_2, Delta_2: the min and max of the residual over the whole vector,
    computed independently with torch reductions from the gradients and the
    (row-verified) selection;
  * sampled blocks' codes equal the oracle's quantizer applied with the
    verified delta_2, Delta_2.
The LLaMA-2-7B-shaped case needs about 70 GB of device memory.
"""
import numpy as np
import pytest

import oracle
import state_view
from conftest import cuda_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


def _free_bytes():
    import torch
    free, _ = torch.cuda.mem_get_info()
    return free


def _block_spans(w, nb):
    """(start, length) of every block: per tensor for a per-tensor cut."""
    segs = w.segments()
    if segs is None:
        return [(j * w.Bd, min(w.Bd, w.d - j * w.Bd)) for j in range(nb)]
    out, off = [], 0
    for n in segs:
        out += [(off + b, min(w.Bd, n - b)) for b in range(0, n, w.Bd)]
        off += n
    assert len(out) == nb
    return out


def check_step1_sampled(w, n_random=27, need_bytes=0):
    import torch
    from compressed_state_optimizer_b200 import MicroAdam, workloads
    if _free_bytes() < need_bytes:
        pytest.skip(f"needs {need_bytes / 1e9:.0f} GB of free device memory")
    d, Bd, kb, m = w.d, w.Bd, w.kb, w.m
    mo = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m, segments=w.segments())
    dev = torch.device("cuda", 0)
    params = workloads.make_params(d, seed=7, device=dev)
    grads = workloads.make_grads(w, 1, device=dev)
    nb = mo.layout.blocks
    spans = _block_spans(w, nb)
    rng = np.random.default_rng(11)
    sample = sorted(set([0, 1, nb // 2, nb - 2, nb - 1] + list(rng.integers(0, nb, n_random))))
    p0 = {j: params[spans[j][0]: spans[j][0] + spans[j][1]].cpu().numpy().copy() for j in sample}
    state = mo.new_state(dev)
    hyper = dict(lr=w.lr, beta1=w.beta1, beta2=w.beta2, eps=w.eps, wd=w.wd, seed=w.seed)
    mo.step(params, grads, state, t=1, **hyper)
    torch.cuda.synchronize()

    lay = mo.layout
    kp = lay.row_stride
    win = state[lay.window: lay.bytes].view(torch.int32)
    row = 1 % m
    for j in sample:
        lo, L = spans[j]
        g = workloads.bf16_bits(grads[lo:lo + L])
        ost = oracle.new_state(L, Bd, kb, m)
        p = p0[j].copy()
        oracle.step(ost, p, g, t=1, **hyper)
        gw = win[(j * m + row) * kp: (j * m + row) * kp + kb].cpu().numpy().view(np.uint32)
        gi = (gw & 0xFFFF).astype(np.uint16).view(np.int16)
        gv = (gw >> 16).astype(np.uint16)
        assert np.array_equal(gi, ost.G_idx[row, 0]), f"block {j} indices"
        assert np.array_equal(gv, ost.G_val[row, 0]), f"block {j} values"
        pg = params[lo:lo + L].cpu().numpy().astype(np.float64)
        tol = 1e-5 * np.maximum(np.abs(p.astype(np.float64)), w.lr)
        assert np.all(np.abs(pg - p) <= tol), f"block {j} parameters"

    # delta_2 / Delta_2 from an independent torch reduction: residual = g with
    # the window's row-1 entries zeroed (a_1 = g at t = 1).
    rows = win.view(nb, m, kp)[:, row, :kb].to(torch.int64)
    resid_min, resid_max = 0.0, 0.0
    chunk = 1 << 14
    starts = torch.tensor([s for s, _ in spans], dtype=torch.int64, device=dev)
    for b0 in range(0, nb, chunk):
        b1 = min(nb, b0 + chunk)
        lo = spans[b0][0]
        hi = spans[b1 - 1][0] + spans[b1 - 1][1]
        a = grads[lo:hi].float().clone()
        idx = rows[b0:b1] & 0xFFFF
        valid = idx != 0xFFFF
        flat = (idx + (starts[b0:b1] - lo).unsqueeze(1))[valid]
        a[flat] = 0.0
        resid_min = min(resid_min, float(a.min()))
        resid_max = max(resid_max, float(a.max()))
    lo2, hi2 = state_view.header_scalars(state[:32].cpu().numpy(), 2)
    assert np.float32(lo2) == np.float32(resid_min) + np.float32(0.0)
    assert np.float32(hi2) == np.float32(resid_max) + np.float32(0.0)

    codes = state[lay.codes: lay.codes + (d + 1) // 2]
    for j in sample:
        lo, L = spans[j]
        g = workloads.bf16_bits(grads[lo:lo + L])
        ost = oracle.new_state(L, Bd, kb, m)
        oracle.step(ost, np.zeros(L, np.float32), g, t=1, **hyper)
        a = (g.astype(np.uint32) << 16).view(np.float32).copy()  # a_1 = g
        sel = ost.G_idx[row, 0]
        a[sel[sel >= 0].astype(np.int64)] = 0.0
        want = oracle.quantize(a, float(lo2), float(hi2), t=1, seed=w.seed, base=lo)
        got = codes[lo // 2: lo // 2 + want.size].cpu().numpy()
        if L % 2:
            got = got.copy()
            got[-1] &= 0x0F
        assert np.array_equal(got, want), f"block {j} codes"


def test_llama2_7b_step1_sampled_blocks():
    from compressed_state_optimizer_b200 import workloads
    check_step1_sampled(workloads.llama2_7b(), need_bytes=75e9)


@pytest.mark.parametrize("name", ["flat_134m", "bert_base_2048", "bert_base_8192",
                                  "bert_base_32766", "bert_base_2048_per_tensor"])
def test_workload_step1_sampled_blocks(name):
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    check_step1_sampled(bench.get_workload(name), n_random=40)
