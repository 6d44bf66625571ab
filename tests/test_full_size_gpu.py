"""Full-size parity on the LLaMA-2-7B-shaped vector (d = 6,738,415,616), in the
launch configuration bench.py times, on outputs the oracle can compute one
block at a time.

Step 1 starts from the zero state, so every block is independent of the others
except through delta_2 / Delta_2:
  * sampled blocks: the window row and the parameter update equal the oracle
    run on that block alone (bit for bit / 1e-5);
  * delta_2, Delta_2: the min and max of the residual over the whole vector,
    computed independently with torch reductions from the gradients and the
    (row-verified) selection;
  * sampled blocks' codes equal the oracle's quantizer applied with the
    verified delta_2, Delta_2.
Needs about 70 GB of device memory and a few minutes; skipped on smaller GPUs.
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


def test_llama2_7b_step1_sampled_blocks():
    import torch
    from compressed_state_optimizer_b200 import MicroAdam, workloads
    if _free_bytes() < 75e9:
        pytest.skip("needs ~75 GB of free device memory")
    w = workloads.llama2_7b()
    d, Bd, kb, m = w.d, w.Bd, w.kb, w.m
    mo = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m)
    dev = torch.device("cuda", 0)
    params = workloads.make_params(d, seed=7, device=dev)
    grads = workloads.make_grads(w, 1, device=dev)
    nb = mo.layout.blocks
    rng = np.random.default_rng(11)
    sample = sorted(set([0, 1, nb // 2, nb - 2, nb - 1] + list(rng.integers(0, nb, 27))))
    p0 = {j: params[j * Bd: min(d, (j + 1) * Bd)].cpu().numpy().copy() for j in sample}
    state = mo.new_state(dev)
    hyper = dict(lr=w.lr, beta1=w.beta1, beta2=w.beta2, eps=w.eps, wd=w.wd, seed=w.seed)
    mo.step(params, grads, state, t=1, **hyper)
    torch.cuda.synchronize()

    lay = mo.layout
    kp = lay.row_stride
    win = state[lay.window: lay.bytes].view(torch.int32)
    row = 1 % m
    for j in sample:
        lo, hi = j * Bd, min(d, (j + 1) * Bd)
        g = workloads.bf16_bits(grads[lo:hi])
        ost = oracle.new_state(hi - lo, Bd, kb, m)
        p = p0[j].copy()
        oracle.step(ost, p, g, t=1, **hyper)
        gw = win[(j * m + row) * kp: (j * m + row) * kp + kb].cpu().numpy().view(np.uint32)
        gi = (gw & 0xFFFF).astype(np.uint16).view(np.int16)
        gv = (gw >> 16).astype(np.uint16)
        assert np.array_equal(gi, ost.G_idx[row, 0]), f"block {j} indices"
        assert np.array_equal(gv, ost.G_val[row, 0]), f"block {j} values"
        pg = params[lo:hi].cpu().numpy().astype(np.float64)
        tol = 1e-5 * np.maximum(np.abs(p.astype(np.float64)), w.lr)
        assert np.all(np.abs(pg - p) <= tol), f"block {j} parameters"

    # delta_2 / Delta_2 from an independent torch reduction: residual = g with
    # the window's row-1 entries zeroed (a_1 = g at t = 1).
    resid_min, resid_max = 0.0, 0.0
    chunk_blocks = 1 << 14
    for b0 in range(0, nb, chunk_blocks):
        b1 = min(nb, b0 + chunk_blocks)
        lo, hi = b0 * Bd, min(d, b1 * Bd)
        a = grads[lo:hi].float().clone()
        rows = win.view(nb, m, kp)[b0:b1, row, :kb].to(torch.int64)
        idx = rows & 0xFFFF
        valid = idx != 0xFFFF
        flat = (idx + (torch.arange(b0, b1, device=dev, dtype=torch.int64) * Bd
                       - lo).unsqueeze(1))[valid]
        a[flat] = 0.0
        resid_min = min(resid_min, float(a.min()))
        resid_max = max(resid_max, float(a.max()))
    lo2, hi2 = state_view.header_scalars(state[:32].cpu().numpy(), 2)
    assert np.float32(lo2) == np.float32(resid_min) + np.float32(0.0)
    assert np.float32(hi2) == np.float32(resid_max) + np.float32(0.0)

    codes = state[lay.codes: lay.codes + (d + 1) // 2]
    for j in sample:
        lo, hi = j * Bd, min(d, (j + 1) * Bd)
        g = workloads.bf16_bits(grads[lo:hi])
        ost = oracle.new_state(hi - lo, Bd, kb, m)
        oracle.step(ost, np.zeros(hi - lo, np.float32), g, t=1, **hyper)
        a = (g.astype(np.uint32) << 16).view(np.float32).copy()  # a_1 = g
        sel = ost.G_idx[row, 0]
        a[sel[sel >= 0].astype(np.int64)] = 0.0
        want = oracle.quantize(a, float(lo2), float(hi2), t=1, seed=w.seed, base=lo)
        got = codes[lo // 2: lo // 2 + want.size].cpu().numpy()
        if (hi - lo) % 2:
            got = got.copy()
            got[-1] &= 0x0F
        assert np.array_equal(got, want), f"block {j} codes"
