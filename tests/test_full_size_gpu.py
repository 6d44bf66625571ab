"""Full-size parity on the benchmark workloads, in the launch configuration
bench.py times, over several steps (the window fills at t = m), on outputs the
oracle can compute one block at a time.

Blocks depend on each other only through delta_t / Delta_t. Before each
step, a sample of blocks' state is read back from the device (codes, all
window rows, parameters) with the global (delta_t, Delta_t); then:
  * each sampled block's new window row (as a set of pairs) and updated
    parameters equal the oracle run on that block alone from that state (bit
    for bit / 1e-5);
  * delta_{t+1}, Delta_{t+1}: the min and max of the residual over the whole
    vector, computed independently with torch from the gradients, a device
    copy of the previous codes and the (row-verified) selection;
  * each sampled block's new codes equal the oracle's quantizer applied to
    its residual with the verified delta_{t+1}, Delta_{t+1}.
The LLaMA-2-7B-shaped case needs about 75 GB of device memory.
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


def check_steps_sampled(w, steps, n_random=27, need_bytes=0):
    import torch
    from compressed_state_optimizer_b200 import MicroAdam, workloads
    if _free_bytes() < need_bytes:
        pytest.skip(f"needs {need_bytes / 1e9:.0f} GB of free device memory")
    d, Bd, kb, m = w.d, w.Bd, w.kb, w.m
    mo = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m, segments=w.segments())
    dev = torch.device("cuda", 0)
    params = workloads.make_params(d, seed=7, device=dev)
    nb = mo.layout.blocks
    spans = _block_spans(w, nb)
    rng = np.random.default_rng(11)
    sample = sorted(set([0, 1, nb // 2, nb - 2, nb - 1] + list(rng.integers(0, nb, n_random))))
    state = mo.new_state(dev)
    hyper = dict(lr=w.lr, beta1=w.beta1, beta2=w.beta2, eps=w.eps, wd=w.wd, seed=w.seed)
    lay = mo.layout
    kp = lay.row_stride
    win = state[lay.window: lay.bytes].view(torch.int32)
    codes = state[lay.codes: lay.codes + (d + 1) // 2]
    starts = torch.tensor([s for s, _ in spans], dtype=torch.int64, device=dev)

    for t in range(1, steps + 1):
        grads = workloads.make_grads(w, t, device=dev)
        # ---- the state before the step
        d0, D0 = state_view.header_scalars(state[:32].cpu().numpy(), t)
        codes_before = codes.clone()
        before = {}
        for j in sample:
            lo, L = spans[j]
            rows = win[j * m * kp: (j + 1) * m * kp].cpu().numpy().view(np.uint32)
            rows = rows.reshape(m, kp)[:, :kb]
            before[j] = dict(
                p=params[lo:lo + L].cpu().numpy().copy(),
                codes=codes[lo // 2: lo // 2 + (L + 1) // 2].cpu().numpy().copy(),
                idx=(rows & 0xFFFF).astype(np.uint16).view(np.int16).reshape(m, 1, kb).copy(),
                val=(rows >> 16).astype(np.uint16).reshape(m, 1, kb).copy())
        mo.step(params, grads, state, t=t, **hyper)
        torch.cuda.synchronize()
        row = t % m

        # ---- sampled blocks: new row and parameters against the oracle
        resid = {}
        for j in sample:
            lo, L = spans[j]
            b = before[j]
            g = workloads.bf16_bits(grads[lo:lo + L])
            ost = oracle.new_state(L, Bd, kb, m)
            ost.codes[:] = b["codes"]
            if L % 2:
                ost.codes[-1] &= 0x0F
            ost.scal[:] = (d0, D0)
            ost.G_idx[:] = b["idx"]
            ost.G_val[:] = b["val"]
            p = b["p"].copy()
            oracle.step(ost, p, g, t=t, **hyper)
            gw = win[(j * m + row) * kp: (j * m + row) * kp + kb].cpu().numpy().view(np.uint32)
            gi, gv = state_view.canonical_words(gw)
            assert np.array_equal(gi, ost.G_idx[row, 0]), f"t={t} block {j} indices"
            assert np.array_equal(gv, ost.G_val[row, 0]), f"t={t} block {j} values"
            pg = params[lo:lo + L].cpu().numpy().astype(np.float64)
            tol = 1e-5 * np.maximum(np.abs(p.astype(np.float64)), w.lr)
            assert np.all(np.abs(pg - p) <= tol), f"t={t} block {j} parameters"
            # the block's residual: a_t = f32(g) + Q^{-1}(e_t), selected entries zeroed
            a = (g.astype(np.uint32) << 16).view(np.float32) + oracle.dequantize(
                b["codes"], L, float(d0), float(D0))
            sel = ost.G_idx[row, 0]
            a[sel[sel >= 0].astype(np.int64)] = 0.0
            resid[j] = a

        # ---- delta_{t+1}, Delta_{t+1} by an independent torch reduction
        u = np.float32(np.float32(D0) - np.float32(d0)) / np.float32(15.0)
        lv = torch.tensor(np.float32(d0) + np.arange(16, dtype=np.float32) * u, device=dev)
        rows_t = win.view(nb, m, kp)[:, row, :kb].to(torch.int64)
        resid_min, resid_max = 0.0, 0.0
        chunk = 1 << 14
        for b0 in range(0, nb, chunk):
            b1 = min(nb, b0 + chunk)
            lo = spans[b0][0]
            hi = spans[b1 - 1][0] + spans[b1 - 1][1]
            cb = codes_before[lo // 2: (hi + 1) // 2]
            nib = torch.stack([cb & 0xF, cb >> 4], dim=1).reshape(-1)[: hi - lo].to(torch.int64)
            a = grads[lo:hi].float() + lv[nib]
            idx = rows_t[b0:b1] & 0xFFFF
            valid = idx != 0xFFFF
            flat = (idx + (starts[b0:b1] - lo).unsqueeze(1))[valid]
            a[flat] = 0.0
            resid_min = min(resid_min, float(a.min()))
            resid_max = max(resid_max, float(a.max()))
        lo2, hi2 = state_view.header_scalars(state[:32].cpu().numpy(), t + 1)
        assert np.float32(lo2) == np.float32(resid_min) + np.float32(0.0), t
        assert np.float32(hi2) == np.float32(resid_max) + np.float32(0.0), t

        # ---- sampled blocks' new codes under the verified delta_{t+1}, Delta_{t+1}
        for j in sample:
            lo, L = spans[j]
            want = oracle.quantize(resid[j], float(lo2), float(hi2), t=t, seed=w.seed, base=lo)
            got = codes[lo // 2: lo // 2 + want.size].cpu().numpy()
            if L % 2:
                got = got.copy()
                got[-1] &= 0x0F
            assert np.array_equal(got, want), f"t={t} block {j} codes"
        del grads, codes_before


def test_llama2_7b_sampled_blocks_through_full_window():
    """The LLaMA-2-7B shape for t = 1 .. m + 2 (the window fills and wraps)."""
    from compressed_state_optimizer_b200 import workloads
    w = workloads.llama2_7b()
    check_steps_sampled(w, w.m + 2, need_bytes=75e9)


@pytest.mark.parametrize("name", ["flat_134m", "bert_base_2048", "bert_base_8192",
                                  "bert_base_32766", "bert_base_2048_per_tensor",
                                  "flat_1m"])
def test_workload_sampled_blocks(name):
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    w = bench.get_workload(name)
    check_steps_sampled(w, 4 if w.d > (1 << 24) else w.m + 2, n_random=40)
