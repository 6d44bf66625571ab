"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, step by
step, on the same seeded inputs.

Bit-exact: the window rows (int16 I, bf16 V; each row as a set of pairs, put
in ascending index order), the 4-bit codes, delta/Delta and the status word.
Within 1e-5: the parameters (relative, with an absolute floor of 1e-5 * lr,
the scale of one update), v_hat (relative) and m_hat
(relative to the cancellation-free magnitude (1-b1)/(1-b1^t) sum b1^r |V|,
since m_hat sums terms of both signs).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import state_view
from conftest import cuda_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

RTOL = 1e-5


def _mods():
    import torch
    from compressed_state_optimizer_b200 import MicroAdam, workloads
    return torch, MicroAdam, workloads


def compare_state(mo, state, ost, t, d, m, kb, what=""):
    sb = state.cpu().numpy()
    lay = mo.layout
    assert np.array_equal(state_view.codes(sb, lay, d), ost.codes), f"codes differ {what} t={t}"
    lo, hi = state_view.header_scalars(sb, t + 1)
    assert np.float32(lo).view(np.uint32) == ost.scal[0:1].view(np.uint32)[0], (what, t, lo, ost.scal)
    assert np.float32(hi).view(np.uint32) == ost.scal[1:2].view(np.uint32)[0], (what, t, hi, ost.scal)
    gi, gv = state_view.canonical_rows(*state_view.window(sb, lay, m, kb))
    for s in range(max(1, t - m + 1), t + 1):
        r = s % m
        assert np.array_equal(gi[r], ost.G_idx[r]), f"window indices differ {what} t={t} row step {s}"
        assert np.array_equal(gv[r], ost.G_val[r]), f"window values differ {what} t={t} row step {s}"
    return sb


def compare_params(p_gpu, p_ref, lr, what=""):
    p = p_gpu.cpu().numpy()
    err = np.abs(p.astype(np.float64) - p_ref.astype(np.float64))
    tol = RTOL * np.maximum(np.abs(p_ref.astype(np.float64)), lr)
    bad = np.flatnonzero(err > tol)
    assert bad.size == 0, f"params differ {what} at {bad[:5]}: {p[bad[:5]]} vs {p_ref[bad[:5]]}"


def compare_stats(mhat, vhat, stats, what=""):
    mh_ref, vh_ref, mabs = stats
    mh = mhat.cpu().numpy().astype(np.float64)
    vh = vhat.cpu().numpy().astype(np.float64)
    touched = mabs > 0
    assert np.all(mh[~touched] == 0) and np.all(vh[~touched] == 0), what
    assert np.all(np.abs(mh - mh_ref) <= RTOL * mabs + 1e-30), what
    assert np.all(np.abs(vh - vh_ref) <= RTOL * vh_ref + 1e-30), what


def run_parity(d, Bd, kb, m, steps, *, kind="normal", seed=0x1234, lr=1e-3, b1=0.9,
               b2=0.999, eps=1e-8, wd=0.0, grads_fn=None, stats=True, use_step=False,
               segments=None):
    torch, MicroAdam, workloads = _mods()
    w = workloads.Workload("parity", d, Bd, kb, m, kind, steps, seed=seed)
    p0 = workloads.make_params(d, seed=7)
    mo = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m, segments=segments)
    state = mo.new_state("cuda")
    p_gpu = p0.cuda()
    ost = oracle.new_state(d, Bd, kb, m, segments=segments)
    p_ref = p0.numpy().copy()
    hyper = dict(lr=lr, beta1=b1, beta2=b2, eps=eps, wd=wd)
    for t in range(1, steps + 1):
        g = grads_fn(t) if grads_fn else workloads.make_grads(w, t)
        g_gpu = g.cuda()
        if use_step:
            mo.step(p_gpu, g_gpu, state, t=t, seed=seed, **hyper)
        else:
            mhat = torch.zeros(d, device="cuda") if stats else None
            vhat = torch.zeros(d, device="cuda") if stats else None
            mo.select(p_gpu, g_gpu, state, t=t, seed=seed, mhat=mhat, vhat=vhat, **hyper)
            mo.apply(p_gpu, g_gpu, state, t=t, seed=seed, mhat=mhat, vhat=vhat, **hyper)
        res = oracle.step(ost, p_ref, workloads.bf16_bits(g), t=t, seed=seed,
                          want_stats=stats and not use_step, **hyper)
        torch.cuda.synchronize()
        what = f"(d={d} Bd={Bd} kb={kb} m={m})"
        compare_state(mo, state, ost, t, d, m, kb, what)
        compare_params(p_gpu, p_ref, lr, what + f" t={t}")
        if stats and not use_step:
            compare_stats(mhat, vhat, res, what + f" t={t}")
    return mo, state, p_gpu


def test_flat_2p20_twenty_steps():
    """d = 2^20, N(0,1) bf16 gradients, B_d = 16384, k_b = 164, m = 10, 20 steps."""
    run_parity(1 << 20, 16384, 164, 10, 20)


def test_flat_2p20_through_mua_step():
    """The production entry point (mua_step) gives the same state as select+apply."""
    run_parity(1 << 20, 16384, 164, 10, 12, use_step=True, kind="t3")


@pytest.mark.parametrize("d,Bd,kb,m,steps,kind", [
    (5 * 2048 + 777, 2048, 21, 3, 8, "t3"),          # ragged odd-length last block
    (3 * 8192 + 8, 8192, 82, 10, 12, "normal"),
    (4 * 1022 + 301, 1022, 11, 4, 8, "normal"),      # B_d % 8 != 0: scalar path
    (2 * 32766 + 1000, 32766, 328, 2, 4, "t3"),      # largest block, 1024 threads
    (1000, 16384, 164, 10, 6, "normal"),             # d < B_d: one partial block
    (1, 2, 1, 1, 4, "normal"),                       # d = 1
    (37, 8, 1, 1, 6, "normal"),                      # k_b = 1, m = 1, tiny blocks
    (3 * 16384, 16384, 164, 37, 40, "normal"),       # m = 37 (the m_max bound)
    (64 * 33, 64, 64, 12, 12, "normal"),             # k_b = B_d: every entry kept
    (2 * 16384 + 3000, 16384, 1536, 10, 12, "t3"),   # largest window: m * kp = 15360
    (2 * 16384 + 100, 16384, 164, 20, 22, "normal"),  # apply smem just under 48 KB
])
def test_shapes(d, Bd, kb, m, steps, kind):
    run_parity(d, Bd, kb, m, steps, kind=kind)


def test_weight_decay():
    run_parity(9 * 4096 + 100, 4096, 41, 5, 6, wd=0.1, lr=1e-2)


def test_ties_and_zero_blocks():
    """Heavy ties (few distinct magnitudes) and an all-zero block."""
    torch, _, workloads = _mods()
    d, Bd = 6 * 1024, 1024
    rng = np.random.default_rng(3)

    def grads(t):
        x = rng.choice([-2.0, -1.0, -0.5, 0.5, 1.0, 2.0], d).astype(np.float32)
        x[Bd:2 * Bd] = 0.0
        x[3 * Bd:4 * Bd] = 1.0
        return workloads.grads_from_values(x)

    run_parity(d, Bd, 11, 4, 8, grads_fn=grads)


def test_one_signed_blocks():
    """Blocks whose values lie on one side of zero (all positive, all negative)
    beside mixed ones. The select kernel takes a block's residual min and max
    from the candidates it did not select when they reach past every lane's
    threshold; in a one-signed block one side does not, and its extra pass over
    the block's unselected elements decides it."""
    torch, _, workloads = _mods()
    Bd = 16384
    d = 6 * Bd + 4000
    rng = np.random.default_rng(5)

    def grads(t):
        x = np.abs(rng.standard_normal(d)).astype(np.float32)
        x[Bd:2 * Bd] *= -1.0                            # all negative
        x[3 * Bd:4 * Bd] = rng.standard_normal(Bd)      # mixed
        x[5 * Bd:] *= 1e-3                              # small, positive, ragged tail
        return workloads.grads_from_values(x)

    run_parity(d, Bd, 164, 4, 6, grads_fn=grads)


@pytest.mark.parametrize("d,Bd,kb,m,steps,kind,wd", [
    (1 << 20, 16384, 164, 10, 20, "normal", 0.0),      # the 2^20 vector, 20 steps
    (5 * 2048 + 777, 2048, 21, 3, 8, "t3", 0.0),       # ragged odd-length last block
    (4 * 1022 + 301, 1022, 11, 4, 8, "normal", 0.0),   # B_d % 8 != 0: scalar path
    (9 * 4096 + 100, 4096, 41, 5, 6, "t3", 0.1),       # weight decay
    (3 * 16384, 16384, 164, 37, 40, "normal", 0.0),    # m = 37
])
def test_fused_step(d, Bd, kb, m, steps, kind, wd):
    """mua_step as ONE launch (blocks fit the device at once) against the oracle,
    every step."""
    torch, MicroAdam, _ = _mods()
    assert MicroAdam(d, block_size=Bd, k_per_block=kb, window=m).step_launches() == 1
    run_parity(d, Bd, kb, m, steps, kind=kind, use_step=True, wd=wd,
               lr=1e-2 if wd else 1e-3)


def test_fused_equals_two_kernels():
    """The fused step and select + apply give the same bytes, step after step
    (the window rows as sets of pairs: the two paths list a row in different
    orders)."""
    torch, MicroAdam, workloads = _mods()
    d, Bd, kb, m = 7 * 16384 + 4000, 16384, 164, 5
    w = workloads.Workload("pair", d, Bd, kb, m, "t3", 12, seed=4)
    hyper = dict(lr=1e-3, beta1=.9, beta2=.999, eps=1e-8, wd=0., seed=21)
    mo = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m)
    assert mo.step_launches() == 1
    sa, sb = mo.new_state(), mo.new_state()
    pa = workloads.make_params(d).cuda()
    pb = pa.clone()
    for t in range(1, 13):
        g = workloads.make_grads(w, t).cuda()
        mo.step(pa, g, sa, t=t, **hyper)
        mo.select(pb, g, sb, t=t, **hyper)
        mo.apply(pb, g, sb, t=t, **hyper)
        torch.cuda.synchronize()
        lay = mo.layout
        assert torch.equal(sa[:20], sb[:20]), t
        assert torch.equal(sa[lay.codes:lay.window], sb[lay.codes:lay.window]), t
        assert state_view.same_window_sets(sa.cpu().numpy(), sb.cpu().numpy(), lay), t
        assert torch.equal(pa, pb), t


def test_fused_barrier_timeout_sets_status():
    """A CTA that waits longer than the limit at the fused step's grid barrier
    sets MUA_STATUS_TIMEOUT and returns; the kernel ends, the context stays
    usable and a fresh state then steps normally."""
    torch, MicroAdam, workloads = _mods()
    from compressed_state_optimizer_b200.binding import MUA_STATUS_TIMEOUT
    d, Bd, kb, m = 32 * 16384, 16384, 164, 4
    w = workloads.Workload("timeout", d, Bd, kb, m, "normal", 5, seed=6)
    hyper = dict(lr=1e-3, beta1=.9, beta2=.999, eps=1e-8, wd=0., seed=3)
    mo = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m)
    assert mo.step_launches() == 1
    mo.set_wait_limit_ns(0)  # give up at once
    state = mo.new_state()
    p = workloads.make_params(d).cuda()
    for t in range(1, 6):
        mo.step(p, workloads.make_grads(w, t).cuda(), state, t=t, **hyper)
    torch.cuda.synchronize()
    assert mo.status(state) & MUA_STATUS_TIMEOUT
    mo.set_wait_limit_ns(2_000_000_000)
    run_parity(d, Bd, kb, m, 3, use_step=True)


def run_parity_bf16(d, Bd, kb, m, steps, *, kind="t3", seed=0x77, lr=1e-3, wd=0.0,
                    use_step=True, segments=None):
    """bf16 parameters against the oracle's bf16-parameter step. Each step the
    oracle starts from the GPU's parameters; the window rows, codes and
    delta/Delta must agree bit for bit. The kernel forms each new parameter in
    fp32, the oracle in fp64, so the GPU's bf16 value must lie within half a
    bf16 step of the oracle's exact value plus the fp32 tolerance of the fp32
    tests, 1e-5 * max(|exact|, lr): away from cancellation that admits the
    nearest-even value only, or its neighbour where the exact value is within
    1e-5 of a rounding midpoint; where p*(1 - lr*wd) and lr*u nearly cancel,
    the fp32 rounding of the two terms (about 1e-9 at lr = 1e-2) can exceed a
    bf16 step of the tiny result, and the absolute floor admits that."""
    torch, MicroAdam, workloads = _mods()
    w = workloads.Workload("bf16", d, Bd, kb, m, kind, steps, seed=seed)
    mo = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m, segments=segments)
    state = mo.new_state("cuda")
    p_gpu = workloads.make_params(d, seed=7).to(torch.bfloat16).cuda()
    ost = oracle.new_state(d, Bd, kb, m, segments=segments)
    hyper = dict(lr=lr, beta1=0.9, beta2=0.999, eps=1e-8, wd=wd)
    exact = np.zeros(d, dtype=np.float64)
    changed = 0
    for t in range(1, steps + 1):
        g = workloads.make_grads(w, t)
        p_ref = workloads.bf16_bits(p_gpu)
        before = p_ref.copy()
        if use_step:
            mo.step(p_gpu, g.cuda(), state, t=t, seed=seed, **hyper)
        else:
            mo.select(p_gpu, g.cuda(), state, t=t, seed=seed, **hyper)
            mo.apply(p_gpu, g.cuda(), state, t=t, seed=seed, **hyper)
        oracle.step(ost, p_ref, workloads.bf16_bits(g), t=t, seed=seed, p_exact=exact, **hyper)
        torch.cuda.synchronize()
        compare_state(mo, state, ost, t, d, m, kb, f"(bf16 params d={d})")
        got = workloads.bf16_bits(p_gpu)
        gf = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        nxt = ((got.astype(np.uint32) + 1) << 16).view(np.float32).astype(np.float64)
        half_ulp = np.abs(nxt - gf) / 2
        bound = half_ulp + RTOL * np.maximum(np.abs(exact), lr)
        bad = np.flatnonzero(np.abs(gf - exact) > bound)
        assert bad.size == 0, (t, bad[:5], got[bad[:5]], p_ref[bad[:5]], exact[bad[:5]])
        changed += int(np.count_nonzero(got != before))
    assert changed > 0


@pytest.mark.parametrize("d,Bd,kb,m,steps,kind,wd,use_step", [
    (1 << 20, 16384, 164, 10, 12, "normal", 0.0, True),     # fused one-launch step
    (1 << 20, 16384, 164, 10, 8, "t3", 0.1, False),         # select + apply, weight decay
    (5 * 2048 + 777, 2048, 21, 3, 6, "t3", 0.05, True),     # ragged
    (4 * 1022 + 302, 1022, 11, 4, 6, "normal", 0.0, False),  # B_d % 8 != 0: scalar path
])
def test_bf16_params(d, Bd, kb, m, steps, kind, wd, use_step):
    run_parity_bf16(d, Bd, kb, m, steps, kind=kind, wd=wd, use_step=use_step,
                    lr=1e-2 if wd else 1e-3)


def test_bf16_params_segmented():
    segs = [3 * 4096 + 64, 512, 4096]
    run_parity_bf16(sum(segs), 4096, 41, 5, 6, segments=segs, wd=0.05, lr=1e-2)


def test_adam_reduction_on_gpu():
    """k_b = B_d, m >= T: the GPU step is Adam; the residual stays exactly 0."""
    mo, state, _ = run_parity(4 * 250 + 16, 250 + 6, 256, 8, 8, lr=1e-2)
    sb = state.cpu().numpy()
    assert not state_view.codes(sb, mo.layout, mo.d).any()


def test_nonfinite_sets_status():
    torch, MicroAdam, workloads = _mods()
    d = 4096
    mo = MicroAdam(d, block_size=1024, k_per_block=11, window=2)
    state = mo.new_state()
    p = workloads.make_params(d).cuda()
    g = torch.zeros(d, dtype=torch.bfloat16, device="cuda")
    mo.step(p, g, state, lr=1e-3, beta1=.9, beta2=.999, eps=1e-8, wd=0., t=1, seed=1)
    assert mo.status(state) == 0
    g[1234] = float("nan")
    mo.step(p, g, state, lr=1e-3, beta1=.9, beta2=.999, eps=1e-8, wd=0., t=2, seed=1)
    assert mo.status(state) & 1
    g[1234] = float("inf")
    mo.step(p, g, state, lr=1e-3, beta1=.9, beta2=.999, eps=1e-8, wd=0., t=3, seed=1)
    assert mo.status(state) & 1


def test_deterministic_and_resumable():
    """Two runs give identical bytes; a run saved after 5 steps and resumed from
    a copy of its state matches the uninterrupted run bit for bit."""
    torch, MicroAdam, workloads = _mods()
    d, Bd, kb, m = 5 * 16384 + 3000, 16384, 164, 4
    w = workloads.Workload("det", d, Bd, kb, m, "t3", 10)
    hyper = dict(lr=1e-3, beta1=.9, beta2=.999, eps=1e-8, wd=0.)

    def run(n, state=None, p=None, t0=1):
        mo = MicroAdam(d, block_size=Bd, k_per_block=kb, window=m)
        state = mo.new_state() if state is None else state
        p = workloads.make_params(d).cuda() if p is None else p
        for t in range(t0, t0 + n):
            mo.step(p, workloads.make_grads(w, t).cuda(), state, t=t, seed=9, **hyper)
        torch.cuda.synchronize()
        return state, p

    s1, p1 = run(10)
    s2, p2 = run(10)
    assert torch.equal(s1, s2) and torch.equal(p1, p2)
    s3, p3 = run(5)
    saved_s, saved_p = s3.cpu().clone(), p3.cpu().clone()
    s4, p4 = run(5, saved_s.cuda(), saved_p.cuda(), t0=6)
    assert torch.equal(s4, s1) and torch.equal(p4, p1)


def _structured_grads(d, Bd, seed):
    """Blocks built to drive the select kernel through each of its paths.

    Block j % 4 == 0: the large values sit only on the 512 elements the
    threshold sample reads (64 runs of 8 at stride 256), so the first
    candidate pass finds too few entries; 1: all large values on one
    lane's elements (elements 40..47 of every 256), so that lane holds the
    whole Top-k; 2: plain; 3: one lane's elements 30 % larger than the rest
    (that lane's region tends to fill). The oracle decides what is right."""
    import torch

    def fn(t):
        rng = np.random.default_rng(seed + t)
        g = (rng.standard_normal(d) * 0.01).astype(np.float32)
        steps = np.arange(64)[:, None] * 256
        for j in range(d // Bd):
            base = j * Bd
            if j % 4 == 0:
                pos = (steps + np.arange(8)).ravel()
                g[base + pos] = rng.standard_normal(pos.size)
            elif j % 4 == 1:
                pos = (steps + 40 + np.arange(8)).ravel()
                g[base + pos] = rng.standard_normal(pos.size)
            elif j % 4 == 3:
                pos = (steps + 24 + np.arange(8)).ravel()
                g[base + pos] *= 1.3
        return torch.from_numpy(g).to(torch.bfloat16)
    return fn


@pytest.mark.parametrize("kb", [164, 600])
def test_select_paths(kb):
    d, Bd = 8 * 16384 + 999, 16384
    run_parity(d, Bd, kb, 3, 4, grads_fn=_structured_grads(d, Bd, 99 + kb))


SEGMENTED = [
    # (B_d, k_b, m, steps, tensor lengths, kind)
    (16384, 164, 4, 8, [2 * 16384 + 1000, 8000, 16384, 4096 + 8, 30000], "t3"),
    (2048, 21, 3, 6, [5000, 2, 2048, 3070, 6], "normal"),  # lengths not all 8k: scalar path
    (8192, 82, 10, 12, [8192 * 3, 4104, 9000, 1000], "t3"),
]


@pytest.mark.parametrize("Bd,kb,m,steps,segs,kind", SEGMENTED)
def test_segmented(Bd, kb, m, steps, segs, kind):
    """A tensor list cut per tensor (each tensor's last block ragged) against the
    oracle's per-tensor cut."""
    run_parity(sum(segs), Bd, kb, m, steps, kind=kind, segments=segs)


def test_segmented_step():
    segs = [3 * 4096 + 64, 512, 4096]
    run_parity(sum(segs), 4096, 41, 5, 8, kind="t3", segments=segs, use_step=True, wd=0.05)
