"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each ``check_*`` function raises AssertionError when the oracle disagrees with
what the page, the mathematics or an independent library fixes. The functions
take no arguments (or only sizes) and call whatever oracle library is loaded,
so that ``test_oracle_mutants.py`` can run them against deliberately broken
oracle builds and confirm that every planted mistake is caught.

[MicroAdam ¶n] is paragraph n of "MicroAdam (Sparse-Gradient Adaptive
Optimization with Quantized Error Feedback)".
"""
from __future__ import annotations

import functools
import math
import os
import subprocess
import tempfile

import numpy as np
import torch

import oracle
from compressed_state_optimizer_b200 import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


# --------------------------------------------------------------- helpers
def f32_of_bits(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_bits_of(values) -> np.ndarray:
    return workloads.bf16_bits(workloads.grads_from_values(values))


def normal_bf16(n: int, seed: int, scale: float = 1.0) -> np.ndarray:
    g = np.random.default_rng(seed).standard_normal(n).astype(np.float32) * np.float32(scale)
    return bf16_bits_of(g)


def topk_rows_numpy(a: np.ndarray, Bd: int, kb: int):
    """Per block: the indices numpy's stable argsort ranks first by |a| (desc)."""
    rows = []
    for s in range(0, a.size, Bd):
        blk = a[s:s + Bd]
        k = -(-blk.size * kb // Bd)
        order = np.argsort(-np.abs(blk.astype(np.float64)), kind="stable")[:k]
        rows.append(np.sort(order))
    return rows


@functools.lru_cache(maxsize=1)
def _torch_philox_binary() -> str:
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    out = os.path.join(tempfile.mkdtemp(prefix="philox_ref_"), "philox_ref")
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", inc,
                    os.path.join(HERE, "philox_torch_ref.cpp"), "-o", out], check=True)
    return out


def torch_philox(triples) -> np.ndarray:
    """PyTorch's Philox4x32-10 for (seed, subsequence, offset) triples."""
    text = "".join(f"{s} {u} {o}\n" for s, u, o in triples)
    res = subprocess.run([_torch_philox_binary()], input=text, capture_output=True,
                         text=True, check=True)
    return np.array([[int(x) for x in line.split()] for line in res.stdout.splitlines()],
                    dtype=np.uint64).astype(np.uint32)


# --------------------------------------------------------------- Philox
def check_philox_vs_torch(n: int = 512):
    """Oracle Philox4x32-10 == PyTorch's independent engine, word for word."""
    rng = np.random.default_rng(1234)
    words = rng.integers(0, 2**32, size=(n, 6), dtype=np.uint64)
    words[:4] = 0                        # all-zero counter and key
    words[4:8] = 2**32 - 1               # all-ones
    triples, mine = [], []
    for w in words:
        c = [int(x) for x in w[:4]]
        k = [int(x) for x in w[4:]]
        seed = k[0] | (k[1] << 32)
        off = c[0] | (c[1] << 32)
        sub = c[2] | (c[3] << 32)
        triples.append((seed, sub, off))
        mine.append(oracle.philox4x32_10(c, k))
    ref = torch_philox(triples)
    assert np.array_equal(np.array(mine, dtype=np.uint32), ref), "Philox differs from PyTorch's"


def check_draw16_mapping():
    """Element i at step t uses half (i mod 2) of word (i/2 mod 4) of Philox(seed; i/8, t)."""
    seed, t = 0x0123456789ABCDEF, 77
    for i in [0, 1, 2, 3, 6, 7, 8, 15, 2**33 + 5]:
        j = i >> 3
        out = torch_philox([(seed, t, j)])[0]
        word = int(out[(i >> 1) & 3])
        want = (word >> 16) if (i & 1) else (word & 0xFFFF)
        assert oracle.draw16(seed, t, i) == want, i


def check_draw16_uniform():
    """The 16-bit draws are uniform: chi-square over 256 bins of each byte."""
    from scipy import stats
    n = 1 << 16
    x = np.array([oracle.draw16(99, 3, i) for i in range(n)], dtype=np.uint32)
    for part in (x >> 8, x & 0xFF):
        counts = np.bincount(part, minlength=256)
        p = stats.chisquare(counts).pvalue
        assert p > 1e-4, p


# --------------------------------------------------------------- bf16
def check_bf16_rne():
    """fp32 -> bf16 rounding equals PyTorch's (nearest, ties to even)."""
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    bits[:1000] = (bits[:1000] & 0xFFFF0000) | 0x8000           # exact ties
    bits[1000:1100] = (bits[1000:1100] & 0xFFFF0000) | 0x7FFF
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    want = workloads.bf16_bits(torch.from_numpy(x.copy()).to(torch.bfloat16))
    got = np.array([oracle.f32_to_bf16(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, want)
    for h in [0x0000, 0x8000, 0x3F80, 0xBF80, 0x7F7F, 0x0001]:
        assert np.float32(oracle.bf16_to_f32(h)) == f32_of_bits(np.array([h], np.uint16))[0]


# --------------------------------------------------------------- Top-k, min/max
def _run_step1(g_bits, Bd, kb, m, seed=11):
    d = g_bits.size
    st = oracle.new_state(d, Bd, kb, m)
    p = np.zeros(d, dtype=np.float32)
    oracle.step(st, p, g_bits, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0, t=1,
                seed=seed)
    return st


def check_topk_step1():
    """[MicroAdam ¶1] At t = 1, e_0 = 0 so a = g; each block's row is numpy's stable
    arg-sort of |g| (ties to the lower index), k_j entries, ascending, V = g."""
    Bd, kb, m = 512, 6, 3
    d = 3 * Bd + 100
    cases = [normal_bf16(d, 1),
             bf16_bits_of(np.random.default_rng(2).choice([-2.0, -1.0, 1.0, 2.0], d)),
             bf16_bits_of(np.round(np.random.default_rng(3).standard_normal(d) * 4) / 4)]
    for g_bits in cases:
        st = _run_step1(g_bits, Bd, kb, m)
        a = f32_of_bits(g_bits)
        want = topk_rows_numpy(a, Bd, kb)
        for j, rows in enumerate(want):
            idx = st.G_idx[1 % m, j]
            k = rows.size
            assert k == -(-min(Bd, d - j * Bd) * kb // Bd)
            assert np.array_equal(idx[:k], rows), j
            assert np.all(idx[k:] == -1)
            V = f32_of_bits(st.G_val[1 % m, j, :k])
            assert np.array_equal(V, a[j * Bd + rows])


def check_minmax_step1():
    """[MicroAdam ¶1] delta_2, Delta_2 are numpy's min and max of the residual."""
    Bd, kb, m = 256, 5, 2
    d = 4 * Bd + 3
    g_bits = normal_bf16(d, 21)
    st = _run_step1(g_bits, Bd, kb, m)
    a = f32_of_bits(g_bits).copy()
    for j, rows in enumerate(topk_rows_numpy(a, Bd, kb)):
        a[j * Bd + rows] = 0.0
    assert st.scal[0] == np.min(a) and st.scal[1] == np.max(a)
    assert st.scal[0] <= 0.0 <= st.scal[1]


def check_topk_later_steps():
    """[MicroAdam ¶1] At every t the row is the brute-force Top-k of
    a_t = g_t + Q^{-1}(e_t) (with Q^{-1} pinned separately)."""
    Bd, kb, m = 128, 3, 4
    d = 5 * Bd + 17
    st = oracle.new_state(d, Bd, kb, m)
    p = np.zeros(d, dtype=np.float32)
    for t in range(1, 9):
        g_bits = normal_bf16(d, 100 + t)
        deq = oracle.dequantize(st.codes, d, float(st.scal[0]), float(st.scal[1]))
        a = f32_of_bits(g_bits) + deq
        oracle.step(st, p, g_bits, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0, t=t,
                    seed=5)
        for j, rows in enumerate(topk_rows_numpy(a, Bd, kb)):
            assert np.array_equal(st.G_idx[t % m, j, :rows.size], rows), (t, j)
            assert np.array_equal(st.G_val[t % m, j, :rows.size],
                                  bf16_bits_of(a[j * Bd + rows]))


# --------------------------------------------------------------- Q / Q^{-1}
def check_dequant_levels():
    """Q^{-1}(c) = delta + c (Delta - delta)/15: with delta=-3, Delta=12 the levels
    are the integers -3..12; element 2q is the low nibble of byte q."""
    codes = np.array([0x10, 0x32, 0xFE], dtype=np.uint8)
    got = oracle.dequantize(codes, 6, -3.0, 12.0)
    assert np.array_equal(got, np.array([-3, -2, -1, 0, 11, 12], dtype=np.float32) + 0.0)


def check_quant_exact_levels():
    """Values on a level quantize to that level for every draw (delta=0, Delta=15)."""
    x = np.tile(np.arange(16, dtype=np.float32), 8)
    for seed in range(20):
        codes = oracle.quantize(x, 0.0, 15.0, t=3, seed=seed)
        back = oracle.dequantize(codes, x.size, 0.0, 15.0)
        assert np.array_equal(back, x)
        assert codes[0] == 0x10 and codes[1] == 0x32           # packing order


def check_quant_error_bound():
    """|Q^{-1}(Q(x)) - x| < one level spacing u = (Delta - delta)/15, per element."""
    rng = np.random.default_rng(9)
    for trial in range(20):
        x = (rng.standard_normal(3001) * rng.uniform(1e-3, 10)).astype(np.float32)
        lo, hi = float(x.min()), float(x.max())
        back = oracle.dequantize(oracle.quantize(x, lo, hi, t=trial + 1, seed=trial), x.size,
                                 lo, hi)
        u = (hi - lo) / 15
        assert np.all(np.abs(back.astype(np.float64) - x) <= u * (1 + 1e-5))


def check_quant_unbiased():
    """[MicroAdam ¶3] Q is unbiased: over N = 4096 seeds the mean of Q^{-1}(Q(x))
    is within 5 standard errors (u / (2 sqrt N)) of x; the round-up frequency
    follows the fractional position between levels."""
    rng = np.random.default_rng(17)
    x = rng.uniform(-1.0, 2.0, size=64).astype(np.float32)
    x[0], x[1] = -1.0, 2.0
    lo, hi = -1.0, 2.0
    u = (hi - lo) / 15
    N = 4096
    acc = np.zeros(x.size, dtype=np.float64)
    for s in range(N):
        acc += oracle.dequantize(oracle.quantize(x, lo, hi, t=1, seed=s), x.size, lo, hi)
    mean = acc / N
    assert np.all(np.abs(mean - x) <= 5 * u / (2 * math.sqrt(N)) + 1e-7)


def omega(d: int, lo: float, hi: float, b: int = 4) -> float:
    """[MicroAdam ¶3, Lemma 1] omega = sqrt(d-2)/(2^b - 1) * (Delta-delta)/sqrt(Delta^2+delta^2)."""
    return math.sqrt(d - 2) / (2**b - 1) * (hi - lo) / math.sqrt(hi * hi + lo * lo)


def check_lemma1_per_realization():
    """[MicroAdam ¶3, Lemma 1] ||Q^{-1}(Q(x)) - x|| <= omega ||x|| for x whose min and
    max are delta and Delta (the two end points quantize exactly; every other
    coordinate errs by less than one level)."""
    rng = np.random.default_rng(23)
    for trial in range(200):
        d = int(rng.integers(3, 400))
        x = (rng.standard_normal(d) * rng.uniform(0.01, 5) + rng.uniform(-1, 1)).astype(np.float32)
        lo, hi = float(x.min()), float(x.max())
        back = oracle.dequantize(oracle.quantize(x, lo, hi, t=trial, seed=7 * trial), d, lo, hi)
        err = np.linalg.norm(back.astype(np.float64) - x)
        assert err <= omega(d, lo, hi) * np.linalg.norm(x.astype(np.float64)) * (1 + 1e-6)


# --------------------------------------------------------------- AdamStats
def _dense_rows(st, t):
    """The window rows as dense vectors, oldest first: (age, dense V)."""
    out = []
    for r in range(min(t, st.m) - 1, -1, -1):
        row = (t - r) % st.m
        dense = np.zeros(st.d, dtype=np.float64)
        for j in range(st.nb):
            idx = st.G_idx[row, j]
            ok = idx >= 0
            dense[j * st.Bd + idx[ok].astype(np.int64)] = f32_of_bits(st.G_val[row, j][ok])
        out.append((r, dense))
    return out


def check_adamstats_vs_dense_ema():
    """[MicroAdam ¶1] AdamStats(beta, G) equals Adam's recurrence z <- beta z + (1-beta) x
    run from zero over the densified window rows (oldest first), bias-corrected
    by 1/(1 - beta^t); likewise for v_hat with the squared rows."""
    Bd, kb, m = 256, 8, 4
    d = 2 * Bd + 37
    b1, b2 = 0.9, 0.999
    st = oracle.new_state(d, Bd, kb, m)
    p = np.zeros(d, dtype=np.float32)
    for t in range(1, 8):
        mhat, vhat, _ = oracle.step(st, p, normal_bf16(d, 300 + t), lr=1e-3, beta1=b1,
                                    beta2=b2, eps=1e-8, wd=0.0, t=t, seed=1, want_stats=True)
        B1, B2 = float(np.float32(b1)), float(np.float32(b2))
        z1 = np.zeros(d)
        z2 = np.zeros(d)
        for _, dense in _dense_rows(st, t):
            z1 = B1 * z1 + (1 - B1) * dense
            z2 = B2 * z2 + (1 - B2) * dense * dense
        np.testing.assert_allclose(mhat, z1 / (1 - B1**t), rtol=1e-12, atol=1e-300)
        np.testing.assert_allclose(vhat, z2 / (1 - B2**t), rtol=1e-12, atol=1e-300)


def check_closed_form_m1_t1():
    """m = 1, t = 1: m_hat = V, v_hat = V^2, so p <- p - lr V/(eps + |V|) on the selected
    entries and no other parameter moves."""
    Bd, kb = 64, 4
    d = 3 * Bd
    g_bits = normal_bf16(d, 41)
    p0 = np.random.default_rng(3).standard_normal(d).astype(np.float32)
    p = p0.copy()
    st = oracle.new_state(d, Bd, kb, 1)
    lr, eps = 1e-2, 1e-8
    oracle.step(st, p, g_bits, lr=lr, beta1=0.9, beta2=0.999, eps=eps, wd=0.0, t=1, seed=2)
    want = p0.astype(np.float64).copy()
    sel = np.zeros(d, bool)
    for j, rows in enumerate(topk_rows_numpy(f32_of_bits(g_bits), Bd, kb)):
        q = j * Bd + rows
        V = f32_of_bits(g_bits)[q].astype(np.float64)
        want[q] -= float(np.float32(lr)) * V / (float(np.float32(eps)) + np.abs(V))
        sel[q] = True
    assert np.array_equal(p[~sel], p0[~sel])
    np.testing.assert_allclose(p, want.astype(np.float32), rtol=0, atol=0)


def _adam_reference(g_list, p0, lr, b1, b2, eps, wd):
    p = torch.from_numpy(p0.copy()).requires_grad_(True)
    opt = (torch.optim.AdamW([p], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd) if wd
           else torch.optim.Adam([p], lr=lr, betas=(b1, b2), eps=eps))
    out = []
    for g in g_list:
        p.grad = torch.from_numpy(f32_of_bits(g).copy())
        opt.step()
        out.append(p.detach().numpy().copy())
    return out


def check_reduces_to_adam(wd: float = 0.0):
    """With k_b = B_d (every entry selected) and m >= T the residual is zero and
    MicroAdam is exactly Adam (AdamW when wd > 0) on the bf16 gradients:
    compare with torch.optim over T = 8 steps."""
    Bd = 250
    d, T = 4 * Bd, 8
    lr, b1, b2, eps = 1e-2, 0.9, 0.999, 1e-8
    p0 = (np.random.default_rng(8).standard_normal(d) * 0.02).astype(np.float32)
    grads = [normal_bf16(d, 500 + t) for t in range(1, T + 1)]
    ref = _adam_reference(grads, p0, lr, b1, b2, eps, wd)
    st = oracle.new_state(d, Bd, Bd, T)
    p = p0.copy()
    for t in range(1, T + 1):
        oracle.step(st, p, grads[t - 1], lr=lr, beta1=b1, beta2=b2, eps=eps, wd=wd, t=t, seed=3)
        assert st.scal[0] == 0.0 and st.scal[1] == 0.0 and not st.codes.any()
        np.testing.assert_allclose(p, ref[t - 1], rtol=2e-6, atol=2e-6 * lr)


# --------------------------------------------------------------- bf16 parameters
def _bf16_table():
    """Every finite bf16 value (exact, as float64) with its bit pattern, sorted."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):  # the NaN patterns, dropped below
        vals = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    keep = np.isfinite(vals)
    vals, bits = vals[keep], bits[keep].astype(np.uint16)
    order = np.argsort(vals, kind="stable")
    vals, bits = vals[order], bits[order]
    # -0 and +0 compare equal: keep +0 only for the neighbour search
    keep = ~((vals == 0) & (bits == 0x8000))
    return vals[keep], bits[keep]


def _nearest_bf16(x: float, vals, bits) -> int:
    """Nearest bf16 of x by search over the whole bf16 set: the two values that
    bracket x, the nearer one in exact rational arithmetic, a tie to the even
    bit pattern."""
    from fractions import Fraction
    if x == 0.0:
        return 0x8000 if np.signbit(x) else 0
    i = int(np.searchsorted(vals, x))
    cands = [j for j in (i - 1, i) if 0 <= j < vals.size]
    fx = Fraction(x)
    dist = [abs(Fraction(float(vals[j])) - fx) for j in cands]
    best = min(dist)
    pick = [cands[k] for k in range(len(cands)) if dist[k] == best]
    if len(pick) == 2:
        pick = [j for j in pick if (int(bits[j]) & 1) == 0]
    b = int(bits[pick[0]])
    if float(vals[pick[0]]) == 0.0 and x < 0:
        b = 0x8000
    return b


def check_f64_to_bf16_rne():
    """The oracle's one-step fp64 -> bf16 rounding equals the nearest bf16 found
    by search over all bf16 values (ties to even), on random values across
    magnitudes, exact midpoints, and the subnormal range."""
    vals, bits = _bf16_table()
    rng = np.random.default_rng(77)
    xs = list(rng.standard_normal(300) * 10.0 ** rng.integers(-30, 30, 300))
    xs += list(rng.standard_normal(100) * 1e-39)               # subnormal bf16 range
    b16 = rng.integers(0x0080, 0x7F00, 200).astype(np.uint32)  # midpoints of neighbours
    lo = (b16 << 16).view(np.float32).astype(np.float64)
    hi = ((b16 + 1) << 16).view(np.float32).astype(np.float64)
    xs += list((lo + hi) / 2) + list(-(lo + hi) / 2)
    xs += list(np.nextafter((lo + hi) / 2, np.inf)) + list(np.nextafter((lo + hi) / 2, -np.inf))
    for x in xs:
        assert oracle.f64_to_bf16(float(x)) == _nearest_bf16(float(x), vals, bits), x


def _bf16_midpoint_distance(x: np.ndarray) -> np.ndarray:
    """Relative distance of each fp64 value to the nearest midpoint between two
    neighbouring bf16 values (where a rounding decision can flip)."""
    f = x.astype(np.float32)
    b = (f.view(np.uint32) >> 16).astype(np.uint32)
    lo = (b << 16).view(np.float32).astype(np.float64)
    hi = ((b + 1) << 16).view(np.float32).astype(np.float64)
    mid = (lo + hi) / 2
    return np.abs(x - mid) / np.maximum(np.abs(x), 1e-30)


def check_bf16_params_reduce_to_adam(wd: float = 0.0):
    """bf16 parameters: with k_b = B_d and m >= T the step is Adam (AdamW when
    wd > 0) on the bf16 gradients with the parameter stored back in bf16 after
    every step. Reference: torch.optim on an fp32 copy of the bf16 parameter
    each step, stored with torch's own bf16 conversion. The two may disagree by
    one bf16 step only where the exact value sits within 1e-5 of a rounding
    midpoint (torch rounds an fp32 intermediate)."""
    Bd = 250
    d, T = 4 * Bd, 8
    lr, b1, b2, eps = 1e-2, 0.9, 0.999, 1e-8
    p0 = torch.from_numpy((np.random.default_rng(18).standard_normal(d) * 0.02)
                          .astype(np.float32)).to(torch.bfloat16)
    grads = [normal_bf16(d, 900 + t) for t in range(1, T + 1)]
    q = torch.zeros(d, dtype=torch.float32, requires_grad=True)
    opt = (torch.optim.AdamW([q], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd) if wd
           else torch.optim.Adam([q], lr=lr, betas=(b1, b2), eps=eps))
    p_ref = p0.clone()
    st = oracle.new_state(d, Bd, Bd, T)
    p = p0.view(torch.int16).numpy().view(np.uint16).copy()
    exact = np.zeros(d, dtype=np.float64)
    moved = 0
    for t in range(1, T + 1):
        with torch.no_grad():
            q.copy_(p_ref.float())
        q.grad = torch.from_numpy(f32_of_bits(grads[t - 1]).copy())
        opt.step()
        p_ref = q.detach().to(torch.bfloat16)
        want = p_ref.view(torch.int16).numpy().view(np.uint16)
        oracle.step(st, p, grads[t - 1], lr=lr, beta1=b1, beta2=b2, eps=eps, wd=wd, t=t,
                    seed=3, p_exact=exact)
        diff = np.flatnonzero(p != want)
        assert np.all(_bf16_midpoint_distance(exact[diff]) < 1e-5), (t, diff[:5])
        assert diff.size <= 2
        moved += int(np.count_nonzero(p != p0.view(torch.int16).numpy().view(np.uint16)))
        p_ref = torch.from_numpy(p.view(np.int16).copy()).view(torch.bfloat16)  # resync
    assert moved > 0


# --------------------------------------------------------------- Lemma 3 / sparsity
def check_lemma3_bound(Bd: int = 8, kb: int = 4, steps: int = 200, seeds: int = 64):
    """[MicroAdam ¶3, Lemma 3] ||e_t||^2 <= 4 q_w^2 G^2 / (1 - q_w^2)^2 on tiny runs,
    q_w = (1 + omega) sqrt(1 - k/d), omega the largest Lemma 1 value seen and G the
    largest gradient norm."""
    d = Bd
    q = math.sqrt(1 - kb / d)
    for s in range(seeds):
        rng = np.random.default_rng(1000 + s)
        st = oracle.new_state(d, Bd, kb, 2)
        p = np.zeros(d, dtype=np.float32)
        G = 0.0
        w_max = 0.0
        enorms = []
        for t in range(1, steps + 1):
            x = rng.standard_t(3, d) if s % 2 else rng.standard_normal(d)
            g_bits = bf16_bits_of(x.astype(np.float32))
            G = max(G, float(np.linalg.norm(f32_of_bits(g_bits).astype(np.float64))))
            oracle.step(st, p, g_bits, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0,
                        t=t, seed=s)
            lo, hi = float(st.scal[0]), float(st.scal[1])
            if hi > lo:
                w_max = max(w_max, omega(d, lo, hi))
            e = oracle.dequantize(st.codes, d, lo, hi).astype(np.float64)
            enorms.append(float(e @ e))
        qw = (1 + w_max) * q
        assert qw < 1
        bound = 4 * qw * qw * G * G / (1 - qw * qw) ** 2
        assert max(enorms) <= bound * (1 + 1e-6), (s, max(enorms), bound)


def check_update_sparsity():
    """[MicroAdam ¶5] With m = 10 and k = d/100 at least 90 % of the update is zero."""
    Bd, kb, m = 4096, 41, 10
    d = 16 * Bd
    st = oracle.new_state(d, Bd, kb, m)
    p = np.random.default_rng(4).standard_normal(d).astype(np.float32)
    for t in range(1, 13):
        before = p.copy()
        mhat, _, _ = oracle.step(st, p, normal_bf16(d, 700 + t), lr=1e-3, beta1=0.9,
                                 beta2=0.999, eps=1e-8, wd=0.0, t=t, seed=4, want_stats=True)
        changed = np.count_nonzero(p != before)
        assert changed <= min(t, m) * (d // Bd) * kb
        assert changed <= 0.1 * d + 1e-9 * d
        assert np.count_nonzero(mhat) <= min(t, m) * (d // Bd) * kb


def check_block_locality():
    """Blocks are independent apart from delta/Delta: at t = 1 each block's row of a
    d-vector run equals the row of a run on that block alone."""
    Bd, kb, m = 200, 7, 2
    d = 3 * Bd + 50
    g_bits = normal_bf16(d, 61)
    full = _run_step1(g_bits, Bd, kb, m)
    for j in range(full.nb):
        part = _run_step1(g_bits[j * Bd:(j + 1) * Bd].copy(), Bd, kb, m)
        assert np.array_equal(part.G_idx[1 % m, 0], full.G_idx[1 % m, j])
        assert np.array_equal(part.G_val[1 % m, 0], full.G_val[1 % m, j])


# --------------------------------------------------------------- tensor lists
def _seg_blocks(segs, Bd):
    """(start, length) of every block when each tensor is cut on its own."""
    out, off = [], 0
    for n in segs:
        out += [(off + b, min(Bd, n - b)) for b in range(0, n, Bd)]
        off += n
    return out


def check_segmented_topk_minmax_step1():
    """A tensor list cut per tensor: at t = 1 each tensor's blocks (its own
    ragged last block included) hold numpy's stable arg-sort of |g| inside the
    block, k_j = ceil(L_j k_b / B_d) entries; delta_2, Delta_2 are numpy's min
    and max of the residual over all tensors [MicroAdam ¶1]."""
    Bd, kb, m = 256, 5, 2
    segs = [3 * 256 + 40, 100, 256, 2 * 256 + 2]
    d = sum(segs)
    g_bits = normal_bf16(d, 31)
    st = oracle.new_state(d, Bd, kb, m, segments=segs)
    p = np.zeros(d, dtype=np.float32)
    oracle.step(st, p, g_bits, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0, t=1, seed=3)
    a = f32_of_bits(g_bits).copy()
    blocks = _seg_blocks(segs, Bd)
    assert st.nb == len(blocks)
    for j, (b0, L) in enumerate(blocks):
        rows = topk_rows_numpy(a[b0:b0 + L], Bd, kb)[0]
        k = rows.size
        assert np.array_equal(st.G_idx[1 % m, j, :k], rows), j
        assert np.all(st.G_idx[1 % m, j, k:] == -1), j
        assert np.array_equal(f32_of_bits(st.G_val[1 % m, j, :k]), a[b0 + rows])
    for j, (b0, L) in enumerate(blocks):
        k = -(-L * kb // Bd)
        a[b0 + st.G_idx[1 % m, j, :k].astype(np.int64)] = 0.0
    assert st.scal[0] == np.min(a) and st.scal[1] == np.max(a)


def check_segmented_update_support():
    """With a tensor list, the update touches exactly the window's indices
    placed at their tensor's block starts (wd = 0) [MicroAdam ¶1, ¶5]."""
    Bd, kb, m = 128, 4, 3
    segs = [300, 128, 77, 250]
    d = sum(segs)
    st = oracle.new_state(d, Bd, kb, m, segments=segs)
    p = np.random.default_rng(4).standard_normal(d).astype(np.float32)
    blocks = _seg_blocks(segs, Bd)
    for t in range(1, 6):
        before = p.copy()
        oracle.step(st, p, normal_bf16(d, 60 + t), lr=1e-2, beta1=0.9, beta2=0.999, eps=1e-8,
                    wd=0.0, t=t, seed=9)
        want = set()
        for r in range(min(t, m)):
            for j, (b0, _) in enumerate(blocks):
                idx = st.G_idx[(t - r) % m, j]
                want.update(int(b0 + i) for i in idx[idx >= 0])
        assert set(np.flatnonzero(p != before).tolist()) == want, t


def check_segmented_whole_blocks_equal_flat():
    """Tensors that are whole multiples of B_d are cut exactly as the flat
    vector, and so is a single tensor: the states agree bit for bit."""
    Bd, kb, m = 128, 3, 3
    for segs in ([5 * 128 + 17], [2 * 128, 128, 3 * 128]):
        d = sum(segs)
        flat, seg = oracle.new_state(d, Bd, kb, m), oracle.new_state(d, Bd, kb, m, segments=segs)
        pf = np.random.default_rng(5).standard_normal(d).astype(np.float32)
        ps = pf.copy()
        for t in range(1, 6):
            g = normal_bf16(d, 80 + t)
            hyper = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.01, t=t, seed=2)
            oracle.step(flat, pf, g, **hyper)
            oracle.step(seg, ps, g, **hyper)
        for x, y in ((flat.codes, seg.codes), (flat.scal, seg.scal), (flat.G_idx, seg.G_idx),
                     (flat.G_val, seg.G_val), (pf, ps)):
            assert np.array_equal(x, y)


ALL = [check_philox_vs_torch, check_draw16_mapping, check_draw16_uniform, check_bf16_rne,
       check_topk_step1, check_minmax_step1, check_topk_later_steps, check_dequant_levels,
       check_quant_exact_levels, check_quant_error_bound, check_quant_unbiased,
       check_lemma1_per_realization, check_adamstats_vs_dense_ema, check_closed_form_m1_t1,
       check_reduces_to_adam, functools.partial(check_reduces_to_adam, wd=0.1),
       check_f64_to_bf16_rne, check_bf16_params_reduce_to_adam,
       functools.partial(check_bf16_params_reduce_to_adam, wd=0.1),
       check_lemma3_bound, check_update_sparsity, check_block_locality,
       check_segmented_topk_minmax_step1, check_segmented_update_support,
       check_segmented_whole_blocks_equal_flat]
