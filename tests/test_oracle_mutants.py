"""The pins catch plausible mistakes: each case plants one mistake in a copy of
the oracle's C source (on the CPU, in a temporary build), loads that build in
place of the real one and requires at least one pin in ``pins.ALL`` to fail.
The real oracle source is never modified.
"""
import contextlib
import os
import subprocess
import tempfile

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "mua_oracle.c")

MUTANTS = {
    "topk_ties_to_higher_index": (
        "return (a->key > b->key) ? -1 : 1;\n    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);",
        "return (a->key > b->key) ? -1 : 1;\n    return (a->idx > b->idx) ? -1 : (a->idx < b->idx);"),
    "topk_signed_not_magnitude": (
        "order[q].key = bits_from_f32(a[start + q]) & 0x7FFFFFFFu;",
        "order[q].key = bits_from_f32(a[start + q]);"),
    "ragged_k_floor": (
        "return (L * (int64_t)kb + Bd - 1) / Bd;",
        "return (L * (int64_t)kb) / Bd;"),
    "V_stored_as_magnitude": (
        "rv[s] = mua_oracle_f32_to_bf16(a[start + q]);",
        "rv[s] = mua_oracle_f32_to_bf16(fabsf(a[start + q]));"),
    "selected_not_zeroed": (
        "for (int64_t s = 0; s < k; ++s) a[start + order[s].idx] = 0.0f;",
        ";"),
    "row_written_off_by_one": (
        "const int64_t row = t % m;",
        "const int64_t row = (t + 1) % m;"),
    "nibble_order_swapped": (
        "return (i & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 0xFu);",
        "return (i & 1) ? (unsigned)(byte & 0xFu) : (unsigned)(byte >> 4);"),
    "dequant_drops_delta_in_step": (
        "float deq = delta_t + level;",
        "float deq = level;"),
    "dequant_unit_over_16": (
        "float unit = (Delta - delta) / 15.0f;",
        "float unit = (Delta - delta) / 16.0f;"),
    "quantize_scale_16": (
        "float inv16 = (Delta == delta) ? 0.0f : (15.0f / (Delta - delta)) * 65536.0f;",
        "float inv16 = (Delta == delta) ? 0.0f : (16.0f / (Delta - delta)) * 65536.0f;"),
    "quantize_round_to_nearest": (
        "uint32_t q = (S + r) >> 16;",
        "uint32_t q = (S + 32768u) >> 16;"),
    "quantize_rounds_down_only": (
        "uint32_t q = (S + r) >> 16;",
        "uint32_t q = S >> 16;"),
    "philox_multiplier_swapped": (
        "uint64_t prod0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;",
        "uint64_t prod0 = (uint64_t)PHILOX_M1 * (uint64_t)c0;"),
    "philox_key_bumped_before_first_round": (
        "if (round > 0) {",
        "if (1) {"),
    "draw16_halves_swapped": (
        "return (i & 1) ? (word >> 16) : (word & 0xFFFFu);",
        "return (i & 1) ? (word & 0xFFFFu) : (word >> 16);"),
    "adamstats_age_reversed": (
        "const double w1 = pow(beta1, (double)r);",
        "const double w1 = pow(beta1, (double)(rows - 1 - r));"),
    "adamstats_no_bias_correction": (
        "const double f1 = (1.0 - beta1) / (1.0 - pow(beta1, (double)t));",
        "const double f1 = (1.0 - beta1);"),
    "vhat_of_abs_not_square": (
        "z2[q] += wr2[r] * (V * V);",
        "z2[q] += wr2[r] * fabs(V);"),
    "update_sign_flipped": (
        "pq = pq - lr * (m_hat / (eps + sqrt(v_hat)));",
        "pq = pq + lr * (m_hat / (eps + sqrt(v_hat)));"),
    "eps_inside_sqrt": (
        "pq = pq - lr * (m_hat / (eps + sqrt(v_hat)));",
        "pq = pq - lr * (m_hat / sqrt(v_hat + eps));"),
    "weight_decay_dropped": (
        "if (wd != 0.0) pq = pq * decay;",
        ";"),
    "bf16_params_truncated": (
        "if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;",
        ";"),
    "bf16_params_ties_away_from_zero": (
        "if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;",
        "if (frac >= 0.5) r += 1.0;"),
    "bf16_params_widened_as_integers": (
        "double pq = p32 ? (double)p32[q] : (double)mua_oracle_bf16_to_f32(p16[q]);",
        "double pq = p32 ? (double)p32[q] : (double)p16[q];"),
    "segment_cut_ignored": (
        "blen[j] = (seg[s] - b < Bd) ? (seg[s] - b) : Bd;",
        "blen[j] = (d - (off + b) < Bd) ? (d - (off + b)) : Bd;"),
}


@contextlib.contextmanager
def mutant_library(old: str, new: str):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique in the oracle: {old!r}"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    c_path = os.path.join(tmp, "mutant.c")
    so_path = os.path.join(tmp, "libmutant.so")
    with open(c_path, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", so_path, c_path, "-lm"], check=True)
    saved_path, saved_lib = oracle._LIB, oracle._lib
    oracle._lib = None
    oracle._LIB = so_path
    try:
        yield
    finally:
        oracle._lib, oracle._LIB = saved_lib, saved_path


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(oracle_lib, name):
    old, new = MUTANTS[name]
    with mutant_library(old, new):
        caught = None
        for check in pins.ALL:
            try:
                check()
            except AssertionError:
                caught = check
                break
    assert caught is not None, f"no pin catches the planted mistake '{name}'"
