"""Decode the library's state buffer (layout of include/mua.h) into the oracle's
shapes, so that tests can compare the two element by element."""
from __future__ import annotations

import numpy as np


def header_scalars(state_bytes: np.ndarray, t_next: int) -> tuple[np.float32, np.float32]:
    """(delta, Delta) the state holds for step ``t_next`` (pair t_next mod 2)."""
    words = state_bytes[:32].view(np.uint32)
    w = 2 if (t_next & 1) else 0
    neg = words[w:w + 1].view(np.float32)[0]
    mx = words[w + 1:w + 2].view(np.float32)[0]
    return np.float32(np.float32(0.0) - neg), np.float32(mx)


def status_word(state_bytes: np.ndarray) -> int:
    return int(state_bytes[:32].view(np.uint32)[4])


def codes(state_bytes: np.ndarray, layout, d: int) -> np.ndarray:
    return state_bytes[layout.codes: layout.codes + (d + 1) // 2]


def window(state_bytes: np.ndarray, layout, m: int, kb: int):
    """G as (idx int16 [m, n_b, k_b], bf16 bits uint16 [m, n_b, k_b])."""
    nb, kp = layout.blocks, layout.row_stride
    w = state_bytes[layout.window: layout.window + 4 * nb * m * kp].view(np.uint32)
    w = w.reshape(nb, m, kp)[:, :, :kb].transpose(1, 0, 2)
    idx = (w & 0xFFFF).astype(np.uint16).view(np.int16)
    val = (w >> 16).astype(np.uint16)
    return np.ascontiguousarray(idx), np.ascontiguousarray(val)


def canonical_rows(idx: np.ndarray, val: np.ndarray):
    """Each row's k (index, value) pairs in ascending index order, empty slots
    (index -1) last: the order the oracle writes. The order inside a row is
    not part of the method (every later use of a row is per index), so rows
    are compared as sets of pairs in this form."""
    key = idx.astype(np.int32)
    key[key < 0] = 1 << 20
    o = np.argsort(key, axis=-1, kind="stable")
    return np.take_along_axis(idx, o, -1), np.take_along_axis(val, o, -1)


def canonical_words(words: np.ndarray):
    """The same for packed row words (int16 I | bf16 V << 16): (idx, val)."""
    w = np.asarray(words, dtype=np.uint32)
    return canonical_rows((w & 0xFFFF).astype(np.uint16).view(np.int16), (w >> 16).astype(np.uint16))


def window_words(state_bytes: np.ndarray, layout) -> np.ndarray:
    """The window as packed words [n_b, m, kp] (all kp slots of each row)."""
    nb, kp = layout.blocks, layout.row_stride
    m = (layout.bytes - layout.window) // (4 * nb * kp)
    return state_bytes[layout.window: layout.bytes].view(np.uint32).reshape(nb, m, kp)


def same_window_sets(a_bytes: np.ndarray, b_bytes: np.ndarray, layout) -> bool:
    """Two states' windows hold the same rows, each row compared as a set."""
    ai, av = canonical_words(window_words(a_bytes, layout))
    bi, bv = canonical_words(window_words(b_bytes, layout))
    return np.array_equal(ai, bi) and np.array_equal(av, bv)
