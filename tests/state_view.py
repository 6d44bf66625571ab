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
