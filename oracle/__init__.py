"""Plain CPU oracle for the MicroAdam step (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never imports, links or calls it, and shares no code with
it.

The arithmetic lives in ``mua_oracle.c`` (plain C, built with
``-ffp-contract=off``); this module only marshals numpy arrays through ctypes
and keeps the oracle's state in the page's own shape: the 4-bit codes ``e``,
the scalars ``delta``/``Delta`` and the window ``G`` as ``m`` rows of
``(I, V)`` per block ("MicroAdam (Sparse-Gradient Adaptive Optimization with
Quantized Error Feedback)", paragraph 1).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mua_oracle.c")
_LIB = os.path.join(_HERE, "libmua_oracle.so")
_LIB_OMP = os.path.join(_HERE, "libmua_oracle_omp.so")  # the same source with -fopenmp

# gcc flags: IEEE fp32 with every operation rounded, no contraction into FMA.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def _compile(out: str, extra, force: bool):
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, *extra, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``mua_oracle.c`` into ``libmua_oracle.so`` and, with OpenMP over
    blocks, ``libmua_oracle_omp.so`` (both next to it)."""
    _compile(_LIB_OMP, ["-fopenmp"], force)
    return _compile(_LIB, [], force)


_lib = None
_lib_omp = None


def lib_openmp() -> ctypes.CDLL:
    """The OpenMP build (bit-identical results; threads from OMP_NUM_THREADS or
    ``set_threads``)."""
    global _lib_omp
    if _lib_omp is None:
        _compile(_LIB_OMP, ["-fopenmp"], False)
        _lib_omp = _declare(ctypes.CDLL(_LIB_OMP))
    return _lib_omp


def set_threads(n: int):
    """Threads of the OpenMP build."""
    lib_openmp().omp_set_num_threads(int(n))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = _declare(ctypes.CDLL(_LIB))
    return _lib


def _declare(L: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    i64, i32, u64, f32, f64 = (ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64,
                               ctypes.c_float, ctypes.c_double)
    L.mua_oracle_philox4x32_10.argtypes = [P, P, P]
    L.mua_oracle_philox4x32_10.restype = None
    L.mua_oracle_draw16.argtypes = [u64, i64, i64]
    L.mua_oracle_draw16.restype = ctypes.c_uint32
    L.mua_oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.mua_oracle_bf16_to_f32.restype = f32
    L.mua_oracle_f32_to_bf16.argtypes = [f32]
    L.mua_oracle_f32_to_bf16.restype = ctypes.c_uint16
    L.mua_oracle_f64_to_bf16.argtypes = [f64]
    L.mua_oracle_f64_to_bf16.restype = ctypes.c_uint16
    L.mua_oracle_dequantize.argtypes = [P, i64, f32, f32, P]
    L.mua_oracle_dequantize.restype = None
    L.mua_oracle_quantize.argtypes = [P, i64, i64, f32, f32, i64, u64, P]
    L.mua_oracle_quantize.restype = None
    L.mua_oracle_block_k.argtypes = [i64, i32, i32]
    L.mua_oracle_block_k.restype = i64
    L.mua_oracle_step.argtypes = [i64, i32, i32, i32, P, P, P, P, P, P,
                                  f64, f64, f64, f64, f64, i64, u64, P, P, P]
    L.mua_oracle_step.restype = ctypes.c_int
    L.mua_oracle_step_seg.argtypes = [P, i32, i32, i32, i32, P, P, P, P, P, P,
                                      f64, f64, f64, f64, f64, i64, u64, P, P, P]
    L.mua_oracle_step_seg.restype = ctypes.c_int
    L.mua_oracle_step_seg_bf16.argtypes = [P, i32, i32, i32, i32, P, P, P, P, P, P, P,
                                           f64, f64, f64, f64, f64, i64, u64, P, P, P]
    L.mua_oracle_step_seg_bf16.restype = ctypes.c_int
    L.mua_oracle_num_blocks.argtypes = [P, i32, i32]
    L.mua_oracle_num_blocks.restype = i64
    return L


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- primitives
def philox4x32_10(counter, key) -> np.ndarray:
    """Philox4x32-10 of one 4x32 counter under one 2x32 key."""
    c = np.ascontiguousarray(np.asarray(counter, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    lib().mua_oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def draw16(seed: int, t: int, i: int) -> int:
    """The 16-bit uniform draw of element ``i`` at step ``t``."""
    return int(lib().mua_oracle_draw16(seed, t, i))


def bf16_to_f32(h: int) -> float:
    return float(lib().mua_oracle_bf16_to_f32(h))


def f32_to_bf16(x: float) -> int:
    return int(lib().mua_oracle_f32_to_bf16(x))


def f64_to_bf16(x: float) -> int:
    """bf16 bits of an fp64 value rounded once, to nearest with ties to even."""
    return int(lib().mua_oracle_f64_to_bf16(x))


def block_k(L: int, Bd: int, kb: int) -> int:
    return int(lib().mua_oracle_block_k(L, Bd, kb))


def dequantize(codes: np.ndarray, n: int, delta: float, Delta: float) -> np.ndarray:
    """Q^{-1}: the fp32 values of ``n`` packed 4-bit codes."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    assert codes.size >= (n + 1) // 2
    out = np.zeros(n, dtype=np.float32)
    lib().mua_oracle_dequantize(_ptr(codes), n, delta, Delta, _ptr(out))
    return out


def quantize(x: np.ndarray, delta: float, Delta: float, t: int, seed: int,
             base: int = 0) -> np.ndarray:
    """Q: stochastic 4-bit codes of fp32 ``x`` (global index of x[0] = base)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros((x.size + 1) // 2, dtype=np.uint8)
    lib().mua_oracle_quantize(_ptr(x), x.size, base, delta, Delta, t, seed, _ptr(codes))
    return codes


# ---------------------------------------------------------------- the step
@dataclass
class OracleState:
    """MicroAdam optimizer state in the page's shape.

    codes  uint8[ceil(d/2)]   the 4-bit error feedback e (even index = low nibble)
    scal   float32[2]         (delta, Delta)
    G_idx  int16[m, n_b, k_b] block-relative indices of the window rows (-1 empty)
    G_val  uint16[m, n_b, k_b] bf16 bits of the window values
    segs   int64[n] segment (tensor) lengths, blocks cut per segment; one
           segment of length d is the flat cut
    """
    d: int
    Bd: int
    kb: int
    m: int
    codes: np.ndarray
    scal: np.ndarray
    G_idx: np.ndarray
    G_val: np.ndarray
    segs: np.ndarray | None = None

    @property
    def nb(self) -> int:
        return self.G_idx.shape[1]

    def copy(self) -> "OracleState":
        return OracleState(self.d, self.Bd, self.kb, self.m, self.codes.copy(),
                           self.scal.copy(), self.G_idx.copy(), self.G_val.copy(),
                           None if self.segs is None else self.segs.copy())


def num_blocks(segs, Bd: int) -> int:
    segs = np.ascontiguousarray(segs, dtype=np.int64)
    return int(lib().mua_oracle_num_blocks(_ptr(segs), segs.size, Bd))


def new_state(d: int, Bd: int, kb: int, m: int, segments=None) -> OracleState:
    """The initial state: e_0 = 0 with delta = Delta = 0 and an empty window.
    ``segments``: tensor lengths summing to d, blocks cut per tensor."""
    segs = None
    if segments is not None:
        segs = np.ascontiguousarray(segments, dtype=np.int64)
        assert int(segs.sum()) == d and np.all(segs > 0)
        nb = num_blocks(segs, Bd)
    else:
        nb = (d + Bd - 1) // Bd
    return OracleState(d, Bd, kb, m,
                       codes=np.zeros((d + 1) // 2, dtype=np.uint8),
                       scal=np.zeros(2, dtype=np.float32),
                       G_idx=np.full((m, nb, kb), -1, dtype=np.int16),
                       G_val=np.zeros((m, nb, kb), dtype=np.uint16),
                       segs=segs)


def step(st: OracleState, p: np.ndarray, g_bits: np.ndarray, *, lr: float, beta1: float,
         beta2: float, eps: float, wd: float, t: int, seed: int,
         want_stats: bool = False, p_exact: np.ndarray | None = None, openmp: bool = False):
    """One MicroAdam step in place on ``st`` and ``p``.

    ``p`` holds the parameters: float32[d], or uint16[d] bf16 bits (each changed
    parameter is then rounded once to bf16; ``p_exact``, float64[d], receives
    the values before that rounding). ``g_bits`` is the bf16 gradient as
    uint16 bits. The fp32 hyper-parameters are widened exactly to fp64.
    Returns ``(m_hat, v_hat, m_abs)`` as fp64 arrays when ``want_stats`` is
    set, else None. ``openmp``: run the OpenMP build (same results).
    """
    L = lib_openmp() if openmp else lib()
    assert p.dtype in (np.float32, np.uint16) and p.size == st.d and p.flags["C_CONTIGUOUS"]
    g_bits = np.ascontiguousarray(g_bits, dtype=np.uint16)
    assert g_bits.size == st.d
    stats = None
    if want_stats:
        stats = tuple(np.zeros(st.d, dtype=np.float64) for _ in range(3))
    f = lambda v: float(np.float32(v))  # noqa: E731  (the fp32 value the kernels see)
    segs = st.segs if st.segs is not None else np.array([st.d], dtype=np.int64)
    tail = (f(lr), f(beta1), f(beta2), f(eps), f(wd), t, seed,
            *(_ptr(s) for s in (stats or (None,) * 3)))
    if p.dtype == np.uint16:
        if p_exact is not None:
            assert p_exact.dtype == np.float64 and p_exact.size == st.d
        rc = L.mua_oracle_step_seg_bf16(_ptr(segs), segs.size, st.Bd, st.kb, st.m, _ptr(p),
                                            _ptr(p_exact), _ptr(g_bits), _ptr(st.codes),
                                            _ptr(st.scal), _ptr(st.G_idx), _ptr(st.G_val), *tail)
    elif st.segs is None:
        rc = L.mua_oracle_step(st.d, st.Bd, st.kb, st.m, _ptr(p), _ptr(g_bits),
                                   _ptr(st.codes), _ptr(st.scal), _ptr(st.G_idx),
                                   _ptr(st.G_val), *tail)
    else:
        rc = L.mua_oracle_step_seg(_ptr(st.segs), st.segs.size, st.Bd, st.kb, st.m,
                                       _ptr(p), _ptr(g_bits), _ptr(st.codes), _ptr(st.scal),
                                       _ptr(st.G_idx), _ptr(st.G_val), *tail)
    if rc != 0:
        raise ValueError("oracle step rejected its arguments")
    return stats
