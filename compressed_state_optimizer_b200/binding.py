"""ctypes binding of libmua.so (include/mua.h): argument marshalling only.

Every entry point of the C ABI is reachable here under the same name
(``library().mua_step`` ...); :class:`MicroAdam` wraps a handle with tensor
checks. Tensors are passed as raw device pointers, streams as
``torch.cuda.Stream.cuda_stream``.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmua.so")

MUA_OK = 0
MUA_ERR_ARG = -1
MUA_ERR_UNSUPPORTED = -2
MUA_ERR_ALIGN = -3
MUA_ERR_CUDA = -4
MUA_STATUS_NONFINITE = 1
MUA_STATUS_TIMEOUT = 2

# Every symbol include/mua.h declares, with its ctypes signature.
_P = ctypes.c_void_p
_i64, _i32, _u64, _f32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64, ctypes.c_float
SIGNATURES = {
    "mua_create": (ctypes.c_int, [_i64, _i32, _i32, _i32, _i32, ctypes.POINTER(_P)]),
    "mua_create_shard": (ctypes.c_int, [_i64, _i32, _i32, _i32, _i32, _i64, _i64,
                                        ctypes.POINTER(_P)]),
    "mua_create_segmented": (ctypes.c_int, [ctypes.POINTER(_i64), _i32, _i32, _i32, _i32, _i32,
                                            ctypes.POINTER(_P)]),
    "mua_destroy": (None, [_P]),
    "mua_state_bytes": (_i64, [_P]),
    "mua_state_layout": (ctypes.c_int, [_P, ctypes.POINTER(_i64)]),
    "mua_step": (ctypes.c_int, [_P, _P, _P, _P, _f32, _f32, _f32, _f32, _f32, _i64, _u64, _P]),
    "mua_select": (ctypes.c_int, [_P, _P, _P, _P, _f32, _f32, _f32, _f32, _f32, _i64, _u64, _P,
                                  _P, _P]),
    "mua_minmax_offset": (_i64, [_P, _i64]),
    "mua_apply": (ctypes.c_int, [_P, _P, _P, _P, _f32, _f32, _f32, _f32, _f32, _i64, _u64, _P,
                                 _P, _P]),
    "mua_get_status": (ctypes.c_int, [_P, _P, _P, ctypes.POINTER(ctypes.c_int32)]),
    "mua_step_launches": (ctypes.c_int, [_P, _i32]),
    "mua_step_bf16": (ctypes.c_int, [_P, _P, _P, _P, _f32, _f32, _f32, _f32, _f32, _i64, _u64,
                                     _P]),
    "mua_apply_bf16": (ctypes.c_int, [_P, _P, _P, _P, _f32, _f32, _f32, _f32, _f32, _i64, _u64,
                                      _P, _P, _P]),
    "mua_set_wait_limit_ns": (ctypes.c_int, [_P, _i64]),
    "mua_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "mua_last_cuda_error": (ctypes.c_char_p, []),
    "mua_version": (ctypes.c_char_p, []),
}

_lib = None


class MuaError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what}: {strerror(code)} ({code})"
        if code == MUA_ERR_CUDA:
            msg += f" [{library().mua_last_cuda_error().decode()}]"
        super().__init__(msg)
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def library() -> ctypes.CDLL:
    """Load libmua.so; raises ImportError if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python compressed_state_optimizer_b200/build.py`")
        lib = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def strerror(code: int) -> str:
    return library().mua_strerror(code).decode()


def _check(code: int, what: str):
    if code != MUA_OK:
        raise MuaError(code, what)


def _stream_ptr(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


@dataclass
class Layout:
    header: int
    codes: int
    window: int
    row_stride: int
    blocks: int
    bytes: int


class MicroAdam:
    """One MicroAdam problem: d parameters in blocks of B_d, k_b kept per block,
    a window of m rows, b = 4 bits (optionally one rank's shard of the blocks,
    or, with ``segments``, a tensor list whose tensors are cut into blocks one
    by one; ``d`` must then be their total length).

    The optimizer state is a caller-owned ``torch.uint8`` tensor of
    ``state_bytes`` bytes (see :meth:`new_state`), zero at t = 0.
    """

    def __init__(self, d: int, block_size: int = 16384, k_per_block: int | None = None,
                 window: int = 10, bits: int = 4, *, shard: tuple[int, int] | None = None,
                 segments=None):
        if k_per_block is None:
            k_per_block = max(1, math.ceil(block_size / 100 - 1e-9))
        lib = library()
        h = ctypes.c_void_p()
        self.segments = None if segments is None else [int(n) for n in segments]
        if self.segments is not None:
            if shard is not None or sum(self.segments) != d:
                raise ValueError("segments: whole vector only, lengths summing to d")
            arr = (_i64 * len(self.segments))(*self.segments)
            _check(lib.mua_create_segmented(arr, len(self.segments), block_size, k_per_block,
                                            window, bits, ctypes.byref(h)),
                   "mua_create_segmented")
        elif shard is None:
            _check(lib.mua_create(d, block_size, k_per_block, window, bits, ctypes.byref(h)),
                   "mua_create")
        else:
            _check(lib.mua_create_shard(d, block_size, k_per_block, window, bits, shard[0],
                                        shard[1], ctypes.byref(h)), "mua_create_shard")
        self._h = h
        self.d_total = d
        self.block_size = block_size
        self.k_per_block = k_per_block
        self.window = window
        self.bits = bits
        self.shard = shard
        self.state_bytes = int(lib.mua_state_bytes(h))
        arr = (ctypes.c_int64 * 6)()
        _check(lib.mua_state_layout(h, arr), "mua_state_layout")
        self.layout = Layout(*[int(x) for x in arr])
        nb_total = self.layout.blocks if self.segments is not None else -(-d // block_size)
        if shard is None:
            self.first_block, self.blocks = 0, nb_total
        else:
            self.first_block, self.blocks = shard
        self.offset = self.first_block * block_size
        self.d = min(d, (self.first_block + self.blocks) * block_size) - self.offset

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.mua_destroy(h)
            self._h = None

    # ------------------------------------------------------------ state
    def new_state(self, device="cuda"):
        import torch
        return torch.zeros(self.state_bytes, dtype=torch.uint8, device=device)

    def _check_tensors(self, params, grads, state):
        import torch
        if params is not None:
            assert params.dtype in (torch.float32, torch.bfloat16)
            assert params.is_cuda and params.is_contiguous()
            assert params.numel() == self.d, (params.numel(), self.d)
        assert grads.dtype == torch.bfloat16 and grads.is_cuda and grads.is_contiguous()
        assert grads.numel() == self.d
        assert state.dtype == torch.uint8 and state.is_cuda and state.numel() >= self.state_bytes

    # ------------------------------------------------------------ steps
    def step(self, params, grads, state, *, lr, beta1, beta2, eps, wd, t, seed, stream=None):
        """One full step t on ``stream`` (default: the current stream);
        ``params`` fp32 (mua_step) or bf16 (mua_step_bf16)."""
        import torch
        self._check_tensors(params, grads, state)
        name = "mua_step_bf16" if params.dtype == torch.bfloat16 else "mua_step"
        _check(getattr(library(), name)(self._h, params.data_ptr(), grads.data_ptr(),
                                        state.data_ptr(), lr, beta1, beta2, eps, wd, t, seed,
                                        _stream_ptr(stream)), name)

    def select(self, params, grads, state, *, lr, beta1, beta2, eps, wd, t, seed, mhat=None,
               vhat=None, stream=None):
        """First half of step t (Top-k, window row, min/max partials)."""
        self._half("mua_select", params, grads, state, lr, beta1, beta2, eps, wd, t, seed, mhat,
                   vhat, stream)

    def _half(self, name, params, grads, state, lr, beta1, beta2, eps, wd, t, seed, mhat, vhat,
              stream):
        import torch
        self._check_tensors(params, grads, state)
        if params is not None and params.dtype == torch.bfloat16:
            if name == "mua_select":
                params = None  # not touched by the select kernel
            else:
                name = name + "_bf16"
        for x in (mhat, vhat):
            if x is not None:
                assert x.is_cuda and x.numel() == self.d and x.is_contiguous()
        fn = getattr(library(), name)
        _check(fn(self._h, params.data_ptr() if params is not None else None, grads.data_ptr(),
                  state.data_ptr(), lr, beta1,
                  beta2, eps, wd, t, seed, mhat.data_ptr() if mhat is not None else None,
                  vhat.data_ptr() if vhat is not None else None, _stream_ptr(stream)), name)

    def minmax_offset(self, t: int) -> int:
        off = int(library().mua_minmax_offset(self._h, t))
        if off < 0:
            raise MuaError(off, "mua_minmax_offset")
        return off

    def apply(self, params, grads, state, *, lr, beta1, beta2, eps, wd, t, seed, mhat=None,
              vhat=None, stream=None):
        """Second half of step t (4-bit quantization of the residual and the
        AdamStats update of the parameters)."""
        self._half("mua_apply", params, grads, state, lr, beta1, beta2, eps, wd, t, seed, mhat,
                   vhat, stream)

    def step_launches(self, bf16_params: bool = False) -> int:
        """Kernel launches of one ``step`` on the current device (1: fused)."""
        n = int(library().mua_step_launches(self._h, 1 if bf16_params else 0))
        if n < 0:
            raise MuaError(n, "mua_step_launches")
        return n

    def set_wait_limit_ns(self, ns: int):
        """Bound on the fused step's grid-barrier wait (<= 0: give up at once)."""
        _check(library().mua_set_wait_limit_ns(self._h, int(ns)), "mua_set_wait_limit_ns")

    def status(self, state, stream=None) -> int:
        out = ctypes.c_int32()
        _check(library().mua_get_status(self._h, state.data_ptr(), _stream_ptr(stream),
                                        ctypes.byref(out)), "mua_get_status")
        return int(out.value)
