"""Python binding of the beam-parallel Gated DeltaNet decode library (C ABI in include/ola.h).

Argument marshalling only: every step of the decode runs in the library's CUDA kernels.
The functions named ``ola_*`` mirror the C entry points one to one and take raw device
pointers (ints); :class:`Decoder` and :func:`prefill` take torch tensors, check their
device, dtype, shape and contiguity, and pass ``data_ptr()`` and the current CUDA stream.

There is no fallback: if the shared object has not been built, importing works but every
call raises :class:`LibraryMissing`.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

__all__ = ["OlaError", "LibraryMissing", "Geometry", "lib", "Decoder", "prefill",
           "OLA_F32", "OLA_BF16", "OLA_PATH_REPLAY", "OLA_PATH_FULLSTATE", "OLA_PATH_REPLAYSSM",
           "OLA_MATH_FP32",
           "OLA_MATH_TENSOR", "LIB_PATH", "HEADER_PATH", "declared_symbols"]

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "_build", "libola.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG_DIR), "include", "ola.h")

OLA_OK, OLA_ERR_INVALID_ARG, OLA_ERR_UNSUPPORTED, OLA_ERR_CAPACITY = 0, 1, 2, 3
OLA_ERR_BAD_PARENT, OLA_ERR_OOM, OLA_ERR_CUDA, OLA_ERR_TIMEOUT = 4, 5, 6, 7
OLA_ERR_SCRATCH_LIMIT = 8
OLA_NOALLOC_SCRATCH_BYTES = 16 << 20
OLA_F32, OLA_BF16 = 0, 1
OLA_PATH_REPLAY, OLA_PATH_FULLSTATE, OLA_PATH_REPLAYSSM = 0, 1, 2
OLA_MATH_FP32, OLA_MATH_TENSOR = 0, 1


class LibraryMissing(RuntimeError):
    pass


class OlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().ola_strerror(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


class Geometry(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int32), ("H", ctypes.c_int32), ("d_k", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("B", ctypes.c_int32), ("T_max", ctypes.c_int32),
                ("in_dtype", ctypes.c_int32), ("path", ctypes.c_int32),
                ("math", ctypes.c_int32)]


_LIB: Optional[ctypes.CDLL] = None
_P = ctypes.c_void_p


def _declare(L: ctypes.CDLL) -> None:
    i32, u64p = ctypes.c_int32, ctypes.POINTER(ctypes.c_uint64)
    sig = {
        "ola_version": (i32, []),
        "ola_strerror": (ctypes.c_char_p, [i32]),
        "ola_workspace_bytes": (i32, [ctypes.POINTER(Geometry), u64p]),
        "ola_create": (i32, [ctypes.POINTER(Geometry), _P, _P, ctypes.POINTER(_P)]),
        "ola_step": (i32, [_P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "ola_step_host": (i32, [_P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "ola_step_host_async": (i32, [_P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "ola_host_sync": (i32, [_P]),
        "ola_reset": (i32, [_P]),
        "ola_current_step": (i32, [_P]),
        "ola_get_ancestry": (i32, [_P, _P, _P]),
        "ola_get_error": (i32, [_P]),
        "ola_compact": (i32, [_P, ctypes.POINTER(ctypes.c_int32), _P]),
        "ola_destroy": (i32, [_P]),
        "ola_prefill": (i32, [i32, i32, i32, i32, i32, i32, _P, _P, _P, _P, _P, _P]),
        "ola_noalloc_scratch_bytes": (ctypes.c_uint64, [ctypes.POINTER(Geometry)]),
        "ola_decode_noalloc": (i32, [ctypes.POINTER(Geometry), _P, _P, _P, _P, _P, _P, _P, _P,
                                     _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def lib() -> ctypes.CDLL:
    """The loaded shared object (raises LibraryMissing if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise LibraryMissing(
                f"{LIB_PATH} is missing: build it with "
                "`python -m linear_attention_beam_gdn_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        _declare(L)
        _LIB = L
    return _LIB


def declared_symbols(header: str = HEADER_PATH):
    """Names of the functions declared in the C header."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ola_[a-z_]+)\s*\(", text)))


def _check(status: int, where: str) -> None:
    if status != OLA_OK:
        raise OlaError(status, where)


# ------------------------------------------------------------------ raw C entry points

def ola_version() -> int:
    return lib().ola_version()


def ola_strerror(status: int) -> str:
    return lib().ola_strerror(status).decode()


def ola_workspace_bytes(geom: Geometry) -> int:
    out = ctypes.c_uint64(0)
    _check(lib().ola_workspace_bytes(ctypes.byref(geom), ctypes.byref(out)),
           "ola_workspace_bytes")
    return out.value


def ola_create(geom: Geometry, S_ctx_ptr: int, stream: int) -> int:
    h = _P()
    _check(lib().ola_create(ctypes.byref(geom), S_ctx_ptr, stream, ctypes.byref(h)),
           "ola_create")
    return h.value


def ola_step(h, q, k, v, g, beta, parent_idx, out_o, stream) -> int:
    return lib().ola_step(h, q, k, v, g, beta, parent_idx, out_o, stream)


def ola_step_host(h, q, k, v, g, beta, parent_idx, out_o, stream) -> int:
    return lib().ola_step_host(h, q, k, v, g, beta, parent_idx, out_o, stream)


def ola_step_host_async(h, q, k, v, g, beta, parent_idx, out_o, stream) -> int:
    return lib().ola_step_host_async(h, q, k, v, g, beta, parent_idx, out_o, stream)


def ola_host_sync(h) -> int:
    return lib().ola_host_sync(h)


def ola_reset(h) -> int:
    return lib().ola_reset(h)


def ola_current_step(h) -> int:
    return lib().ola_current_step(h)


def ola_get_ancestry(h, out, stream) -> int:
    return lib().ola_get_ancestry(h, out, stream)


def ola_get_error(h) -> int:
    return lib().ola_get_error(h)


def ola_destroy(h) -> int:
    return lib().ola_destroy(h)


def ola_compact(h, stream) -> tuple:
    """(status, number of folded steps)."""
    n = ctypes.c_int32(0)
    st = lib().ola_compact(h, ctypes.byref(n), stream)
    return st, n.value


def ola_prefill(R, H, d_k, d_v, P, in_dtype, k, v, g, beta, S_out, stream) -> int:
    return lib().ola_prefill(R, H, d_k, d_v, P, in_dtype, k, v, g, beta, S_out, stream)


def ola_noalloc_scratch_bytes(geom: Geometry) -> int:
    return lib().ola_noalloc_scratch_bytes(ctypes.byref(geom))


def ola_decode_noalloc(geom: Geometry, S_ctx, q, k, v, g, beta, parent_idx, out_o,
                       stream) -> int:
    return lib().ola_decode_noalloc(ctypes.byref(geom), S_ctx, q, k, v, g, beta, parent_idx,
                                    out_o, stream)


# ------------------------------------------------------------------ torch-facing wrappers

def _torch():
    import torch
    return torch


def _stream_ptr(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _dtype_code(dt) -> int:
    torch = _torch()
    if dt == torch.bfloat16:
        return OLA_BF16
    if dt == torch.float32:
        return OLA_F32
    raise TypeError(f"unsupported input dtype {dt}")


def _need(x, shape, dtype, name, device):
    torch = _torch()
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if x.device != device:
        raise ValueError(f"{name} is on {x.device}, expected {device}")
    if tuple(x.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(x.shape)}, expected {tuple(shape)}")
    if x.dtype != dtype:
        raise TypeError(f"{name} has dtype {x.dtype}, expected {dtype}")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return x.data_ptr()


def prefill(k, v, g, beta, stream=None):
    """Shared post-prefill state S [R, H, d_v, d_k] fp32 from prompt tokens
    k [R, P, H, d_k], v [R, P, H, d_v] (bf16 or fp32), g, beta [R, P, H] fp32."""
    torch = _torch()
    R, P, H, d_k = k.shape
    d_v = v.shape[-1]
    dev = k.device
    dt = k.dtype
    S = torch.empty((R, H, d_v, d_k), device=dev, dtype=torch.float32)
    args = [_need(k, (R, P, H, d_k), dt, "k", dev), _need(v, (R, P, H, d_v), dt, "v", dev),
            _need(g, (R, P, H), torch.float32, "g", dev),
            _need(beta, (R, P, H), torch.float32, "beta", dev)]
    _check(ola_prefill(R, H, d_k, d_v, P, _dtype_code(dt), *args, S.data_ptr(),
                       _stream_ptr(stream)), "ola_prefill")
    return S


class Decoder:
    """One GDN layer's beam decoder for R requests (owns an ola handle)."""

    def __init__(self, S_ctx, B: int, T_max: int, in_dtype, path: int = OLA_PATH_REPLAY,
                 math: int = OLA_MATH_TENSOR, stream=None):
        torch = _torch()
        R, H, d_v, d_k = S_ctx.shape
        self.geom = Geometry(R, H, d_k, d_v, B, T_max, _dtype_code(in_dtype), path, math)
        self.device = S_ctx.device
        self.in_dtype = in_dtype
        ptr = _need(S_ctx, (R, H, d_v, d_k), torch.float32, "S_ctx", self.device)
        self.handle = ola_create(self.geom, ptr, _stream_ptr(stream))

    # shapes
    @property
    def R(self): return self.geom.R

    @property
    def H(self): return self.geom.H

    @property
    def B(self): return self.geom.B

    @property
    def d_k(self): return self.geom.d_k

    @property
    def d_v(self): return self.geom.d_v

    @property
    def t(self) -> int:
        return ola_current_step(self.handle)

    def _ptrs(self, q, k, v, g, beta, parent_idx, out):
        torch = _torch()
        R, B, H, dk, dv = self.R, self.B, self.H, self.d_k, self.d_v
        dev, dt = self.device, self.in_dtype
        return [_need(q, (R, B, H, dk), dt, "q", dev), _need(k, (R, B, H, dk), dt, "k", dev),
                _need(v, (R, B, H, dv), dt, "v", dev),
                _need(g, (R, B, H), torch.float32, "g", dev),
                _need(beta, (R, B, H), torch.float32, "beta", dev),
                _need(parent_idx, (R, B), torch.int32, "parent_idx", dev),
                _need(out, (R, B, H, dv), torch.float32, "out_o", dev)]

    def step(self, q, k, v, g, beta, parent_idx, out=None, stream=None):
        """Run one decode step; returns o [R, B, H, d_v] fp32."""
        torch = _torch()
        if out is None:
            out = torch.empty((self.R, self.B, self.H, self.d_v), device=self.device,
                              dtype=torch.float32)
        _check(ola_step(self.handle, *self._ptrs(q, k, v, g, beta, parent_idx, out),
                        _stream_ptr(stream)), "ola_step")
        return out

    def step_host(self, q, k, v, g, beta, parent_idx, out, stream=None):
        """ola_step_host: all tensors on the CPU (pinned for asynchronous copies)."""
        torch = _torch()
        cpu = torch.device("cpu")
        R, B, H, dk, dv = self.R, self.B, self.H, self.d_k, self.d_v
        dt = self.in_dtype
        ptrs = [_need(q, (R, B, H, dk), dt, "q", cpu), _need(k, (R, B, H, dk), dt, "k", cpu),
                _need(v, (R, B, H, dv), dt, "v", cpu),
                _need(g, (R, B, H), torch.float32, "g", cpu),
                _need(beta, (R, B, H), torch.float32, "beta", cpu),
                _need(parent_idx, (R, B), torch.int32, "parent_idx", cpu),
                _need(out, (R, B, H, dv), torch.float32, "out_o", cpu)]
        _check(ola_step_host(self.handle, *ptrs, _stream_ptr(stream)), "ola_step_host")
        return out

    def step_host_async(self, q, k, v, g, beta, parent_idx, out, stream=None):
        """ola_step_host_async: CPU tensors (pinned); `out` is complete after host_sync()."""
        torch = _torch()
        cpu = torch.device("cpu")
        R, B, H, dk, dv = self.R, self.B, self.H, self.d_k, self.d_v
        dt = self.in_dtype
        ptrs = [_need(q, (R, B, H, dk), dt, "q", cpu), _need(k, (R, B, H, dk), dt, "k", cpu),
                _need(v, (R, B, H, dv), dt, "v", cpu),
                _need(g, (R, B, H), torch.float32, "g", cpu),
                _need(beta, (R, B, H), torch.float32, "beta", cpu),
                _need(parent_idx, (R, B), torch.int32, "parent_idx", cpu),
                _need(out, (R, B, H, dv), torch.float32, "out_o", cpu)]
        _check(ola_step_host_async(self.handle, *ptrs, _stream_ptr(stream)),
               "ola_step_host_async")
        return out

    def host_sync(self) -> None:
        _check(ola_host_sync(self.handle), "ola_host_sync")

    def ancestry(self, stream=None):
        """Chains of the current beams: [R, B, t] int32 (device)."""
        torch = _torch()
        t = self.t
        out = torch.empty((self.R, self.B, t), device=self.device, dtype=torch.int32)
        _check(ola_get_ancestry(self.handle, out.data_ptr(), _stream_ptr(stream)),
               "ola_get_ancestry")
        return out

    def error(self) -> int:
        return ola_get_error(self.handle)

    def compact(self, stream=None) -> int:
        """Fold the chain steps every live beam shares into S_ctx and free their slots
        (ola_compact); returns the number of folded steps."""
        st, n = ola_compact(self.handle, _stream_ptr(stream))
        _check(st, "ola_compact")
        return n

    def reset(self) -> None:
        _check(ola_reset(self.handle), "ola_reset")

    def close(self) -> None:
        if getattr(self, "handle", None):
            ola_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
