"""B200 (sm_100a) Kimi Delta Attention library (prefill forward and decode step): Python binding.

The work happens in ``libkda.so`` (hand-written CUDA kernels behind the C ABI
declared in ``include/kda.h``). This module only marshals torch tensors into
that ABI: pointers, sizes, dtype codes and the current CUDA stream. There is
no fallback: if the library is missing or the tensors are not on a CUDA
device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda.so")

# entry points declared in include/kda.h
EXPORTS = ("kda_decode", "kda_device_error", "kda_fwd", "kda_fwd_noalloc", "kda_status_string", "kda_version")

# (sequence, head) pairs per kda_fwd_noalloc call (KDA_NOALLOC_MAX_UNITS in include/kda.h)
NOALLOC_MAX_UNITS = 32

KDA_DTYPE_NONE, KDA_DTYPE_BF16, KDA_DTYPE_FP32 = 0, 1, 2

_lock = threading.Lock()
_lib = None


class KdaError(RuntimeError):
    """A non-zero kda_status returned by the library."""

    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


def load_library(path: str | None = None):
    """Load ``libkda.so`` (built by ``kimi_delta_attention_27_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"CUDA library not built: {p} is missing "
                               "(run python -m kimi_delta_attention_27_b200.build)")
        lib = ctypes.CDLL(p)
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        fwd_args = [P, P, P, P, P, ctypes.c_float, P, i32, i32, i64, i32, i32, i32,
                    P, ctypes.c_int, P, ctypes.c_int, P, P]
        for name in ("kda_fwd", "kda_fwd_noalloc"):
            getattr(lib, name).restype = ctypes.c_int
            getattr(lib, name).argtypes = fwd_args
        lib.kda_decode.restype = ctypes.c_int
        lib.kda_decode.argtypes = [P, P, P, P, P, ctypes.c_float, i32, i32, i32, i32, P, P, ctypes.c_int, P, P]
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_status_string.argtypes = [ctypes.c_int]
        lib.kda_version.restype = ctypes.c_int32
        lib.kda_version.argtypes = []
        lib.kda_device_error.restype = ctypes.c_int
        lib.kda_device_error.argtypes = []
        if path is None:
            _lib = lib
        return lib


def device_error() -> int:
    """Synchronise and read/clear the device-side error word (0 = no kernel gave up)."""
    return int(load_library().kda_device_error())


def status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def _dtype_code(t) -> int:
    import torch
    if t is None:
        return KDA_DTYPE_NONE
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_FP32
    return -1


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(name, t, dtype, ndim=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (no CPU path exists)")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def kda_fwd(q, k, v, g, beta, scale: float | None = None, cu_seqlens=None,
            initial_state=None, final_state=None, out=None, final_state_dtype=None,
            stream=None):
    """Chunkwise KDA forward (see include/kda.h for the full contract).

    q, k, v: bf16 [B, T, H, 128]; g: fp32 [B, T, H, 128] (raw log alpha);
    beta: fp32 [B, T, H]; cu_seqlens: int32 [N + 1] on the device (then B == 1)
    or None; initial_state: [N, H, 128, 128] bf16/fp32 or None.
    ``final_state`` may be passed preallocated; otherwise one is allocated when
    ``final_state_dtype`` is given. ``out`` may be passed preallocated.
    Returns (out, final_state or None).
    """
    return _fwd("kda_fwd", q, k, v, g, beta, scale, cu_seqlens, initial_state, final_state, out,
                final_state_dtype, stream)


def kda_fwd_noalloc(q, k, v, g, beta, out, scale: float | None = None, cu_seqlens=None,
                    initial_state=None, final_state=None, stream=None):
    """``kda_fwd`` through the allocation-free entry point of include/kda.h.

    The caller provides ``out`` (and ``final_state`` if the final states are
    wanted): neither this wrapper nor the library allocates. At most
    ``NOALLOC_MAX_UNITS`` (sequence, head) pairs per call; calls whose work
    overlaps in time race on the library's fixed scratch. Returns
    (out, final_state or None).
    """
    if out is None:
        raise ValueError("kda_fwd_noalloc needs a preallocated out tensor")
    return _fwd("kda_fwd_noalloc", q, k, v, g, beta, scale, cu_seqlens, initial_state, final_state,
                out, None, stream)


def _fwd(entry, q, k, v, g, beta, scale, cu_seqlens, initial_state, final_state, out,
         final_state_dtype, stream):
    import torch
    _check("q", q, torch.bfloat16, 4)
    _check("k", k, torch.bfloat16, 4)
    _check("v", v, torch.bfloat16, 4)
    _check("g", g, torch.float32, 4)
    _check("beta", beta, torch.float32, 3)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != q.shape[:3] or beta.shape != (B, T, H):
        raise ValueError("q/k/g must share [B, T, H, 128]; v [B, T, H, 128]; beta [B, T, H]")
    if cu_seqlens is not None:
        _check("cu_seqlens", cu_seqlens, torch.int32, 1)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if initial_state is not None:
        _check("initial_state", initial_state, None, 4)
    if out is None:
        out = torch.empty((B, T, H, Dv), dtype=torch.bfloat16, device=q.device)
    else:
        _check("out", out, torch.bfloat16, 4)
    if final_state is None and final_state_dtype is not None:
        final_state = torch.empty((N, H, Dk, Dv), dtype=final_state_dtype, device=q.device)
    if final_state is not None:
        _check("final_state", final_state, None, 4)
    if scale is None:
        scale = Dk ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    lib = load_library()
    ic, fc = _dtype_code(initial_state), _dtype_code(final_state)
    st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                             _ptr(cu_seqlens), int(N), int(B), int(T), int(H), int(Dk), int(Dv),
                             _ptr(initial_state), ic if ic >= 0 else 99,
                             _ptr(final_state), fc if fc >= 0 else 99,
                             _ptr(out), ctypes.c_void_p(int(stream)))
    if st != 0:
        raise KdaError(st, lib.kda_status_string(st).decode())
    return out, final_state


def kda_decode(q, k, v, g, beta, state_in=None, state_out=None, scale: float | None = None, out=None,
               state_dtype=None, stream=None):
    """One recurrent step for a batch of requests (see include/kda.h, kda_decode).

    q, k, v: bf16 [B, H, 128]; g: fp32 [B, H, 128] (raw log alpha); beta: fp32 [B, H];
    state_in: [B, H, 128, 128] bf16/fp32 or None (zero states). ``state_out`` may be
    ``state_in`` itself (update in place) or a separate buffer; if it is None and
    ``state_dtype`` is given, one is allocated. ``out`` may be passed preallocated.
    Returns (out, state_out or None).
    """
    import torch
    _check("q", q, torch.bfloat16, 3)
    _check("k", k, torch.bfloat16, 3)
    _check("v", v, torch.bfloat16, 3)
    _check("g", g, torch.float32, 3)
    _check("beta", beta, torch.float32, 2)
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape[:2] != q.shape[:2] or beta.shape != (B, H):
        raise ValueError("q/k/g must share [B, H, 128]; v [B, H, 128]; beta [B, H]")
    if state_in is not None:
        _check("state_in", state_in, None, 4)
    if state_out is None and state_dtype is not None:
        state_out = torch.empty((B, H, Dk, Dv), dtype=state_dtype, device=q.device)
    if state_out is not None:
        _check("state_out", state_out, None, 4)
    if state_in is not None and state_out is not None and state_in.dtype != state_out.dtype:
        raise ValueError("state_in and state_out must have the same dtype")
    st_t = state_in if state_in is not None else state_out
    code = _dtype_code(st_t)
    if out is None:
        out = torch.empty((B, H, Dv), dtype=torch.bfloat16, device=q.device)
    else:
        _check("out", out, torch.bfloat16, 3)
    if scale is None:
        scale = Dk ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    lib = load_library()
    st = lib.kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), int(B), int(H),
                        int(Dk), int(Dv), _ptr(state_in), _ptr(state_out), code if code >= 0 else 99,
                        _ptr(out), ctypes.c_void_p(int(stream)))
    if st != 0:
        raise KdaError(st, lib.kda_status_string(st).decode())
    return out, state_out
