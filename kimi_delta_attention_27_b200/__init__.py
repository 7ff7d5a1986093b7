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
EXPORTS = ("kda_bwd", "kda_bwd_workspace", "kda_decode", "kda_device_error", "kda_fwd", "kda_fwd_ex",
           "kda_fwd_noalloc", "kda_fwd_segmented", "kda_fwd_segmented_workspace", "kda_status_string",
           "kda_version")

# kda_fwd_ex gate kinds and flags (include/kda.h)
KDA_GATE_FP32, KDA_GATE_BF16, KDA_GATE_SCALAR_FP32 = 0, 1, 2
KDA_FLAG_L2NORM_QK, KDA_FLAG_GATE_LOGSIGMOID = 1, 2

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
        lib.kda_fwd_ex.restype = ctypes.c_int
        lib.kda_fwd_ex.argtypes = [P, P, P, P, i32, P, ctypes.c_float, P, i32, i32, i64, i32, i32, i32,
                                   P, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_uint32, P]
        lib.kda_fwd_segmented.restype = ctypes.c_int
        lib.kda_fwd_segmented.argtypes = [P, P, P, P, P, ctypes.c_float, i32, i64, i32, i32, i32, P, ctypes.c_int,
                                          P, ctypes.c_int, P, i64, P, ctypes.c_size_t, P]
        lib.kda_fwd_segmented_workspace.restype = ctypes.c_size_t
        lib.kda_fwd_segmented_workspace.argtypes = [i32, i64, i32, i64]
        lib.kda_bwd.restype = ctypes.c_int
        lib.kda_bwd.argtypes = [P, P, P, P, P, ctypes.c_float, P, i32, i32, i64, i32, i32, i32, P, ctypes.c_int,
                                P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.kda_bwd_workspace.restype = ctypes.c_size_t
        lib.kda_bwd_workspace.argtypes = [i64, i32, i32]
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


def _check(name, t, dtype, ndim=None, shape=None):
    """Validate one tensor argument. ``shape`` (a tuple) is required exactly: the C
    ABI receives bare pointers and cannot tell an undersized buffer from a right one."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_devices(**tensors):
    """Every given tensor on one CUDA device (the first one's); returns that device."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError(f"{name} must be on a CUDA device (no CPU path exists)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} must be on {dev}, got {t.device}")
    return dev


def kda_fwd(q, k, v, g, beta, scale: float | None = None, cu_seqlens=None,
            initial_state=None, final_state=None, out=None, final_state_dtype=None,
            stream=None, l2norm_qk: bool = False, gate_logsigmoid: bool = False):
    """Chunkwise KDA forward (see include/kda.h for the full contract).

    q, k, v: bf16 [B, T, H, 128]; g: log alpha, fp32 [B, T, H, 128] (kda_fwd), or
    bf16 [B, T, H, 128], or fp32 [B, T, H] (one decay per token and head: Gated
    DeltaNet); beta: fp32 [B, T, H]; cu_seqlens: int32 [N + 1] on the device (then
    B == 1) or None; initial_state: [N, H, 128, 128] bf16/fp32 or None.
    ``l2norm_qk``: the kernel L2-normalises q and k first; ``gate_logsigmoid``: g
    holds the gate's pre-activation and log alpha = logsigmoid(g). Any of these
    variants goes through kda_fwd_ex, the plain case through kda_fwd.
    ``final_state`` may be passed preallocated; otherwise one is allocated when
    ``final_state_dtype`` is given. ``out`` may be passed preallocated.
    Returns (out, final_state or None).
    """
    import torch
    kind = KDA_GATE_FP32
    if isinstance(g, torch.Tensor):
        if g.dtype == torch.bfloat16:
            kind = KDA_GATE_BF16
        elif g.dim() == 3:
            kind = KDA_GATE_SCALAR_FP32
    flags = (KDA_FLAG_L2NORM_QK if l2norm_qk else 0) | (KDA_FLAG_GATE_LOGSIGMOID if gate_logsigmoid else 0)
    entry = "kda_fwd" if kind == KDA_GATE_FP32 and flags == 0 else "kda_fwd_ex"
    return _fwd(entry, q, k, v, g, beta, scale, cu_seqlens, initial_state, final_state, out,
                final_state_dtype, stream, gate_kind=kind, flags=flags)


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
         final_state_dtype, stream, gate_kind=0, flags=0):
    import torch
    _check("q", q, torch.bfloat16, 4)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1] if v.dim() == 4 else -1
    _check("k", k, torch.bfloat16, shape=q.shape)
    _check("v", v, torch.bfloat16, shape=(B, T, H, Dv))
    if gate_kind == KDA_GATE_SCALAR_FP32:
        _check("g", g, torch.float32, shape=(B, T, H))
    else:
        _check("g", g, torch.bfloat16 if gate_kind == KDA_GATE_BF16 else torch.float32, shape=q.shape)
    _check("beta", beta, torch.float32, shape=(B, T, H))
    if cu_seqlens is not None:
        _check("cu_seqlens", cu_seqlens, torch.int32, 1)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    state_shape = (N, H, Dk, Dv)
    if initial_state is not None:
        _check("initial_state", initial_state, None, shape=state_shape)
    if out is not None:
        _check("out", out, torch.bfloat16, shape=(B, T, H, Dv))
    if final_state is not None:
        _check("final_state", final_state, None, shape=state_shape)
    dev = _check_devices(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu_seqlens, initial_state=initial_state,
                         out=out, final_state=final_state)
    if out is None:
        out = torch.empty((B, T, H, Dv), dtype=torch.bfloat16, device=dev)
    if final_state is None and final_state_dtype is not None:
        final_state = torch.empty(state_shape, dtype=final_state_dtype, device=dev)
    if scale is None:
        scale = Dk ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    lib = load_library()
    ic, fc = _dtype_code(initial_state), _dtype_code(final_state)
    # the library works on the current device: make it q's
    with torch.cuda.device(dev):
        if entry == "kda_fwd_ex":
            st = lib.kda_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), int(gate_kind), _ptr(beta), float(scale),
                                _ptr(cu_seqlens), int(N), int(B), int(T), int(H), int(Dk), int(Dv),
                                _ptr(initial_state), ic if ic >= 0 else 99,
                                _ptr(final_state), fc if fc >= 0 else 99,
                                _ptr(out), int(flags), ctypes.c_void_p(int(stream)))
        else:
            st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                     _ptr(cu_seqlens), int(N), int(B), int(T), int(H), int(Dk), int(Dv),
                                     _ptr(initial_state), ic if ic >= 0 else 99,
                                     _ptr(final_state), fc if fc >= 0 else 99,
                                     _ptr(out), ctypes.c_void_p(int(stream)))
    if st != 0:
        raise KdaError(st, lib.kda_status_string(st).decode())
    return out, final_state


def kda_fwd_segmented(q, k, v, g, beta, segment_len: int, scale: float | None = None, initial_state=None,
                      final_state=None, out=None, final_state_dtype=None, workspace=None, stream=None):
    """kda_fwd over fixed-length rows split into pieces of ``segment_len`` tokens that run at
    once (see include/kda.h, kda_fwd_segmented). q, k, v, g, beta, states and out as for
    ``kda_fwd`` without cu_seqlens. ``workspace`` (a uint8 CUDA tensor of at least
    ``segmented_workspace_bytes(...)`` bytes) is allocated here when not given.
    Returns (out, final_state or None)."""
    import torch
    _check("q", q, torch.bfloat16, 4)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1] if v.dim() == 4 else -1
    _check("k", k, torch.bfloat16, shape=q.shape)
    _check("v", v, torch.bfloat16, shape=(B, T, H, Dv))
    _check("g", g, torch.float32, shape=q.shape)
    _check("beta", beta, torch.float32, shape=(B, T, H))
    state_shape = (B, H, Dk, Dv)
    if initial_state is not None:
        _check("initial_state", initial_state, None, shape=state_shape)
    if out is not None:
        _check("out", out, torch.bfloat16, shape=(B, T, H, Dv))
    if final_state is not None:
        _check("final_state", final_state, None, shape=state_shape)
    lib = load_library()
    need = int(lib.kda_fwd_segmented_workspace(int(B), int(T), int(H), int(segment_len)))
    if workspace is not None:
        _check("workspace", workspace, torch.uint8, 1)
    dev = _check_devices(q=q, k=k, v=v, g=g, beta=beta, initial_state=initial_state, out=out,
                         final_state=final_state, workspace=workspace)
    if out is None:
        out = torch.empty((B, T, H, Dv), dtype=torch.bfloat16, device=dev)
    if final_state is None and final_state_dtype is not None:
        final_state = torch.empty(state_shape, dtype=final_state_dtype, device=dev)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if scale is None:
        scale = Dk ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    ic, fc = _dtype_code(initial_state), _dtype_code(final_state)
    with torch.cuda.device(dev):
        st = lib.kda_fwd_segmented(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), int(B), int(T),
                                   int(H), int(Dk), int(Dv), _ptr(initial_state), ic if ic >= 0 else 99,
                                   _ptr(final_state), fc if fc >= 0 else 99, _ptr(out), int(segment_len),
                                   _ptr(workspace), int(workspace.numel()), ctypes.c_void_p(int(stream)))
    if st != 0:
        raise KdaError(st, lib.kda_status_string(st).decode())
    return out, final_state


def kda_bwd(q, k, v, g, beta, dout, scale: float | None = None, cu_seqlens=None, initial_state=None,
            dfinal_state=None, want_dinitial_state: bool = True, workspace=None, stream=None):
    """Gradients of sum(dout * out) + sum(dfinal_state * final_state) of ``kda_fwd`` with
    respect to q, k, v, g, beta and the initial state (see include/kda.h, kda_bwd).

    Inputs as for ``kda_fwd`` (fp32 per-channel g), plus dout bf16 [B, T, H, 128] and
    dfinal_state fp32 [N, H, 128, 128] or None. Returns a dict of fp32 tensors: dq, dk, dv,
    dg [B, T, H, 128], dbeta [B, T, H] and dh0 [N, H, 128, 128] (None unless asked).
    ``workspace`` (uint8, at least ``bwd_workspace_bytes(...)``) is allocated when not given."""
    import torch
    _check("q", q, torch.bfloat16, 4)
    B, T, H, Dk = q.shape
    Dv = v.shape[-1] if v.dim() == 4 else -1
    _check("k", k, torch.bfloat16, shape=q.shape)
    _check("v", v, torch.bfloat16, shape=(B, T, H, Dv))
    _check("g", g, torch.float32, shape=q.shape)
    _check("beta", beta, torch.float32, shape=(B, T, H))
    _check("dout", dout, torch.bfloat16, shape=(B, T, H, Dv))
    if cu_seqlens is not None:
        _check("cu_seqlens", cu_seqlens, torch.int32, 1)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    state_shape = (N, H, Dk, Dv)
    if initial_state is not None:
        _check("initial_state", initial_state, None, shape=state_shape)
    if dfinal_state is not None:
        _check("dfinal_state", dfinal_state, torch.float32, shape=state_shape)
    if workspace is not None:
        _check("workspace", workspace, torch.uint8, 1)
    dev = _check_devices(q=q, k=k, v=v, g=g, beta=beta, dout=dout, cu_seqlens=cu_seqlens,
                         initial_state=initial_state, dfinal_state=dfinal_state, workspace=workspace)
    lib = load_library()
    rows = T if cu_seqlens is not None else B * T
    if workspace is None:
        workspace = torch.empty(max(1, int(lib.kda_bwd_workspace(int(rows), int(N), int(H)))),
                                dtype=torch.uint8, device=dev)
    out = {n: torch.empty((B, T, H, Dk if n != "dv" else Dv), dtype=torch.float32, device=dev)
           for n in ("dq", "dk", "dv", "dg")}
    out["dbeta"] = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    out["dh0"] = torch.empty(state_shape, dtype=torch.float32, device=dev) if want_dinitial_state else None
    if scale is None:
        scale = Dk ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    ic = _dtype_code(initial_state)
    with torch.cuda.device(dev):
        st = lib.kda_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(cu_seqlens), int(N),
                         int(B), int(T), int(H), int(Dk), int(Dv), _ptr(initial_state), ic if ic >= 0 else 99,
                         _ptr(dout), _ptr(dfinal_state), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                         _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dh0"]), _ptr(workspace),
                         int(workspace.numel()), ctypes.c_void_p(int(stream)))
    if st != 0:
        raise KdaError(st, lib.kda_status_string(st).decode())
    return out


def bwd_workspace_bytes(total_tokens: int, num_seqs: int, num_heads: int) -> int:
    """Bytes of workspace kda_bwd needs."""
    return int(load_library().kda_bwd_workspace(int(total_tokens), int(num_seqs), int(num_heads)))


def segmented_workspace_bytes(batch: int, seq_len: int, num_heads: int, segment_len: int) -> int:
    """Bytes of workspace kda_fwd_segmented needs (0 for a bad segment_len)."""
    return int(load_library().kda_fwd_segmented_workspace(int(batch), int(seq_len), int(num_heads),
                                                          int(segment_len)))


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
    B, H, Dk = q.shape
    Dv = v.shape[-1] if v.dim() == 3 else -1
    _check("k", k, torch.bfloat16, shape=q.shape)
    _check("v", v, torch.bfloat16, shape=(B, H, Dv))
    _check("g", g, torch.float32, shape=q.shape)
    _check("beta", beta, torch.float32, shape=(B, H))
    state_shape = (B, H, Dk, Dv)
    if state_in is not None:
        _check("state_in", state_in, None, shape=state_shape)
    if state_out is not None:
        _check("state_out", state_out, None, shape=state_shape)
    if out is not None:
        _check("out", out, torch.bfloat16, shape=(B, H, Dv))
    dev = _check_devices(q=q, k=k, v=v, g=g, beta=beta, state_in=state_in, state_out=state_out, out=out)
    if state_out is None and state_dtype is not None:
        state_out = torch.empty(state_shape, dtype=state_dtype, device=dev)
    if state_in is not None and state_out is not None and state_in.dtype != state_out.dtype:
        raise ValueError("state_in and state_out must have the same dtype")
    st_t = state_in if state_in is not None else state_out
    code = _dtype_code(st_t)
    if out is None:
        out = torch.empty((B, H, Dv), dtype=torch.bfloat16, device=dev)
    if scale is None:
        scale = Dk ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), int(B), int(H),
                            int(Dk), int(Dv), _ptr(state_in), _ptr(state_out), code if code >= 0 else 99,
                            _ptr(out), ctypes.c_void_p(int(stream)))
    if st != 0:
        raise KdaError(st, lib.kda_status_string(st).decode())
    return out, state_out
