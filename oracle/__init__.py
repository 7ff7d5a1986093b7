"""fp64 CPU oracle for the Kimi Delta Attention forward pass (and its gradients).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``. The product package never imports
it, and it never imports the product package.

The arithmetic lives in ``kda_oracle.c`` (the token-by-token recurrence of the
Kimi Linear feature page, chapter 4, state-update equation). This module only
builds that file with gcc and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build(mutant: int = 0, out_path: str | None = None) -> str:
    """Compile the oracle with gcc. ``mutant`` != 0 plants one of the numbered
    mistakes (used only by the mutation tests) and requires ``out_path``."""
    if mutant and not out_path:
        raise ValueError("a mutant build needs its own output path")
    path = out_path or _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
           f"-DKDA_ORACLE_MUTANT={int(mutant)}", _SRC, "-o", path, "-lm"]
    subprocess.run(cmd, check=True)
    return path


def _load(path: str | None = None):
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
        _declare(lib)
        return lib
    with _lock:
        if _lib is None:
            if (not os.path.exists(_LIB_PATH)
                    or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
                build()
            _lib = ctypes.CDLL(_LIB_PATH)
            _declare(_lib)
    return _lib


def _declare(lib):
    P = ctypes.c_void_p
    lib.kda_oracle_fwd.restype = ctypes.c_int
    lib.kda_oracle_fwd.argtypes = [P, P, P, P, P, ctypes.c_double, P, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   P, P, P, ctypes.c_int]
    i64 = ctypes.c_int64
    lib.kda_oracle_bwd.restype = ctypes.c_int
    lib.kda_oracle_bwd.argtypes = [P, P, P, P, P, ctypes.c_double, P, i64, i64, i64, i64,
                                   P, P, P, P, P, P, P, P, P, ctypes.c_int]


def _f32(x) -> np.ndarray:
    """Widen to a C-contiguous float32 numpy array (exact for bf16 and fp32)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float32).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def kda_oracle(q, k, v, g, beta, scale, cu_seqlens=None, h0=None, nthreads=None,
               lib_path: str | None = None):
    """Run the fp64 recurrence.

    q, k, g: [Ttot, H, Dk] (or [B, T, H, Dk] with ``cu_seqlens`` None: then the
    B rows are B independent sequences of length T); v: [..., Dv];
    beta: [Ttot, H] (or [B, T, H]); cu_seqlens: int sequence of N+1 offsets or
    None; h0: [N, H, Dk, Dv] or None. ``scale`` is used exactly as given
    (pass the float32 value the GPU call receives).

    Returns (out [same leading shape, Dv] float64, hT [N, H, Dk, Dv] float64).
    """
    qa, ka, va, ga, ba = (_f32(t) for t in (q, k, v, g, beta))
    lead = qa.shape[:-1]
    if cu_seqlens is None:
        if qa.ndim == 4:
            B, T = qa.shape[0], qa.shape[1]
        else:
            B, T = 1, qa.shape[0]
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int64))
    Dk, Dv = qa.shape[-1], va.shape[-1]
    H = qa.shape[-2]
    N = len(cu) - 1
    qa = qa.reshape(-1, H, Dk); ka = ka.reshape(-1, H, Dk); ga = ga.reshape(-1, H, Dk)
    va = va.reshape(-1, H, Dv); ba = ba.reshape(-1, H)
    Ttot = qa.shape[0]
    if cu[-1] != Ttot and cu_seqlens is not None and cu[-1] > Ttot:
        raise ValueError("cu_seqlens runs past the packed tensors")
    h0a = None if h0 is None else _f64(h0).reshape(N, H, Dk, Dv)
    out = np.zeros((Ttot, H, Dv), dtype=np.float64)
    hT = np.zeros((N, H, Dk, Dv), dtype=np.float64)
    nt = nthreads or os.cpu_count() or 1
    lib = _load(lib_path)
    P = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
    rc = lib.kda_oracle_fwd(P(qa), P(ka), P(va), P(ga), P(ba), float(scale), P(cu),
                            N, H, Dk, Dv, P(h0a), P(out), P(hT), int(nt))
    if rc != 0:
        raise ValueError("kda_oracle_fwd rejected its arguments")
    return out.reshape(*lead, Dv), hT


def _cu_of(qa, cu_seqlens):
    if cu_seqlens is None:
        B, T = (qa.shape[0], qa.shape[1]) if qa.ndim == 4 else (1, qa.shape[0])
        return np.arange(B + 1, dtype=np.int64) * T
    return np.ascontiguousarray(np.asarray(
        cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))


def kda_oracle_bwd(q, k, v, g, beta, scale, dout, cu_seqlens=None, h0=None, dhT=None, nthreads=None,
                   lib_path: str | None = None):
    """Gradients of ``sum(dout * out) + sum(dhT * hT)`` of the fp64 recurrence.

    Same inputs and layouts as ``kda_oracle`` (taken as float64 here, exactly), plus ``dout``
    shaped like ``out`` and ``dhT`` shaped like ``hT`` (or None). Returns a dict of float64
    arrays: dq, dk, dv, dg, dbeta shaped like their inputs, and dh0 [N, H, Dk, Dv].
    """
    qa, ka, va, ga, ba, da = (_f64(t) for t in (q, k, v, g, beta, dout))
    cu = _cu_of(qa, cu_seqlens)
    Dk, Dv, H = qa.shape[-1], va.shape[-1], qa.shape[-2]
    N = len(cu) - 1
    shapes = dict(dq=qa.shape, dk=ka.shape, dv=va.shape, dg=ga.shape, dbeta=ba.shape)
    qa, ka, ga = (a.reshape(-1, H, Dk) for a in (qa, ka, ga))
    va, da = va.reshape(-1, H, Dv), da.reshape(-1, H, Dv)
    ba = ba.reshape(-1, H)
    if cu[-1] > qa.shape[0]:
        raise ValueError("cu_seqlens runs past the packed tensors")
    h0a = None if h0 is None else _f64(h0).reshape(N, H, Dk, Dv)
    dhTa = None if dhT is None else _f64(dhT).reshape(N, H, Dk, Dv)
    out = {n: np.zeros(qa.shape if n in ("dq", "dk", "dg") else (va.shape if n == "dv" else ba.shape))
           for n in ("dq", "dk", "dv", "dg", "dbeta")}
    dh0 = np.zeros((N, H, Dk, Dv))
    lib = _load(lib_path)
    P = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
    rc = lib.kda_oracle_bwd(P(qa), P(ka), P(va), P(ga), P(ba), float(scale), P(cu), N, H, Dk, Dv,
                            P(h0a), P(da), P(dhTa), P(out["dq"]), P(out["dk"]), P(out["dv"]),
                            P(out["dg"]), P(out["dbeta"]), P(dh0), int(nthreads or os.cpu_count() or 1))
    if rc != 0:
        raise ValueError("kda_oracle_bwd rejected its arguments")
    res = {n: a.reshape(shapes[n]) for n, a in out.items()}
    res["dh0"] = dh0
    return res
