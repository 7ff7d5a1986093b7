"""Shared helpers for the GPU parity tests: run the CUDA library through its
binding, run the oracle on the same inputs (optionally on a subset of heads
or a token prefix), and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import kimi_delta_attention_27_b200 as kda

OUT_TOL = 1e-2        # max|d out| / max|out| for bf16 outputs
STATE_TOL = {torch.float32: 2e-3, torch.bfloat16: 1e-2}


def rel(a, b) -> float:
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    den = float(np.abs(b).max()) if b.size else 0.0
    if den == 0.0:
        return float(np.abs(a - b).max()) if a.size else 0.0
    return float(np.abs(a - b).max() / den)


def to_device(inp: dict, device="cuda") -> dict:
    d = dict(inp)
    for key in ("q", "k", "v", "g", "beta", "cu_seqlens", "h0"):
        if d.get(key) is not None:
            d[key] = d[key].to(device)
    return d


def run_gpu(inp: dict, final=True):
    out, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["scale"],
                          cu_seqlens=inp["cu_seqlens"], initial_state=inp["h0"],
                          final_state_dtype=inp["final_dtype"] if final else None)
    torch.cuda.synchronize()
    return out, hT


def run_oracle(inp: dict, heads=None, prefix=None):
    """Oracle on the inputs; ``heads`` restricts to a list of heads (packed as
    separate heads), ``prefix`` to the first tokens of every row (fixed-length
    batches only). Returns (out [B, T', H', 128] fp64, hT [N, H', 128, 128])."""
    sel = (lambda t: t) if heads is None else (lambda t: t[:, :, heads])
    cut = (lambda t: t) if prefix is None else (lambda t: t[:, :prefix])
    q, k, v, g = (cut(sel(inp[n])).cpu().float().contiguous() for n in ("q", "k", "v", "g"))
    beta = cut(sel(inp["beta"])).cpu().contiguous()
    h0 = inp["h0"]
    if h0 is not None:
        h0 = h0.cpu().double()
        if heads is not None:
            h0 = h0[:, heads].contiguous()
    cu = inp["cu_seqlens"]
    if cu is not None:
        assert prefix is None
        cu = cu.cpu().numpy().astype(np.int64)
        return oracle.kda_oracle(q[0], k[0], v[0], g[0], beta[0], inp["scale"], cu_seqlens=cu,
                                 h0=h0)
    return oracle.kda_oracle(q, k, v, g, beta, inp["scale"], h0=h0)


def record(r_out, r_state, note=""):
    """Print the measured errors and, when KDA_PARITY_LOG names a file, append them to it
    (one line per check: test id, out error, state error), so that a run keeps its margins."""
    import os
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    st = "-" if r_state is None else f"{r_state:.3e}"
    line = f"{test}{(' ' + note) if note else ''}\tout {r_out:.3e}\tstate {st}"
    print(line)
    path = os.environ.get("KDA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(line + "\n")


def check(inp, out_gpu, hT_gpu, heads=None, prefix=None, state=True, out_tol=OUT_TOL, note=""):
    eo, eh = run_oracle(inp, heads=heads, prefix=prefix)
    og = out_gpu
    if heads is not None:
        og = og[:, :, heads]
    if prefix is not None:
        og = og[:, :prefix]
    og = og.float().cpu().numpy().reshape(eo.shape)
    r_out = rel(og, eo)
    r_state = None
    if state and hT_gpu is not None:
        hg = hT_gpu if heads is None else hT_gpu[:, heads]
        hg = hg.float().cpu().numpy()
        r_state = rel(hg, eh)
    record(r_out, r_state, note)
    if r_state is not None:
        assert r_state <= STATE_TOL[hT_gpu.dtype], f"state rel err {r_state:.3e}"
    assert np.isfinite(og).all(), "non-finite output"
    assert r_out <= out_tol, f"out rel err {r_out:.3e}"
    return r_out, r_state
