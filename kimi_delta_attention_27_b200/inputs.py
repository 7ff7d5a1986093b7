"""Seeded synthetic inputs for the KDA forward pass.

This module holds no arithmetic of the method: it only draws random tensors
with the shapes and value distributions of the workloads below, for the CUDA
library, its tests, the oracle tests and the benchmark alike.

Recipe (all draws from one ``torch.Generator`` per tensor, seeded by
``seed * 16 + tensor_index``, filled in slices of ``_SLICE`` tokens so that a
million-token workload needs no giant temporaries):

* q, k : float32 N(0, 1) per element, L2-normalised over the 128 channels of
  each (token, head), then rounded to bf16;
* v    : float32 N(0, 1) rounded to bf16;
* g    : log-decay per (token, head, channel), float32 logsigmoid(N(mu, 1));
* beta : per (token, head), float32 sigmoid(N(0, 1));
* h0   : per (sequence, head), N(0, 0.1) (mean 0, std 0.1) in the state dtype;
* varlen lengths: integers uniform in [lo, hi] from numpy's PCG64 seeded with
  ``seed``, packed back to back behind int32 ``cu_seqlens``.

The pages print no workload data; these stand in for the prefill shapes they
talk about (head dim 128, chunk 64, packed variable-length batches, 1M-token
context).
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

HEAD_DIM = 128
_SLICE = 1 << 16

# name -> workload. ``lengths`` is None for fixed-length batches (B rows of T
# tokens, no cu_seqlens) or (count, lo, hi) for a packed varlen batch (B = 1).
CONFIGS = {
    "t256_h1": dict(B=1, T=256, H=1, lengths=None, g_mu=3.0,
                    init=None, final="fp32", seed=0),
    "t4k_h32": dict(B=1, T=4096, H=32, lengths=None, g_mu=3.0,
                    init="fp32", final="fp32", seed=1),
    "varlen16_h32": dict(B=1, T=None, H=32, lengths=(16, 512, 16384), g_mu=3.0,
                         init="fp32", final="fp32", seed=2),
    "b8_t8k_h32": dict(B=8, T=8192, H=32, lengths=None, g_mu=5.0,
                       init="bf16", final="bf16", seed=3),
    "t1m_h32": dict(B=1, T=1 << 20, H=32, lengths=None, g_mu=3.0,
                    init=None, final="fp32", seed=4),
}

_DT = {None: None, "fp32": torch.float32, "bf16": torch.bfloat16}


def varlen_lengths(count: int, lo: int, hi: int, seed: int) -> list[int]:
    rng = np.random.Generator(np.random.PCG64(seed))
    return [int(x) for x in rng.integers(lo, hi, size=count, endpoint=True)]


def _gen(device, seed: int, idx: int) -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed * 16 + idx)
    return gen


def _fill(shape, device, seed, idx, make):
    """Allocate ``shape`` (tokens on dim 1) and fill it slice by slice."""
    gen = _gen(device, seed, idx)
    out = None
    T = shape[1]
    for t0 in range(0, max(T, 1), _SLICE):
        t1 = min(T, t0 + _SLICE)
        sl = make((shape[0], t1 - t0) + tuple(shape[2:]), gen)
        if out is None:
            out = torch.empty(shape, dtype=sl.dtype, device=device)
        out[:, t0:t1] = sl
    if out is None:
        out = make(tuple(shape), gen)
    return out


def _unit_bf16(shape, gen):
    x = torch.randn(shape, generator=gen, device=gen.device, dtype=torch.float32)
    x = x / x.norm(dim=-1, keepdim=True)
    return x.to(torch.bfloat16)


def make_inputs(cfg, device="cpu", **overrides) -> dict:
    """Build one workload.

    ``cfg`` is a name from ``CONFIGS`` or a dict with the same keys; keyword
    overrides replace keys (e.g. ``T=128`` or ``H=2`` for reduced parity cases).
    Returns a dict with q, k, v (bf16), g, beta (fp32), cu_seqlens (int32 or
    None), h0 (or None), final_dtype (torch dtype or None), scale (the float32
    value 1/sqrt(128) as a Python float), B, T (tokens per row), H, N (number of
    sequences), lengths (list).
    """
    c = dict(CONFIGS[cfg]) if isinstance(cfg, str) else dict(cfg)
    c.update(overrides)
    H, seed = int(c["H"]), int(c["seed"])
    D = HEAD_DIM
    if c.get("lengths") is not None:
        count, lo, hi = c["lengths"]
        lengths = varlen_lengths(count, lo, hi, seed)
        B, T = 1, int(sum(lengths))
        cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32, device=device)
        N = len(lengths)
    else:
        B, T = int(c["B"]), int(c["T"])
        lengths = [T] * B
        cu = None
        N = B
    g_mu = float(c["g_mu"])

    q = _fill((B, T, H, D), device, seed, 0, _unit_bf16)
    k = _fill((B, T, H, D), device, seed, 1, _unit_bf16)
    v = _fill((B, T, H, D), device, seed, 2,
              lambda s, gen: torch.randn(s, generator=gen, device=gen.device).to(torch.bfloat16))
    g = _fill((B, T, H, D), device, seed, 3,
              lambda s, gen: F.logsigmoid(torch.randn(s, generator=gen, device=gen.device) + g_mu))
    beta = _fill((B, T, H), device, seed, 4,
                 lambda s, gen: torch.sigmoid(torch.randn(s, generator=gen, device=gen.device)))
    h0 = None
    if c.get("init") is not None:
        gen = _gen(device, seed, 5)
        h0 = (0.1 * torch.randn((N, H, D, D), generator=gen, device=device)).to(_DT[c["init"]])
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu, h0=h0,
                final_dtype=_DT[c.get("final")], scale=float(np.float32(1.0 / math.sqrt(D))),
                B=B, T=T, H=H, N=N, lengths=lengths, name=cfg if isinstance(cfg, str) else "custom")

