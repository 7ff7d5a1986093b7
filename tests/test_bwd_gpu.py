"""GPU parity of kda_bwd, the backward pass, against the fp64 backward oracle
(kda_oracle_bwd, itself pinned by finite differences in test_oracle_bwd.py): every
gradient element by element, on the same seeded inputs and cotangents.

Bar: max|d grad| / max|grad| <= 1e-3 for each of dq, dk, dv, dg, dbeta, dh0. The kernel
works in fp32 from inputs the oracle sees exactly (bf16 q, k, v, dout; fp32 g, beta,
states), so the gap is fp32 rounding carried through the state's reverse recurrence;
1e-3 leaves room for 1e4 sequential chunk steps at fp32 precision without admitting a
wrong term, which errs by O(1) relative.
"""
import numpy as np
import pytest
import torch

import oracle
import kimi_delta_attention_27_b200 as kda
from kimi_delta_attention_27_b200.inputs import make_inputs
from kda_testutil import record, rel

pytestmark = pytest.mark.gpu
BWD_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kimi_delta_attention_27_b200 import build
    build.build()


def with_cotangents(inp, seed):
    gen = torch.Generator().manual_seed(seed)
    inp["dout"] = torch.randn(inp["v"].shape, generator=gen).to(torch.bfloat16)
    N = inp["N"]
    inp["dhT"] = torch.randn((N, inp["H"], 128, 128), generator=gen)
    return inp


def check_bwd(inp, heads=None, note=""):
    dev = {n: (inp[n].cuda() if inp.get(n) is not None else None)
           for n in ("q", "k", "v", "g", "beta", "cu_seqlens", "h0", "dout", "dhT")}
    got = kda.kda_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["dout"], inp["scale"],
                      cu_seqlens=dev["cu_seqlens"], initial_state=dev["h0"], dfinal_state=dev["dhT"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    sel = (lambda t: t) if heads is None else (lambda t: t[:, :, heads])
    cu = inp["cu_seqlens"]
    if cu is not None:
        lead = lambda t: sel(t)[0]
        cu_np = cu.numpy().astype(np.int64)
    else:
        lead = sel
        cu_np = None
    h0 = inp["h0"]
    if h0 is not None:
        h0 = h0.double()
        if heads is not None:
            h0 = h0[:, heads]
    dhT = inp["dhT"].double() if heads is None else inp["dhT"].double()[:, heads]
    ref = oracle.kda_oracle_bwd(*(lead(inp[n]).double() for n in ("q", "k", "v", "g", "beta")), inp["scale"],
                                lead(inp["dout"]).double(), cu_seqlens=cu_np, h0=h0, dhT=dhT)
    errs = {}
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        g = got[n].cpu()
        g = (g[:, :, heads] if heads is not None else g)
        g = g[0] if cu is not None else g
        errs[n] = rel(g.numpy(), ref[n].reshape(g.shape))
    dh0 = got["dh0"].cpu() if heads is None else got["dh0"].cpu()[:, heads]
    errs["dh0"] = rel(dh0.numpy(), ref["dh0"])
    record(max(errs.values()), None, note + " " + " ".join(f"{k} {v:.2e}" for k, v in errs.items()))
    for n, e in errs.items():
        assert np.isfinite(e) and e <= BWD_TOL, f"{n}: {e:.3e}"
    return errs


def varlen(lengths, H=2, seed=31, g_mu=3.0, init="fp32"):
    inp = make_inputs({"B": 1, "T": sum(lengths), "H": H, "lengths": None, "g_mu": g_mu, "init": None,
                       "final": "fp32", "seed": seed}, device="cpu")
    inp["cu_seqlens"] = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    inp["N"] = len(lengths)
    if init is not None:
        gen = torch.Generator().manual_seed(seed + 1)
        inp["h0"] = (0.1 * torch.randn((len(lengths), H, 128, 128), generator=gen)).to(
            torch.float32 if init == "fp32" else torch.bfloat16)
    return with_cotangents(inp, seed + 2)


def test_ragged_varlen():
    check_bwd(varlen([70, 1, 0, 64, 65, 200, 17]), note="ragged varlen")


def test_bf16_initial_state_and_no_initial_state():
    check_bwd(varlen([130, 40], init="bf16"), note="bf16 h0")
    check_bwd(varlen([130, 40], init=None), note="no h0")


@pytest.mark.parametrize("mu", [-1.0, -4.0])
def test_strong_decay(mu):
    check_bwd(varlen([300, 77], g_mu=mu), note=f"g=logsigmoid(N({mu},1))")


def test_t4k_h32_sampled_heads():
    inp = with_cotangents(make_inputs("t4k_h32", device="cpu"), 41)
    check_bwd(inp, heads=[0, 13, 31], note="t4k_h32 heads 0,13,31")


def test_fixed_batch_rows():
    inp = with_cotangents(make_inputs({"B": 3, "T": 333, "H": 2, "lengths": None, "g_mu": 3.0,
                                       "init": "fp32", "final": "fp32", "seed": 43}, device="cpu"), 44)
    check_bwd(inp, note="B=3 T=333")
