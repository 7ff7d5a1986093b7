"""GPU parity of the input variants (kda_fwd_ex, through the binding) against the fp64
oracle: a bf16 gate, a per-token (Gated DeltaNet) gate, q and k normalised in the kernel,
and the gate's log-sigmoid taken in the kernel. The oracle gets the variant's own
definition applied to the same inputs: the bf16 gate widened, the per-token gate copied
to every channel, q / ||q|| and k / ||k|| and logsigmoid(x) in fp64.
"""
import numpy as np
import pytest
import torch

import oracle
import kimi_delta_attention_27_b200 as kda
from kimi_delta_attention_27_b200.inputs import make_inputs
from kda_testutil import OUT_TOL, STATE_TOL, record, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kimi_delta_attention_27_b200 import build
    build.build()


def ragged(lengths, H=2, seed=5, g_mu=3.0):
    T = sum(lengths)
    inp = make_inputs({"B": 1, "T": T, "H": H, "lengths": None, "g_mu": g_mu, "init": None,
                       "final": "fp32", "seed": seed}, device="cpu")
    inp["cu_seqlens"] = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    gen = torch.Generator().manual_seed(seed)
    inp["h0"] = 0.1 * torch.randn((len(lengths), H, 128, 128), generator=gen)
    return inp


def logsigmoid64(x):
    x = np.asarray(x, dtype=np.float64)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def unit64(x):
    x = np.asarray(x, dtype=np.float64)
    n = np.sqrt((x * x).sum(-1, keepdims=True))
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)


def run_and_check(inp, g_kernel, g_oracle, q_oracle=None, k_oracle=None, **flags):
    dev = {n: inp[n].cuda() for n in ("q", "k", "v", "beta", "cu_seqlens", "h0")}
    out, hT = kda.kda_fwd(dev["q"], dev["k"], dev["v"], g_kernel.cuda(), dev["beta"], inp["scale"],
                          cu_seqlens=dev["cu_seqlens"], initial_state=dev["h0"],
                          final_state_dtype=torch.float32, **flags)
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    q = inp["q"][0].float().numpy() if q_oracle is None else q_oracle
    k = inp["k"][0].float().numpy() if k_oracle is None else k_oracle
    eo, eh = oracle.kda_oracle(q, k, inp["v"][0].float(), np.asarray(g_oracle)[0], inp["beta"][0], inp["scale"],
                               cu_seqlens=inp["cu_seqlens"].numpy().astype(np.int64), h0=inp["h0"].double())
    go = out[0].float().cpu().numpy()
    r_out, r_state = rel(go, eo), rel(hT.cpu().numpy(), eh)
    record(r_out, r_state)
    assert np.isfinite(go).all()
    assert r_out <= OUT_TOL and r_state <= STATE_TOL[torch.float32], (r_out, r_state)


LENGTHS = [300, 1, 64, 130, 0, 77]


@pytest.mark.parametrize("g_mu", [3.0, -4.0])
def test_bf16_gate(g_mu):
    inp = ragged(LENGTHS, g_mu=g_mu)
    gb = inp["g"].to(torch.bfloat16)
    run_and_check(inp, gb, gb.double().numpy())


@pytest.mark.parametrize("g_mu", [3.0, -4.0])
def test_per_token_gate_is_gated_deltanet(g_mu):
    inp = ragged(LENGTHS, g_mu=g_mu)
    gs = inp["g"][..., 0].contiguous()            # one log alpha per token and head
    g_all = gs[..., None].expand(*gs.shape, 128).double().numpy()
    run_and_check(inp, gs, g_all)


def test_l2_normalised_in_the_kernel():
    inp = ragged(LENGTHS)
    gen = torch.Generator().manual_seed(11)
    # unnormalised bf16 keys and queries of varied norms, one zero key
    qr = (torch.randn(inp["q"].shape, generator=gen) * 3.0).to(torch.bfloat16)
    kr = (torch.randn(inp["k"].shape, generator=gen) * 0.2).to(torch.bfloat16)
    kr[0, 5, 1] = 0
    inp["q"], inp["k"] = qr, kr
    run_and_check(inp, inp["g"], inp["g"].double().numpy(), q_oracle=unit64(qr[0].float().numpy()),
                  k_oracle=unit64(kr[0].float().numpy()), l2norm_qk=True)


@pytest.mark.parametrize("kind", ["fp32", "bf16", "per_token"])
def test_logsigmoid_in_the_kernel(kind):
    inp = ragged(LENGTHS)
    gen = torch.Generator().manual_seed(12)
    x = torch.randn(inp["g"].shape, generator=gen) + 3.0
    if kind == "bf16":
        x = x.to(torch.bfloat16)
    if kind == "per_token":
        x = x[..., 0].contiguous()
        ref = logsigmoid64(x.double().numpy())[..., None].repeat(128, axis=-1)
    else:
        ref = logsigmoid64(x.double().numpy())
    run_and_check(inp, x, ref, gate_logsigmoid=True)


def test_all_fused_with_strong_decay():
    # pre-activations near -4: a log-decay of about -4 per token, every chunk on the sub-block path
    inp = ragged(LENGTHS)
    gen = torch.Generator().manual_seed(13)
    x = (torch.randn(inp["g"].shape, generator=gen) - 4.0).to(torch.bfloat16)
    qr = (torch.randn(inp["q"].shape, generator=gen) * 2.0).to(torch.bfloat16)
    kr = (torch.randn(inp["k"].shape, generator=gen) * 2.0).to(torch.bfloat16)
    inp["q"], inp["k"] = qr, kr
    run_and_check(inp, x, logsigmoid64(x.double().numpy()), q_oracle=unit64(qr[0].float().numpy()),
                  k_oracle=unit64(kr[0].float().numpy()), l2norm_qk=True, gate_logsigmoid=True)
