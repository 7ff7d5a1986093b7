"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs.

Bars: max|d out| / max|out| <= 1e-2 (bf16 outputs), final state <= 2e-3 when
fp32 and <= 1e-2 when bf16 (global maxima over each tensor).
"""
import numpy as np
import pytest
import torch

from kimi_delta_attention_27_b200.inputs import make_inputs
from kda_testutil import check, rel, run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kimi_delta_attention_27_b200 import build
    build.build()


def gpu_inputs(cfg, **kw):
    return to_device(make_inputs(cfg, device="cpu", **kw))


# -- the five workloads -------------------------------------------------------

def test_t256_h1_full():
    inp = gpu_inputs("t256_h1")
    out, hT = run_gpu(inp)
    check(inp, out, hT)


def test_t4k_h32_full():
    inp = gpu_inputs("t4k_h32")
    out, hT = run_gpu(inp)
    check(inp, out, hT)


def test_varlen16_h32_full_size_two_heads():
    inp = make_inputs("varlen16_h32", device="cuda")
    out, hT = run_gpu(inp)
    check(inp, out, hT, heads=[0, 17])


def test_b8_t8k_h32_full_size_two_heads_bf16_state():
    inp = make_inputs("b8_t8k_h32", device="cuda")
    out, hT = run_gpu(inp)
    assert hT.dtype == torch.bfloat16
    check(inp, out, hT, heads=[3, 30])


@pytest.mark.slow
def test_t1m_h32_full_size_sampled():
    """Full million-token run; the oracle checks every output and the final
    state of one head, and the first 16K tokens of all heads."""
    inp = make_inputs("t1m_h32", device="cuda")
    out, hT = run_gpu(inp)
    assert torch.isfinite(out.float()).all()
    check(inp, out, hT, heads=[7])
    check(inp, out, None, prefix=16384, state=False)
    del inp, out, hT
    torch.cuda.empty_cache()


# -- edge cases ---------------------------------------------------------------

def varlen_case(lengths, H=3, init="fp32", final="fp32", seed=7, **kw):
    from kimi_delta_attention_27_b200 import inputs as I
    cfg = dict(B=1, T=None, H=H, lengths=None, g_mu=kw.pop("g_mu", 3.0), init=init, final=final,
               seed=seed)
    T = sum(lengths)
    inp = make_inputs(cfg, device="cpu", T=T, B=1)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    inp["cu_seqlens"] = cu
    inp["N"] = len(lengths)
    if init is not None:
        gen = torch.Generator().manual_seed(seed)
        inp["h0"] = (0.1 * torch.randn((len(lengths), H, 128, 128), generator=gen)).to(I._DT[init])
    return to_device(inp)


@pytest.mark.parametrize("lengths", [[0, 1, 63, 64, 65, 130, 0, 200], [1], [64, 64], [257, 3]])
def test_varlen_ragged(lengths):
    inp = varlen_case(lengths)
    out, hT = run_gpu(inp)
    check(inp, out, hT)
    # empty sequences hand back their initial state exactly
    for s, L in enumerate(lengths):
        if L == 0:
            assert torch.equal(hT[s], inp["h0"][s])


@pytest.mark.parametrize("init,final", [(None, "fp32"), (None, "bf16"), ("bf16", "bf16"),
                                        ("fp32", None), (None, None)])
def test_state_dtypes(init, final):
    inp = varlen_case([100, 37], init=init, final=final)
    out, hT = run_gpu(inp, final=final is not None)
    if final is None:
        assert hT is None
    check(inp, out, hT)


def test_fixed_batch_zero_length_rows():
    inp = gpu_inputs("t4k_h32", T=0, B=2, H=2)
    out, hT = run_gpu(inp)
    assert out.numel() == 0
    assert torch.equal(hT, inp["h0"])


def test_beta_zero_is_pure_decay():
    inp = gpu_inputs("t4k_h32", T=200, H=2)
    inp["beta"] = torch.zeros_like(inp["beta"])
    out, hT = run_gpu(inp)
    check(inp, out, hT)


def test_no_decay_is_deltanet():
    inp = gpu_inputs("t4k_h32", T=300, H=2)
    inp["g"] = torch.zeros_like(inp["g"])
    out, hT = run_gpu(inp)
    check(inp, out, hT)


def test_strong_decay():
    # logsigmoid(N(-1, 1)): about -1.3 per token and channel, so a 64-token chunk
    # spans a log-decay range near -80 on the fastest channels
    inp = gpu_inputs("t4k_h32", T=640, H=2, g_mu=-1.0)
    out, hT = run_gpu(inp)
    check(inp, out, hT)


# -- the whole gate range: any log alpha <= 0 ------------------------------------
# Chunks in which some channel decays by more than 2^-100 over half a chunk take the
# sub-block path; these cases put every chunk, or some chunks, there.

@pytest.mark.parametrize("mu", [-3.0, -6.0])
def test_very_strong_decay_every_chunk(mu):
    # logsigmoid(N(-3, 1)) is about -3 per token: about -200 over 64 tokens;
    # logsigmoid(N(-6, 1)) about -6 per token
    inp = gpu_inputs("t4k_h32", T=650, H=2, g_mu=mu)
    out, hT = run_gpu(inp)
    check(inp, out, hT, note=f"g=logsigmoid(N({mu},1))")


def test_one_channel_at_minus_20_per_token():
    inp = gpu_inputs("t4k_h32", T=650, H=3)
    inp["g"][..., 5] = -20.0
    out, hT = run_gpu(inp)
    check(inp, out, hT)


def test_zero_alpha_tokens():
    # alpha = 0 (g = -inf) on a run of tokens and channels: the state forgets those channels
    inp = gpu_inputs("t4k_h32", T=400, H=2)
    inp["g"][:, 100:140, :, 7:40] = float("-inf")
    out, hT = run_gpu(inp)
    check(inp, out, hT)


def test_strong_decay_in_some_chunks_only():
    # ordinary gates with bursts of fast decay: neighbouring chunks take different paths
    # inside one (sequence, head), on ragged varlen sequences
    inp = varlen_case([700, 130, 0, 321], H=3)
    g = inp["g"]
    for t0, t1 in [(70, 140), (300, 330), (700 + 30, 700 + 100), (830 + 250, 830 + 321)]:
        g[:, t0:t1, 1:, ::3] = -12.0
    out, hT = run_gpu(inp)
    check(inp, out, hT)


def test_malformed_cu_seqlens_is_reported():
    """A cu_seqlens table that does not run 0, ..., T without decreasing is detected on the
    device and reported by kda_device_error; the device keeps working afterwards."""
    import kimi_delta_attention_27_b200 as kda
    KDA_ERR_BAD_CU_SEQLENS = 12
    inp = varlen_case([100, 90, 60], H=2)
    assert kda.device_error() == 0
    for table in ([0, 100, 50, 250], [3, 100, 190, 250], [0, 100, 190, 240]):
        bad = dict(inp, cu_seqlens=torch.tensor(table, dtype=torch.int32, device="cuda"))
        run_gpu(bad)
        assert kda.device_error() == KDA_ERR_BAD_CU_SEQLENS, table
    out, hT = run_gpu(inp)
    assert kda.device_error() == 0
    check(inp, out, hT)


def test_split_call_resume_matches_single_call():
    inp = gpu_inputs("t4k_h32", T=1000, H=4)
    out, hT = run_gpu(inp)
    t0 = 333  # not a multiple of the chunk length
    a = dict(inp, q=inp["q"][:, :t0].contiguous(), k=inp["k"][:, :t0].contiguous(),
             v=inp["v"][:, :t0].contiguous(), g=inp["g"][:, :t0].contiguous(),
             beta=inp["beta"][:, :t0].contiguous())
    o1, h1 = run_gpu(a)
    b = dict(inp, q=inp["q"][:, t0:].contiguous(), k=inp["k"][:, t0:].contiguous(),
             v=inp["v"][:, t0:].contiguous(), g=inp["g"][:, t0:].contiguous(),
             beta=inp["beta"][:, t0:].contiguous(), h0=h1)
    o2, h2 = run_gpu(b)
    assert rel(torch.cat([o1, o2], 1).float().cpu(), out.float().cpu()) < 1e-2
    assert rel(h2.cpu(), hT.cpu()) < 2e-3
    check(inp, torch.cat([o1, o2], 1), h2)


def test_varlen_equals_fixed_rows():
    inp = gpu_inputs("t4k_h32", T=321, B=3, H=2)
    out, hT = run_gpu(inp)
    packed = dict(inp)
    for key in ("q", "k", "v", "g", "beta"):
        packed[key] = inp[key].reshape(1, 3 * 321, *inp[key].shape[2:])
    packed["cu_seqlens"] = torch.tensor([0, 321, 642, 963], dtype=torch.int32, device="cuda")
    out2, hT2 = run_gpu(packed)
    assert torch.equal(out2.reshape(out.shape), out)
    assert torch.equal(hT2, hT)


def test_deterministic():
    inp = gpu_inputs("t4k_h32", T=500, H=3)
    a = run_gpu(inp)
    b = run_gpu(inp)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_runs_on_a_side_stream():
    inp = gpu_inputs("t4k_h32", T=256, H=2)
    ref, _ = run_gpu(inp)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, _ = run_gpu(inp)
    s.synchronize()
    assert torch.equal(out, ref)
