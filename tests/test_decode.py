"""kda_decode, the single-token step, against the fp64 oracle.

A decode step is the recurrence for one token with a state carried in and out,
so the oracle of the forward pass pins it directly: steps run one after another
through kda_decode must match the oracle run over the same tokens as one
sequence. The CPU tests check argument validation, which happens before the
device is touched.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import kimi_delta_attention_27_b200 as kda
from kimi_delta_attention_27_b200.inputs import make_inputs
from kda_testutil import OUT_TOL, STATE_TOL, rel

OK, NULL_PTR, BAD_SHAPE, STATE_DTYPE, CUDA, BAD_ALIGNMENT, STATE_OVERLAP = 0, 1, 2, 4, 5, 7, 11
BF16, FP32 = 1, 2

# A fake, 16-byte-aligned, never-dereferenced address: every CPU call below is
# rejected (or stops at the device query) before any device access.
FAKE = 0x10000


@pytest.fixture(scope="module")
def lib():
    from kimi_delta_attention_27_b200 import build
    build.build()
    return kda.load_library()


def call(lib, q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, batch=2, H=2, dk=128, dv=128, sin=None, sout=None,
         dt=FP32, out=FAKE):
    P = lambda a: None if a is None else ctypes.c_void_p(a)
    return lib.kda_decode(P(q), P(k), P(v), P(g), P(beta), 1.0, batch, H, dk, dv, P(sin), P(sout), dt, P(out),
                          None)


def test_decode_rejects_bad_arguments(lib):
    assert call(lib, dk=64) == BAD_SHAPE
    assert call(lib, dv=256) == BAD_SHAPE
    assert call(lib, batch=-1) == BAD_SHAPE
    assert call(lib, H=0) == BAD_SHAPE
    assert call(lib, sin=FAKE, dt=0) == STATE_DTYPE
    assert call(lib, sout=FAKE, dt=7) == STATE_DTYPE
    assert call(lib, q=None) == NULL_PTR
    assert call(lib, out=None) == NULL_PTR
    assert call(lib, v=FAKE + 8) == BAD_ALIGNMENT
    assert call(lib, beta=FAKE + 2) == BAD_ALIGNMENT
    assert call(lib, sout=FAKE + 8) == BAD_ALIGNMENT
    # distinct state buffers that overlap: 4 pairs of 64 KiB fp32 states, 128 KiB apart
    assert call(lib, sin=FAKE, sout=FAKE + 2 * 65536) == STATE_OVERLAP
    assert call(lib, sin=FAKE + 3 * 65536, sout=FAKE, dt=FP32) == STATE_OVERLAP
    msg = kda.status_string(STATE_OVERLAP)
    assert msg.startswith("KDA_ERR_STATE_OVERLAP")


def test_decode_empty_batch_is_a_no_op(lib):
    assert call(lib, batch=0, q=None, k=None, v=None, g=None, beta=None, out=None) == OK


def test_decode_in_place_and_adjacent_states_pass_validation(lib):
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    # the same pointer in and out is allowed; without a device the call stops at the device query
    assert call(lib, sin=FAKE, sout=FAKE) == CUDA
    # adjacent bf16 state buffers (4 x 32 KiB) do not overlap
    assert call(lib, sin=FAKE, sout=FAKE + 4 * 32768, dt=BF16) == CUDA


# ---------------------------------------------------------------- GPU

def decode_inputs(B, H, steps, state, seed, g_mu=3.0):
    """B requests x H heads, `steps` tokens each, with a random initial state (the
    workloads' N(0, 0.1) recipe) of the given dtype."""
    return make_inputs({"B": B, "T": steps, "H": H, "lengths": None, "g_mu": g_mu, "init": state,
                        "final": state, "seed": seed}, device="cuda")


def step_tensors(inp, t):
    return tuple(inp[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta"))


def oracle_over(inp):
    q, k, v, g = (inp[n].cpu().float() for n in ("q", "k", "v", "g"))
    return oracle.kda_oracle(q, k, v, g, inp["beta"].cpu(), inp["scale"], h0=inp["h0"].cpu().double())


@pytest.mark.gpu
@pytest.mark.parametrize("state", ["fp32", "bf16"])
def test_decode_steps_match_oracle(lib, state):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    steps = 4
    inp = decode_inputs(B=6, H=5, steps=steps, state=state, seed=70)
    ref_out, ref_hT = oracle_over(inp)
    S = inp["h0"].clone()
    for t in range(steps):
        q, k, v, g, beta = step_tensors(inp, t)
        out, _ = kda.kda_decode(q, k, v, g, beta, state_in=S, state_out=S, scale=inp["scale"])
        torch.cuda.synchronize()
        r = rel(out.float().cpu().numpy(), ref_out[:, t])
        assert r <= OUT_TOL, f"step {t}: out rel err {r:.3e}"
    r = rel(S.float().cpu().numpy(), ref_hT)
    assert r <= STATE_TOL[S.dtype], f"state rel err {r:.3e}"


@pytest.mark.gpu
def test_decode_separate_state_buffer_equals_in_place(lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = decode_inputs(B=3, H=4, steps=1, state="fp32", seed=71)
    q, k, v, g, beta = step_tensors(inp, 0)
    out_a, s_a = kda.kda_decode(q, k, v, g, beta, state_in=inp["h0"], state_dtype=torch.float32,
                                scale=inp["scale"])
    s_b = inp["h0"].clone()
    out_b, _ = kda.kda_decode(q, k, v, g, beta, state_in=s_b, state_out=s_b, scale=inp["scale"])
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
    assert torch.equal(s_a, s_b)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_from_zero_state(lib, dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = decode_inputs(B=4, H=3, steps=1, state="fp32", seed=72)
    q, k, v, g, beta = step_tensors(inp, 0)
    out, s = kda.kda_decode(q, k, v, g, beta, state_dtype=dtype, scale=inp["scale"])
    zeros = torch.zeros_like(s)
    out_z, s_z = kda.kda_decode(q, k, v, g, beta, state_in=zeros, state_dtype=dtype, scale=inp["scale"])
    torch.cuda.synchronize()
    assert torch.equal(out, out_z) and torch.equal(s, s_z)
    ref_out, ref_hT = oracle.kda_oracle(*(inp[n].cpu().float() for n in ("q", "k", "v", "g")),
                                        inp["beta"].cpu(), inp["scale"])
    assert rel(out.float().cpu().numpy(), ref_out[:, 0]) <= OUT_TOL
    assert rel(s.float().cpu().numpy(), ref_hT) <= STATE_TOL[dtype]


@pytest.mark.gpu
def test_decode_continues_a_prefill(lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # kda_fwd over 200 tokens, then one decode step for token 200: the oracle over 201 tokens
    inp = make_inputs({"B": 2, "T": 201, "H": 4, "lengths": None, "g_mu": 3.0, "init": "fp32",
                       "final": "fp32", "seed": 73}, device="cuda")
    pre = {n: inp[n][:, :200].contiguous() for n in ("q", "k", "v", "g", "beta")}
    _, S = kda.kda_fwd(pre["q"], pre["k"], pre["v"], pre["g"], pre["beta"], inp["scale"],
                       initial_state=inp["h0"], final_state_dtype=torch.float32)
    q, k, v, g, beta = step_tensors(inp, 200)
    out, _ = kda.kda_decode(q, k, v, g, beta, state_in=S, state_out=S, scale=inp["scale"])
    torch.cuda.synchronize()
    ref_out, ref_hT = oracle_over(inp)
    assert rel(out.float().cpu().numpy(), ref_out[:, 200]) <= OUT_TOL
    assert rel(S.cpu().numpy(), ref_hT) <= STATE_TOL[torch.float32]


@pytest.mark.gpu
def test_decode_serving_batch(lib):
    """256 requests x 32 heads, fp32 states, one step: every (request, head) checked."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = decode_inputs(B=256, H=32, steps=1, state="fp32", seed=74)
    q, k, v, g, beta = step_tensors(inp, 0)
    S = inp["h0"].clone()
    out, _ = kda.kda_decode(q, k, v, g, beta, state_in=S, state_out=S, scale=inp["scale"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    ref_out, ref_hT = oracle_over(inp)
    assert rel(out.float().cpu().numpy(), ref_out[:, 0]) <= OUT_TOL
    assert rel(S.cpu().numpy(), ref_hT) <= STATE_TOL[torch.float32]
    # and per pair, so that one wrong (request, head) cannot hide behind the global maximum
    o = out.float().cpu().numpy()
    err = np.abs(o - ref_out[:, 0]).max(axis=-1) / np.maximum(np.abs(ref_out[:, 0]).max(axis=-1), 1e-30)
    assert float(err.max()) <= 5 * OUT_TOL
