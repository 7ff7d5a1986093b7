"""kda_fwd_noalloc, the allocation-free entry point, against kda_fwd.

The file name sorts last so that pytest collects it after every other test
file; it also passes when run alone in a fresh process. The GPU tests call both
entry points through the C ABI (the ctypes binding) on the same seeded inputs,
twice in a row with different inputs, and require results identical to
kda_fwd's (and within the parity bars of the other GPU tests). The CPU tests check the size limit, which is rejected
before the device is touched.
"""
import ctypes

import pytest
import torch

import kimi_delta_attention_27_b200 as kda
from kimi_delta_attention_27_b200.inputs import make_inputs
from kda_testutil import OUT_TOL, STATE_TOL, rel

KDA_ERR_CUDA, KDA_ERR_NOALLOC_LIMIT = 5, 10

# A fake, 16-byte-aligned, never-dereferenced address: the CPU calls below are
# all rejected (or stop at the device query) before any device access.
FAKE = ctypes.c_void_p(0x10000)


@pytest.fixture(scope="module")
def lib():
    from kimi_delta_attention_27_b200 import build
    build.build()
    return kda.load_library()


def call_noalloc(lib, cu=None, num_seqs=0, batch=1, H=2):
    return lib.kda_fwd_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 1.0, cu, num_seqs, batch, 64, H, 128, 128,
                               None, 0, None, 0, FAKE, None)


def test_noalloc_rejects_more_pairs_than_its_scratch(lib):
    assert kda.NOALLOC_MAX_UNITS == 32
    assert call_noalloc(lib, batch=1, H=33) == KDA_ERR_NOALLOC_LIMIT
    assert call_noalloc(lib, batch=3, H=11) == KDA_ERR_NOALLOC_LIMIT
    assert call_noalloc(lib, cu=FAKE, num_seqs=5, H=7) == KDA_ERR_NOALLOC_LIMIT
    msg = kda.status_string(KDA_ERR_NOALLOC_LIMIT)
    assert msg.startswith("KDA_ERR_NOALLOC_LIMIT") and "32" in msg


def test_noalloc_limit_is_inclusive(lib):
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    # 32 pairs pass validation and stop at the device query (no device here)
    assert call_noalloc(lib, batch=2, H=16) == KDA_ERR_CUDA
    assert call_noalloc(lib, cu=FAKE, num_seqs=4, H=8) == KDA_ERR_CUDA


# ---------------------------------------------------------------- GPU

def varlen_case(seed):
    """4 packed sequences (one empty, ragged tails) x 8 heads = 32 pairs, fp32 states."""
    lens = [300, 0, 1000, 65]
    inp = make_inputs({"B": 1, "T": sum(lens), "H": 8, "lengths": None, "g_mu": 3.0,
                       "init": None, "final": "fp32", "seed": seed}, device="cuda")
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    inp["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed * 16 + 5)
    inp["h0"] = 0.1 * torch.randn((len(lens), 8, 128, 128), generator=gen, device="cuda")
    return inp


def batch_case(seed):
    """2 rows of 777 tokens x 16 heads = 32 pairs, bf16 states."""
    return make_inputs({"B": 2, "T": 777, "H": 16, "lengths": None, "g_mu": 5.0,
                        "init": "bf16", "final": "bf16", "seed": seed}, device="cuda")


def run_fwd(inp):
    return kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["scale"],
                       cu_seqlens=inp["cu_seqlens"], initial_state=inp["h0"],
                       final_state_dtype=inp["h0"].dtype)


def buffers(inp):
    n = inp["h0"].shape[0]
    out = torch.empty_like(inp["v"])
    hT = torch.empty((n, inp["H"], 128, 128), dtype=inp["h0"].dtype, device="cuda")
    return out, hT


def run_noalloc(inp, out, hT):
    return kda.kda_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], out, inp["scale"],
                               cu_seqlens=inp["cu_seqlens"], initial_state=inp["h0"], final_state=hT)


@pytest.mark.gpu
@pytest.mark.parametrize("case", [varlen_case, batch_case], ids=["varlen_fp32_state", "batch_bf16_state"])
def test_noalloc_matches_kda_fwd_on_two_calls_in_a_row(lib, case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inputs = [case(40), case(41)]
    refs = [run_fwd(inp) for inp in inputs]
    bufs = [buffers(inp) for inp in inputs]
    torch.cuda.synchronize()
    allocated = torch.cuda.memory_allocated()
    # two calls in a row on one stream, no host synchronisation between them
    for inp, (out, hT) in zip(inputs, bufs):
        run_noalloc(inp, out, hT)
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    assert torch.cuda.memory_allocated() == allocated
    # both entry points run the same deterministic kernel: the results must be identical,
    # which a ring-indexing mistake perturbing a few chunks would break
    for (ref_out, ref_hT), (out, hT) in zip(refs, bufs):
        r_out = rel(out.float().cpu().numpy(), ref_out.float().cpu().numpy())
        r_state = rel(hT.float().cpu().numpy(), ref_hT.float().cpu().numpy())
        assert r_out <= OUT_TOL, f"out rel err {r_out:.3e}"
        assert r_state <= STATE_TOL[hT.dtype], f"state rel err {r_state:.3e}"
        assert torch.equal(out, ref_out) and torch.equal(hT, ref_hT)
    # once the entry point has run on the device, further calls leave the device's
    # free memory unchanged
    free0 = torch.cuda.mem_get_info()[0]
    for inp, (out, hT) in zip(inputs, bufs):
        run_noalloc(inp, out, hT)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert kda.device_error() == 0


@pytest.mark.gpu
def test_noalloc_refuses_a_call_beyond_its_scratch_on_the_device(lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = make_inputs({"B": 1, "T": 64, "H": 33, "lengths": None, "g_mu": 3.0,
                       "init": None, "final": None, "seed": 42}, device="cuda")
    out = torch.full_like(inp["v"], 7.0)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], out, inp["scale"])
    assert e.value.status == KDA_ERR_NOALLOC_LIMIT
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was enqueued
