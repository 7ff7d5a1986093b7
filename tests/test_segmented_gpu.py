"""GPU parity of kda_fwd_segmented, the segment-parallel forward: rows split into pieces
whose affine maps (S -> M S + B) are scanned, then re-run from the scanned states.
Against the fp64 oracle (outputs and final states), and against kda_fwd on the same
inputs. The segments composing through their affine maps is itself pinned on the oracle
(test_segments_compose_through_their_affine_maps)."""
import numpy as np
import pytest
import torch

import kimi_delta_attention_27_b200 as kda
from kimi_delta_attention_27_b200.inputs import make_inputs
from kda_testutil import check, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kimi_delta_attention_27_b200 import build
    build.build()


def seg_run(inp, seg):
    out, hT = kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], seg, inp["scale"],
                                    initial_state=inp["h0"], final_state_dtype=inp["final_dtype"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    return out, hT


@pytest.mark.parametrize("H", [1, 4])
def test_long_rows_few_heads_against_the_oracle(H):
    # 256K tokens in pieces of 8K: 32 pieces per head
    inp = make_inputs("t1m_h32", device="cuda", T=1 << 18, H=H, init="fp32")
    out, hT = seg_run(inp, 8192)
    check(inp, out, hT, note=f"segmented T=2^18 H={H} pieces of 8192")


@pytest.mark.parametrize("init,final", [("fp32", "fp32"), ("bf16", "bf16"), (None, "fp32"), (None, None)])
def test_ragged_rows_and_state_dtypes(init, final):
    # 2 rows of 1000 tokens in pieces of 192 (the last piece 40 tokens, not a chunk multiple)
    inp = make_inputs({"B": 2, "T": 1000, "H": 3, "lengths": None, "g_mu": 3.0, "init": init,
                       "final": final, "seed": 21}, device="cuda")
    out, hT = seg_run(inp, 192)
    check(inp, out, hT)
    ref_out, ref_hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["scale"],
                                  initial_state=inp["h0"], final_state_dtype=inp["final_dtype"])
    assert rel(out.float().cpu(), ref_out.float().cpu()) < 1e-2
    if final is not None:
        assert rel(hT.float().cpu(), ref_hT.float().cpu()) < (2e-3 if final == "fp32" else 1e-2)


def test_strong_decay_pieces():
    # every chunk on the sub-block path, in the affine runs as in the plain ones
    inp = make_inputs({"B": 1, "T": 2048, "H": 2, "lengths": None, "g_mu": -4.0, "init": "fp32",
                       "final": "fp32", "seed": 22}, device="cuda")
    out, hT = seg_run(inp, 256)
    check(inp, out, hT)


def test_one_piece_is_kda_fwd():
    inp = make_inputs({"B": 2, "T": 300, "H": 2, "lengths": None, "g_mu": 3.0, "init": "fp32",
                       "final": "fp32", "seed": 23}, device="cuda")
    out, hT = seg_run(inp, 320)
    ref_out, ref_hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["scale"],
                                  initial_state=inp["h0"], final_state_dtype=torch.float32)
    assert torch.equal(out, ref_out) and torch.equal(hT, ref_hT)


def test_workspace_checks():
    inp = make_inputs({"B": 1, "T": 1024, "H": 2, "lengths": None, "g_mu": 3.0, "init": None,
                       "final": "fp32", "seed": 24}, device="cuda")
    need = kda.segmented_workspace_bytes(1, 1024, 2, 256)
    assert need == 3 * 4 * 2 * 128 * 128 * 4
    assert kda.segmented_workspace_bytes(1, 1024, 2, 100) == 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(kda.KdaError) as e:
        kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], 256, workspace=small)
    assert e.value.status == 15
    with pytest.raises(kda.KdaError) as e:
        kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], 100)
    assert e.value.status == 2
