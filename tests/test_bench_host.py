"""bench.py's byte and FLOP accounting, against the figures derived by hand from the layouts
(no GPU): the roofline fractions the bench reports are only as good as these."""
import bench


def test_prefill_bytes_per_token_head():
    # q, k, v, out: 128 bf16 each; g: 128 fp32; beta: one fp32
    assert bench.BYTES_PER_TOKEN_HEAD == 4 * 256 + 512 + 4 == 1540


def test_prefill_flops_per_token_head_is_the_pages_count():
    d, c = 128, 64
    assert bench.FLOPS_PER_TOKEN_HEAD == 6 * d * d + 3 * c * d + c * c == 126976
    assert bench.pages_flops(1 << 20, 32) == float((1 << 20) * 32 * 126976)


def test_state_bytes():
    import torch
    # one fp32 state in and out per (sequence, head): 2 x 64 KiB
    assert bench.state_bytes(1, 32, torch.float32, torch.float32) == 32 * 2 * 65536
    assert bench.state_bytes(2, 4, None, torch.bfloat16) == 2 * 4 * 32768
    assert bench.state_bytes(3, 3, None, None) == 0


def test_decode_unit_bytes():
    # the state read and written, plus q, k, v, out (4 x 256 B), g (512 B) and beta (4 B)
    assert bench.decode_unit_bytes("fp32") == 2 * 65536 + 1540 == 132612
    assert bench.decode_unit_bytes("bf16") == 2 * 32768 + 1540 == 67076


def test_backward_flop_and_byte_counts():
    # C = 16, D = 128: eight C x D x D products, two D x D, seven triangular C (C + 1) / 2 x D,
    # four C x C x D and 2 C^3, per chunk of 16 tokens, two FLOPs per multiply-add
    C, D = 16, 128
    per_chunk = 8 * C * D * D + 2 * D * D + 7 * (C * (C + 1) // 2) * D + 4 * C * C * D + 2 * C ** 3
    assert per_chunk == 2391040
    assert bench.bwd_flops_per_token_head() == 2 * per_chunk / C == 298880.0
    # q, k, v, dout in; g, beta in; dq, dk, dv, dg, dbeta out; a 64 KiB checkpoint per 64 tokens, twice
    assert bench.BWD_BYTES_PER_TOKEN_HEAD == 4 * 256 + 512 + 4 + 4 * 512 + 4 + 2 * 1024 == 5640


def test_fp32_alu_peak():
    assert abs(bench.fp32_alu_peak_tflops(1965.0) - 74.45) < 0.01
