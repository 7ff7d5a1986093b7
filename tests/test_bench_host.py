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
