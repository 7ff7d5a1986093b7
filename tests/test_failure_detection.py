"""Failure detection of the forward kernel, with no GPU fault.

Every wait inside the kernel is bounded: one that runs out raises the device
error word and the kernel winds down instead of hanging. Here a test-only build
of the library (``-DKDA_TEST_HOOKS``: 100 ms wait limit, and a hook that keeps
one chunk's operand set from ever being signalled) makes the chain CTA's wait
for that chunk run out. The checks: kda_device_error reports KDA_ERR_TIMEOUT,
the call after it on the same device is correct, and the product library
neither exports the hook nor was built with it.
"""
import ctypes
import re
import subprocess

import pytest
import torch

import kimi_delta_attention_27_b200 as kda
from kimi_delta_attention_27_b200 import build
from kimi_delta_attention_27_b200.inputs import make_inputs
from kda_testutil import check

KDA_OK, KDA_ERR_TIMEOUT = 0, 9


def test_product_library_has_no_test_hook():
    build.build()
    out = subprocess.run(["nm", "-D", "--defined-only", kda.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    assert "kda_test_set_skip_chunk" not in out
    assert re.search(r" T kda_fwd$", out, flags=re.M)


def test_test_hook_library_builds_and_exports_the_hook():
    path = build.build_test_hooks()
    out = subprocess.run(["nm", "-D", "--defined-only", path], check=True,
                         capture_output=True, text=True).stdout
    assert re.search(r" T kda_test_set_skip_chunk$", out, flags=re.M)


def call_fwd(lib, inp, out, hT):
    P = ctypes.c_void_p
    st = lib.kda_fwd(P(inp["q"].data_ptr()), P(inp["k"].data_ptr()), P(inp["v"].data_ptr()),
                     P(inp["g"].data_ptr()), P(inp["beta"].data_ptr()), ctypes.c_float(inp["scale"]),
                     None, 0, inp["B"], inp["T"], inp["H"], 128, 128, None, 0,
                     P(hT.data_ptr()), 2, P(out.data_ptr()),
                     P(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.gpu
def test_a_wait_that_runs_out_is_reported_and_the_device_keeps_working():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = kda.load_library(path=build.build_test_hooks())
    lib.kda_test_set_skip_chunk.restype = ctypes.c_int
    lib.kda_test_set_skip_chunk.argtypes = [ctypes.c_int]
    inp = make_inputs("t4k_h32", device="cuda", T=3 * 64, H=1, init=None)
    out = torch.zeros_like(inp["v"])
    hT = torch.zeros((1, 1, 128, 128), dtype=torch.float32, device="cuda")
    assert lib.kda_device_error() == KDA_OK

    # chunk 1 of 3 is never published: the chain CTA gives up on it
    assert lib.kda_test_set_skip_chunk(1) == 0
    assert call_fwd(lib, inp, out, hT) == KDA_OK   # enqueued; the failure is on the device
    assert lib.kda_device_error() == KDA_ERR_TIMEOUT
    assert lib.kda_device_error() == KDA_OK        # read and cleared

    # the same device, the same library, no hook: a correct result
    assert lib.kda_test_set_skip_chunk(-1) == 0
    assert call_fwd(lib, inp, out, hT) == KDA_OK
    assert lib.kda_device_error() == KDA_OK
    check(inp, out, hT)

    # and the product library on the same device
    out2, hT2 = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["scale"],
                            final_state_dtype=torch.float32)
    assert kda.device_error() == KDA_OK
    check(inp, out2, hT2)
