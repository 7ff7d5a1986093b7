"""The C-ABI library without a GPU: it loads, exports every entry point that
include/kda.h declares, and rejects malformed arguments before touching the
device."""
import ctypes
import os
import re
import subprocess

import pytest

import kimi_delta_attention_27_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(kda_[a-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from kimi_delta_attention_27_b200 import build
    build.build()
    return kda.load_library()


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(kda.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", kda.LIB_PATH], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (kda_\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_status_strings(lib):
    for st in range(0, 16):
        s = kda.status_string(st)
        assert s.startswith("KDA_"), s
    assert kda.status_string(1234) == "KDA_ERR_UNKNOWN"
    assert lib.kda_version() >> 16 == 1


# A fake, 16-byte-aligned, never-dereferenced address: every call below must be
# rejected by validation before any device access.
FAKE = ctypes.c_void_p(0x10000)


def call(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, scale=1.0, cu=None, num_seqs=0, batch=1,
             seq_len=64, H=2, dk=128, dv=128, h0=None, h0dt=0, hT=None, hTdt=0, out=FAKE,
             stream=None)
    a.update(kw)
    return lib.kda_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"], a["cu"],
                       a["num_seqs"], a["batch"], a["seq_len"], a["H"], a["dk"], a["dv"],
                       a["h0"], a["h0dt"], a["hT"], a["hTdt"], a["out"], a["stream"])


def test_rejects_head_dims(lib):
    assert call(lib, dk=64) == 2
    assert call(lib, dv=256) == 2


def test_rejects_negative_sizes(lib):
    assert call(lib, seq_len=-1) == 2
    assert call(lib, H=0) == 2
    assert call(lib, batch=-2) == 2


def test_rejects_varlen_with_batch(lib):
    assert call(lib, cu=FAKE, num_seqs=3, batch=2) == 3


def test_rejects_state_dtypes(lib):
    assert call(lib, h0=FAKE, h0dt=0) == 4
    assert call(lib, hT=FAKE, hTdt=7) == 4
    assert call(lib, h0=FAKE, h0dt=1, hT=FAKE, hTdt=2) == 4


def test_rejects_null_tensors(lib):
    assert call(lib, q=None) == 1
    assert call(lib, out=None) == 1


def test_rejects_misaligned(lib):
    assert call(lib, k=ctypes.c_void_p(0x10008)) == 7
    assert call(lib, beta=ctypes.c_void_p(0x10002)) == 7


def test_rejects_oversized(lib):
    assert call(lib, seq_len=1 << 40) == 8


def test_empty_batch_is_a_no_op(lib):
    # zero sequences: nothing to do, no device needed
    assert call(lib, batch=0, q=None, k=None, v=None, g=None, beta=None, out=None) == 0


def test_no_device_is_reported(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert call(lib) == 5  # KDA_ERR_CUDA: no device to query


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kda.kda_fwd(x, x, x, x.float(), torch.zeros(1, 64, 1))


def _fwd_args():
    import torch
    B, T, H = 1, 64, 2
    q = torch.zeros(B, T, H, 128, dtype=torch.bfloat16)
    return dict(q=q, k=q.clone(), v=q.clone(), g=torch.zeros(B, T, H, 128), beta=torch.zeros(B, T, H))


@pytest.mark.parametrize("name,bad", [
    ("out", lambda t: t.zeros(1, 63, 2, 128, dtype=t.bfloat16)),
    ("initial_state", lambda t: t.zeros(1, 2, 128, 127)),
    ("final_state", lambda t: t.zeros(2, 2, 128, 128)),
    ("v", lambda t: t.zeros(1, 65, 2, 128, dtype=t.bfloat16)),
    ("beta", lambda t: t.zeros(1, 64, 3)),
])
def test_binding_requires_exact_buffer_shapes(name, bad):
    """An undersized buffer would be written out of bounds through the C ABI, which
    sees only pointers: the binding refuses it before anything else."""
    import torch
    a = _fwd_args()
    kw = {}
    if name in a:
        a[name] = bad(torch)
    else:
        kw[name] = bad(torch)
    with pytest.raises(ValueError, match="shape"):
        kda.kda_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], **kw)


def test_binding_requires_exact_decode_shapes():
    import torch
    q = torch.zeros(4, 2, 128, dtype=torch.bfloat16)
    g, beta = torch.zeros(4, 2, 128), torch.zeros(4, 2)
    with pytest.raises(ValueError, match="shape"):
        kda.kda_decode(q, q, q, g, beta, state_in=torch.zeros(4, 2, 128, 64))
    with pytest.raises(ValueError, match="shape"):
        kda.kda_decode(q, q, q, g, beta, out=torch.zeros(3, 2, 128, dtype=torch.bfloat16))


def call_ex(lib, kind=0, flags=0, g=FAKE, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, beta=FAKE, out=FAKE)
    a.update(kw)
    return lib.kda_fwd_ex(a["q"], a["k"], a["v"], g, kind, a["beta"], 1.0, None, 0, 1, 64, 2, 128, 128,
                          None, 0, None, 0, a["out"], flags, None)


def test_fwd_ex_rejects_unknown_options(lib):
    KDA_ERR_BAD_OPTION = 14
    assert call_ex(lib, kind=3) == KDA_ERR_BAD_OPTION
    assert call_ex(lib, kind=-1) == KDA_ERR_BAD_OPTION
    assert call_ex(lib, flags=4) == KDA_ERR_BAD_OPTION
    assert kda.status_string(KDA_ERR_BAD_OPTION).startswith("KDA_ERR_BAD_OPTION")


def test_fwd_ex_gate_alignment(lib):
    # a per-channel gate is loaded by TMA (16 bytes); a per-token one needs only 4
    assert call_ex(lib, kind=1, g=ctypes.c_void_p(0x10004)) == 7
    assert call_ex(lib, kind=2, g=ctypes.c_void_p(0x10002)) == 7
    import torch
    if not torch.cuda.is_available():
        assert call_ex(lib, kind=2, g=ctypes.c_void_p(0x10004), flags=3) == 5   # passes; no device


def test_segmented_workspace_size(lib):
    f = lib.kda_fwd_segmented_workspace
    assert f(1, 1 << 20, 32, 1 << 15) == 3 * 32 * 32 * 128 * 128 * 4
    assert f(2, 1000, 3, 192) == 3 * 2 * 6 * 3 * 128 * 128 * 4
    assert f(1, 1000, 3, 100) == 0 and f(1, 1000, 3, 0) == 0 and f(1, 1000, 0, 64) == 0


def test_bwd_workspace_size(lib):
    f = lib.kda_bwd_workspace
    # one 128 x 128 fp32 state per 64 tokens per head, plus one per sequence and head, plus one
    assert f(4096, 1, 32) == (64 + 1 + 1) * 32 * 65536
    assert f(1000, 3, 2) == (15 + 3 + 1) * 2 * 65536
    assert f(-1, 1, 1) == 0 and f(10, 1, 0) == 0
