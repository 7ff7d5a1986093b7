"""Build the CUDA library ``libkda.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m kimi_delta_attention_27_b200.build`` (or ``build()``).
The CUDA runtime is linked statically, so the library loads on a machine
without a GPU (its symbols can be inspected there; nothing runs without one).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkda.so")
# test-only variant: short wait limits and a hook that withholds one chunk (failure-detection tests)
TEST_HOOKS_LIB = os.path.join(HERE, "libkda_testhooks.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC,-O3", "-shared",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
    deps += glob.glob(os.path.join(ROOT, "include", "*.h")) + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          out: str = LIB) -> str:
    if not force and not _stale(out):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = out + ".tmp"
    cmd = [nvcc, *NVCC_FLAGS, *(extra or []), "-I", os.path.join(ROOT, "include"),
           *sources(), "-o", tmp, "-ldl"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build_test_hooks(force: bool = False, verbose: bool = False) -> str:
    """The test-only library (``-DKDA_TEST_HOOKS``): bounded waits give up after 100 ms and
    ``kda_test_set_skip_chunk`` makes a chunk's operand set never arrive. Never the product."""
    return build(force=force, verbose=verbose, extra=["-DKDA_TEST_HOOKS"], out=TEST_HOOKS_LIB)


if __name__ == "__main__":
    v = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else None
    print(build(force=True, verbose=v, extra=extra))
