"""Builds ``libbitlinear.so`` (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libbitlinear.so")
SOURCES = [os.path.join(HERE, "csrc", "bitlinear_api.cu")]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _deps():
    return glob.glob(os.path.join(HERE, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


# The test build: the same sources with the hooks of include/bitlinear_test_hooks.h
# (settable wait limit and injected copy count), used only by the tests of the
# device status word.  The product library never contains them.
TEST_LIB = os.path.join(HERE, "libbitlinear_testhooks.so")


def _compile(out: str, extra, force: bool, verbose: bool) -> str:
    newest = max(os.path.getmtime(p) for p in _deps())
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, *SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile when the library is missing or older than any source; returns its path."""
    return _compile(LIB, [], force, verbose)


def build_test_hooks(force: bool = False) -> str:
    """Compile the test-hook build of the library (see TEST_LIB); returns its path."""
    return _compile(TEST_LIB, ["-DBITLINEAR_TEST_HOOKS"], force, False)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--test-hooks" in sys.argv:
        print(build_test_hooks(force="--force" in sys.argv))
