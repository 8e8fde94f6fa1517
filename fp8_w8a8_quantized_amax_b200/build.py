"""Build libfp8q.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp8q.so")
SOURCES = ["fp8q.cu"]
DEPS = ["fp8q.cu", "ptx.cuh", "quant.cuh", "gemm_prefill.cuh", "gemm_decode.cuh", "gemv_w8a16.cuh", "calib.cuh", "sched.cuh"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def flags(verbose: bool = False) -> list:
    f = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", "fp8q.h")]
    return any(os.path.getmtime(d) > t for d in deps)


# Test build for the failure-detection tests: waits give up after 2 ms instead
# of 4 s, and a test-only switch makes one decode CTA withhold a release.  It
# is a separate file; the product library never contains the switch.
TEST_LIB = os.path.join(HERE, "libfp8q_testhooks.so")
TEST_FLAGS = ["-DFP8Q_TEST_HOOKS", "-DFP8Q_WAIT_LIMIT_NS=2000000ull"]


def _compile(out: str, extra: list, force: bool, verbose: bool) -> str:
    if not force and not stale(out):
        return out
    cmd = [nvcc()] + flags(verbose) + extra + [os.path.join(CSRC, s) for s in SOURCES] + ["-o", out + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False, verbose: bool = False) -> str:
    return _compile(LIB, [], force, verbose)


def build_test_hooks(force: bool = False) -> str:
    """The test build (libfp8q_testhooks.so) -- for tests only."""
    return _compile(TEST_LIB, TEST_FLAGS, force, False)


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
