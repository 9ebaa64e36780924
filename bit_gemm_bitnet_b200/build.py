"""Build libbitnet_b200.so in-tree with nvcc for sm_100a (B200).

IEEE division and square root are kept (no --use_fast_math): the quantiser's
x / scale must be the correctly rounded fp32 quotient.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
OUT = os.path.join(HERE, "libbitnet_b200.so")
SOURCES = [os.path.join(CSRC, "bitnet.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "bitnet.h")]
# The failure-path test library (tests only): the decode GEMV with a 1 ms
# wait limit and a stage its producer can be told to leave out.
WAIT_TEST_OUT = os.path.join(HERE, "libbitnet_b200_waittest.so")
WAIT_TEST_SOURCES = [os.path.join(CSRC, "wait_test.cu")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def flags():
    return ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
            "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
            "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _build_one(sources, out, force, verbose):
    deps = DEPS + sources
    if not force and os.path.exists(out):
        t = os.path.getmtime(out)
        if all(os.path.getmtime(d) <= t for d in deps):
            return out
    cmd = [NVCC] + flags() + (["-Xptxas", "-v"] if verbose else []) + sources + ["-o", out]
    subprocess.check_call(cmd)
    return out


def build(force: bool = False, verbose: bool = False) -> str:
    """Build the product library (and the failure-path test library);
    returns the product library's path."""
    _build_one(WAIT_TEST_SOURCES, WAIT_TEST_OUT, force, verbose)
    return _build_one(SOURCES, OUT, force, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
