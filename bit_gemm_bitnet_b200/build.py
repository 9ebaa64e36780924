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

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def flags():
    return ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
            "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
            "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(OUT):
        t = os.path.getmtime(OUT)
        if all(os.path.getmtime(d) <= t for d in DEPS):
            return OUT
    cmd = [NVCC] + flags() + (["-Xptxas", "-v"] if verbose else []) + SOURCES + ["-o", OUT]
    subprocess.check_call(cmd)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
