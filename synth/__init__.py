"""Seeded synthetic inputs shaped like the workloads of the bitnet-tc pages.

Shared by the tests, the bench and the oracle side; holds none of the
method's arithmetic (see ``synth.c``). Every tensor is addressed by a key
derived from (workload, layer, tensor, variant), and every element by its
flat index, so a slice can be regenerated without the rest.

Distributions (the workload descriptions of the BitNet b1.58 W1.58A8 layer):
  * ternary weights, P(-1) = P(+1) = 0.3, P(0) = 0.4;
  * per-tensor fp32 weight scale, uniform in [0.01, 0.1);
  * bf16 activations N(0, 1), 0.1 % of entries multiplied by 20 (outliers),
    or no outliers where a workload says so.
"""
import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "synth.c")
OUT = os.path.join(HERE, "libsynth.so")

OUTLIER_P = 0.001
OUTLIER_MULT = 20.0

# tensor ids inside a key
T_WEIGHT, T_ACT, T_SCALE_WT = 1, 2, 3

_lib = None
_THREADS = max(1, min(32, os.cpu_count() or 1))


def build(force: bool = False) -> str:
    if (not force and os.path.exists(OUT)
            and os.path.getmtime(OUT) >= os.path.getmtime(SRC)):
        return OUT
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                           "-pthread", SRC, "-o", OUT, "-lm"])
    return OUT


def _L():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        u64, i64, P = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        L.synth_key.argtypes = [u64, u64, u64, u64]
        L.synth_key.restype = u64
        L.synth_ternary.argtypes = [u64, i64, i64, P, ctypes.c_int]
        L.synth_act_bf16.argtypes = [u64, i64, i64, ctypes.c_double,
                                     ctypes.c_double, P, ctypes.c_int]
        L.synth_uniform_f32.argtypes = [u64, i64, i64, ctypes.c_double,
                                        ctypes.c_double, P, ctypes.c_int]
        _lib = L
    return _lib


def key(workload: int, layer: int, tensor: int, variant: int = 0) -> int:
    return int(_L().synth_key(workload, layer, tensor, variant))


def ternary(k: int, N: int, K: int, row0: int = 0, out=None) -> np.ndarray:
    """int8 [N, K] ternary weights: rows row0 .. row0+N of the tensor."""
    if out is None:
        out = np.empty((N, K), np.int8)
    _L().synth_ternary(k, row0 * K, N * K, out.ctypes.data, _THREADS)
    return out


def act_bf16(k: int, M: int, K: int, row0: int = 0, outliers: bool = True,
             out=None) -> np.ndarray:
    """bf16 bits [M, K]: rows row0 .. row0+M of an N(0,1) activation tensor."""
    if out is None:
        out = np.empty((M, K), np.uint16)
    p = OUTLIER_P if outliers else 0.0
    _L().synth_act_bf16(k, row0 * K, M * K, p, OUTLIER_MULT, out.ctypes.data,
                        _THREADS)
    return out


def uniform_f32(k: int, n: int, lo: float, hi: float) -> np.ndarray:
    out = np.empty((n,), np.float32)
    _L().synth_uniform_f32(k, 0, n, lo, hi, out.ctypes.data, _THREADS)
    return out


def scale_wt(k: int) -> np.ndarray:
    """One fp32 per tensor, uniform in [0.01, 0.1)."""
    return uniform_f32(k, 1, 0.01, 0.1)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)
