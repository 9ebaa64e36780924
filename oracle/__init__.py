"""Scalar CPU oracle for the BitNet b1.58 W1.58A8 linear layer.

TEST INFRASTRUCTURE ONLY: the checker the CUDA library is compared against.
Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
import this package; the product (``bit_gemm_bitnet_b200``) never does, and
this package never imports the product.

Each function wraps one plain definition from ``bitnet_oracle.cpp`` (see the
citations there: the bitnet-cpu page ``torch-ext/bitnet_cpu/__init__.py``).
Arrays are numpy; bf16 values travel as their raw ``uint16`` bits.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_pack.argtypes = [_P, _I64, _I64, _P]
        L.oracle_unpack.argtypes = [_P, _I64, _I64, _P]
        L.oracle_quantize.argtypes = [_P, _I64, _I64, _P, _P]
        L.oracle_quantize_f32.argtypes = [_P, _I64, _I64, _P, _P]
        L.oracle_rmsnorm.argtypes = [_P, _P, ctypes.c_float, _I64, _I64, _P]
        L.oracle_rmsnorm_quantize.argtypes = [_P, _P, ctypes.c_float, _I64, _I64, _P, _P]
        L.oracle_linear_rmsnorm.argtypes = [_P, _P, ctypes.c_float, _P, _P, _I64, _I64, _I64,
                                            _I64, _P]
        L.oracle_linear_bias.argtypes = [_P, _P, _P, _I64, _P, _I64, _I64, _I64, _P]
        L.oracle_ternarize_absmean.argtypes = [_P, _I64, _I64, ctypes.c_int, _P, _P]
        L.oracle_linear_f32.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P]
        L.oracle_acc.argtypes = [_P, _P, _I64, _I64, _I64, _P]
        L.oracle_acc_threads.argtypes = [_P, _P, _I64, _I64, _I64, _P, ctypes.c_int]
        L.oracle_epilogue.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P]
        L.oracle_gemm.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _P]
        L.oracle_linear.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P]
        L.oracle_linear_threads.argtypes = [_P, _P, _P, _I64, _I64, _I64,
                                            _I64, _P, ctypes.c_int]
        L.oracle_gemm_threads.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64,
                                          _I64, _P, ctypes.c_int]
        L.oracle_linear_threads_cols.argtypes = [_P, _P, _P, _I64, _I64, _I64,
                                                 _I64, _P, ctypes.c_int]
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        for name in ("oracle_pack", "oracle_unpack", "oracle_quantize", "oracle_quantize_f32",
                     "oracle_ternarize_absmean", "oracle_linear_bias", "oracle_rmsnorm",
                     "oracle_rmsnorm_quantize", "oracle_linear_rmsnorm",
                     "oracle_linear_f32",
                     "oracle_acc", "oracle_acc_threads", "oracle_epilogue", "oracle_gemm",
                     "oracle_linear", "oracle_linear_threads",
                     "oracle_gemm_threads", "oracle_linear_threads_cols"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


class OracleError(ValueError):
    pass


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(st, what):
    if st != 0:
        raise OracleError(f"{what}: oracle status {st}")


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def pack(w):
    """int8 [N, K] ternary -> uint8 [N, K/4]."""
    w = _c(w, np.int8)
    N, K = w.shape
    out = np.empty((N, K // 4), np.uint8)
    _check(lib().oracle_pack(_ptr(w), N, K, _ptr(out)), "pack")
    return out


def unpack(packed, K):
    """uint8 [N, K/4] -> int8 [N, K] (code - 2)."""
    packed = _c(packed, np.uint8)
    N = packed.shape[0]
    out = np.empty((N, K), np.int8)
    _check(lib().oracle_unpack(_ptr(packed), N, K, _ptr(out)), "unpack")
    return out


def quantize(x_bf16_bits):
    """bf16 bits [M, K] -> (int8 [M, K], bf16 bits [M])."""
    x = _c(x_bf16_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s = np.empty((M,), np.uint16)
    _check(lib().oracle_quantize(_ptr(x), M, K, _ptr(q), _ptr(s)), "quantize")
    return q, s


def quantize_f32(x):
    """float32 [M, K] -> (int8 [M, K], bf16 bits [M])."""
    x = _c(x, np.float32)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s = np.empty((M,), np.uint16)
    _check(lib().oracle_quantize_f32(_ptr(x), M, K, _ptr(q), _ptr(s)), "quantize_f32")
    return q, s


def linear_f32(x, packed, scale_wt):
    """float32 [M, K] -> bf16 bits [M, N]: quantize_f32, then gemm."""
    x = _c(x, np.float32)
    packed = _c(packed, np.uint8)
    sw = _c(scale_wt, np.float32)
    M, K = x.shape
    N = packed.shape[0]
    out = np.empty((M, N), np.uint16)
    _check(lib().oracle_linear_f32(_ptr(x), _ptr(packed), _ptr(sw), sw.size, M, N, K,
                                   _ptr(out)), "linear_f32")
    return out


def ternarize_absmean(w, per_row=True):
    """float32 [N, K] -> (int8 ternary [N, K], float32 scale [N] or [1])."""
    w = _c(w, np.float32)
    N, K = w.shape
    wt = np.empty((N, K), np.int8)
    sc = np.empty((N if per_row else 1,), np.float32)
    _check(lib().oracle_ternarize_absmean(_ptr(w), N, K, 1 if per_row else 0, _ptr(wt), _ptr(sc)),
           "ternarize_absmean")
    return wt, sc


def linear_bias(x_bf16_bits, packed, scale_wt, bias_bf16_bits):
    """bitnet_linear, then + bias (bf16 [N]) as the page's BitLinear.forward."""
    x = _c(x_bf16_bits, np.uint16)
    packed = _c(packed, np.uint8)
    sw = _c(scale_wt, np.float32)
    b = _c(bias_bf16_bits, np.uint16)
    M, K = x.shape
    N = packed.shape[0]
    out = np.empty((M, N), np.uint16)
    _check(lib().oracle_linear_bias(_ptr(x), _ptr(packed), _ptr(sw), sw.size, _ptr(b), M, N, K,
                                    _ptr(out)), "linear_bias")
    return out


def rmsnorm(x_bf16_bits, g_bf16_bits, eps):
    """bf16 bits [M, K], norm weight bf16 bits [K] -> z bf16 bits [M, K]."""
    x = _c(x_bf16_bits, np.uint16)
    g = _c(g_bf16_bits, np.uint16)
    M, K = x.shape
    z = np.empty((M, K), np.uint16)
    _check(lib().oracle_rmsnorm(_ptr(x), _ptr(g), float(eps), M, K, _ptr(z)), "rmsnorm")
    return z


def rmsnorm_quantize(x_bf16_bits, g_bf16_bits, eps):
    x = _c(x_bf16_bits, np.uint16)
    g = _c(g_bf16_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s = np.empty((M,), np.uint16)
    _check(lib().oracle_rmsnorm_quantize(_ptr(x), _ptr(g), float(eps), M, K, _ptr(q), _ptr(s)),
           "rmsnorm_quantize")
    return q, s


def linear_rmsnorm(x_bf16_bits, g_bf16_bits, eps, packed, scale_wt):
    x = _c(x_bf16_bits, np.uint16)
    g = _c(g_bf16_bits, np.uint16)
    packed = _c(packed, np.uint8)
    sw = _c(scale_wt, np.float32)
    M, K = x.shape
    N = packed.shape[0]
    out = np.empty((M, N), np.uint16)
    _check(lib().oracle_linear_rmsnorm(_ptr(x), _ptr(g), float(eps), _ptr(packed), _ptr(sw),
                                       sw.size, M, N, K, _ptr(out)), "linear_rmsnorm")
    return out


def acc(q, packed, N=None):
    """int8 [M, K] x packed [N, K/4] -> int32 [M, N]."""
    q = _c(q, np.int8)
    packed = _c(packed, np.uint8)
    M, K = q.shape
    N = packed.shape[0] if N is None else N
    out = np.empty((M, N), np.int32)
    _check(lib().oracle_acc(_ptr(q), _ptr(packed), M, N, K, _ptr(out)), "acc")
    return out


def acc_threads(q, packed, threads):
    """acc() with the weight rows split over host threads (same result)."""
    q = _c(q, np.int8)
    packed = _c(packed, np.uint8)
    M, K = q.shape
    N = packed.shape[0]
    out = np.empty((M, N), np.int32)
    _check(lib().oracle_acc_threads(_ptr(q), _ptr(packed), M, N, K, _ptr(out), int(threads)),
           "acc_threads")
    return out


def epilogue(acc_i32, scale_act_bits, scale_wt):
    a = _c(acc_i32, np.int32)
    sa = _c(scale_act_bits, np.uint16)
    sw = _c(scale_wt, np.float32).reshape(-1)
    M, N = a.shape
    out = np.empty((M, N), np.uint16)
    _check(lib().oracle_epilogue(_ptr(a), _ptr(sa), _ptr(sw), sw.size, M, N,
                                 _ptr(out)), "epilogue")
    return out


def gemm(q, packed, scale_act_bits, scale_wt):
    """bitnet_gemm: -> bf16 bits [M, N]."""
    q = _c(q, np.int8)
    packed = _c(packed, np.uint8)
    sa = _c(scale_act_bits, np.uint16)
    sw = _c(scale_wt, np.float32).reshape(-1)
    M, K = q.shape
    N = packed.shape[0]
    out = np.empty((M, N), np.uint16)
    _check(lib().oracle_gemm(_ptr(q), _ptr(packed), _ptr(sa), _ptr(sw),
                             sw.size, M, N, K, _ptr(out)), "gemm")
    return out


def linear(x_bf16_bits, packed, scale_wt, threads=1):
    """bitnet_linear / bitnet_gemv_fused: bf16 bits [M, K] -> bf16 bits [M, N]."""
    x = _c(x_bf16_bits, np.uint16)
    packed = _c(packed, np.uint8)
    sw = _c(scale_wt, np.float32).reshape(-1)
    M, K = x.shape
    N = packed.shape[0]
    out = np.empty((M, N), np.uint16)
    if threads <= 1:
        st = lib().oracle_linear(_ptr(x), _ptr(packed), _ptr(sw), sw.size, M,
                                 N, K, _ptr(out))
    else:
        st = lib().oracle_linear_threads(_ptr(x), _ptr(packed), _ptr(sw),
                                         sw.size, M, N, K, _ptr(out), threads)
    _check(st, "linear")
    return out


def linear_cols_threads(x_bf16_bits, packed, scale_wt, threads):
    """linear with the output columns split across host threads."""
    x = _c(x_bf16_bits, np.uint16)
    packed = _c(packed, np.uint8)
    sw = _c(scale_wt, np.float32).reshape(-1)
    M, K = x.shape
    N = packed.shape[0]
    out = np.empty((M, N), np.uint16)
    _check(lib().oracle_linear_threads_cols(_ptr(x), _ptr(packed), _ptr(sw), sw.size,
                                            M, N, K, _ptr(out), threads),
           "linear_cols_threads")
    return out


def gemm_threads(q, packed, scale_act_bits, scale_wt, threads):
    q = _c(q, np.int8)
    packed = _c(packed, np.uint8)
    sa = _c(scale_act_bits, np.uint16)
    sw = _c(scale_wt, np.float32).reshape(-1)
    M, K = q.shape
    N = packed.shape[0]
    out = np.empty((M, N), np.uint16)
    _check(lib().oracle_gemm_threads(_ptr(q), _ptr(packed), _ptr(sa), _ptr(sw),
                                     sw.size, M, N, K, _ptr(out), threads),
           "gemm_threads")
    return out


def f32_to_bf16(f):
    return int(lib().oracle_f32_to_bf16(ctypes.c_float(f)))
