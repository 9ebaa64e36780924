"""The failure path of a bounded wait, on the GPU, without a fault.

libbitnet_b200_waittest.so holds the decode GEMV kernel built with a 1 ms
wait limit and one switch: a ring stage of CTA 0 that its producer leaves
unrequested. The consumers waiting for that stage give up, set the device
error word and return; the producer drains the copies it did issue; the
kernel holds no tensor memory. The test checks that the status reads
BITNET_ERR_TIMEOUT, that the call returned promptly, and that the context is
still usable: the same call without the skip, and then a product-library
call, both match the oracle.
"""
import ctypes
import os
import time

import numpy as np
import pytest
import torch

import oracle
import synth
import bit_gemm_bitnet_b200 as bn
from helpers import bf16_bits, to_dev

pytestmark = pytest.mark.gpu

LIB = os.path.join(os.path.dirname(bn.LIB_PATH), "libbitnet_b200_waittest.so")


def wait_lib():
    L = ctypes.CDLL(LIB)
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    L.bitnet_wait_test_gemv.argtypes = [P, P, P, P, I64, I64, ctypes.c_int, P]
    L.bitnet_wait_test_gemv.restype = ctypes.c_int
    L.bitnet_wait_test_status.argtypes = [P]
    L.bitnet_wait_test_status.restype = ctypes.c_int
    return L


def test_bounded_wait_gives_up_and_context_survives(cuda_ok):
    L = wait_lib()
    K, N = 1024, 8192          # 512 row blocks of 16: CTA 0 owns at least three
    x = synth.act_bf16(synth.key(108, 0, synth.T_ACT), 1, K)
    w = synth.ternary(synth.key(108, 0, synth.T_WEIGHT), N, K)
    sw = np.array([0.05], np.float32)
    ref = oracle.linear(x, oracle.pack(w), sw)
    xd, swd = to_dev(x, torch.bfloat16), to_dev(sw)
    pd = bn.bitnet_pack_weights(to_dev(w))
    out = torch.zeros((1, N), dtype=torch.bfloat16, device="cuda")
    P = ctypes.c_void_p
    st = P(torch.cuda.current_stream().cuda_stream)

    def call(skip):
        return L.bitnet_wait_test_gemv(P(out.data_ptr()), P(xd.data_ptr()), P(pd.data_ptr()),
                                       P(swd.data_ptr()), N, K, skip, st)

    # without the skip: a normal call of the same build
    assert call(-1) == bn.OK
    assert L.bitnet_wait_test_status(st) == bn.OK
    assert np.array_equal(bf16_bits(out), ref)

    # the third stage of CTA 0 is never requested: its wait runs out (1 ms)
    t0 = time.monotonic()
    assert call(2) == bn.OK
    assert L.bitnet_wait_test_status(st) == bn.ERR_TIMEOUT
    assert time.monotonic() - t0 < 2.0
    # the word was cleared when it was read
    assert L.bitnet_wait_test_status(st) == bn.OK

    # the context is still usable: the same call again, then the product
    out.zero_()
    assert call(-1) == bn.OK
    assert L.bitnet_wait_test_status(st) == bn.OK
    assert np.array_equal(bf16_bits(out), ref)
    y = bn.bitnet_gemv_fused(xd, pd, swd)
    bn.bitnet_device_status()
    assert np.array_equal(bf16_bits(y), ref)
