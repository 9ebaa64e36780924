"""bitnet_linear_noalloc: the linear layer for callers that cannot allocate
device memory themselves, such as code inside a framework that owns every
byte of device memory through its own pool, or a path that must not pay for
an allocation's implicit synchronisation. It keeps the quantised activations
in a scratch array built into the library instead of a caller workspace, and
runs the same kernels as bitnet_linear, so its results must be bitnet_linear's
bit for bit. (Its size refusal needs no GPU and is tested in
tests/test_abi_host.py.)

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import bit_gemm_bitnet_b200 as bn
from helpers import bf16_bits, to_dev

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def call_noalloc(x, wp, sw, out, M, N, K):
    """The allocation-free entry point, called through the C ABI."""
    P = ctypes.c_void_p
    st = P(torch.cuda.current_stream().cuda_stream)
    dt = bn.F32 if x.dtype == torch.float32 else bn.BF16
    return bn.lib().bitnet_linear_noalloc(P(out.data_ptr()), P(x.data_ptr()), dt,
                                          P(wp.data_ptr()), P(sw.data_ptr()), sw.numel(),
                                          M, N, K, st)


def host_inputs(seed, M, K, N):
    x = synth.act_bf16(synth.key(77, seed, synth.T_ACT), M, K)
    w = synth.ternary(synth.key(77, seed, synth.T_WEIGHT), N, K)
    sw = synth.uniform_f32(synth.key(77, seed, synth.T_SCALE_WT), N, 0.01, 0.1)
    return x, w, sw


def inputs(seed, M, K, N):
    x, w, sw = host_inputs(seed, M, K, N)
    xd = to_dev(x, torch.bfloat16)
    wp = bn.bitnet_pack_weights(to_dev(w))
    return xd, wp, to_dev(sw)


def test_noalloc_matches_linear_with_workspace_on_two_calls(cuda_ok):
    # two calls in a row on different data: the second must not see anything
    # the first left in the shared scratch
    for seed, (M, K, N) in enumerate([(300, 4096, 1024), (257, 2560, 640)]):
        assert bn.bitnet_linear_workspace_bytes(M, K) <= SCRATCH_BYTES
        xd, wp, sw = inputs(seed, M, K, N)
        ref = bn.bitnet_linear(xd, wp, sw)
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(xd, wp, sw, out, M, N, K) == bn.OK
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(out), bf16_bits(ref)), f"call {seed}"
    bn.bitnet_device_status()


def test_noalloc_matches_oracle(cuda_ok):
    # the allocation-free call against the scalar CPU oracle directly
    M, K, N = 40, 1024, 384
    x, w, sw = host_inputs(20, M, K, N)
    xd, wp, swd = inputs(20, M, K, N)
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(xd, wp, swd, out, M, N, K) == bn.OK
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(out), oracle.linear(x, oracle.pack(w), sw))
    bn.bitnet_device_status()


def test_noalloc_float32_and_small_m(cuda_ok):
    # float32 rows through the scratch (M >= 16), and M < 16, which takes the
    # fused GEMV and needs no scratch: both equal bitnet_linear bit for bit
    for seed, (M, K, N) in enumerate([(64, 2560, 520), (4, 1024, 256)]):
        xd, wp, sw = inputs(10 + seed, M, K, N)
        if M >= 16:
            xd = torch.randn((M, K), generator=torch.Generator().manual_seed(seed),
                             dtype=torch.float32).cuda()
        ref = bn.bitnet_linear(xd, wp, sw)
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(xd, wp, sw, out, M, N, K) == bn.OK
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(out), bf16_bits(ref)), f"M={M}"
    bn.bitnet_device_status()
