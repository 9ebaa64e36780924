"""bitnet_linear_noalloc: the linear layer for callers that cannot allocate
device memory (under stream capture, inside a framework that owns every byte
of device memory through its own pool, or on paths that cannot pay for an
allocation's synchronisation). It keeps the quantised activations in a
scratch array built into the library instead of a caller workspace, so its
results must be those of bitnet_linear with a workspace.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import bit_gemm_bitnet_b200 as bn
from helpers import bf16_bits, bf16_ulp_diff, to_dev

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def call_noalloc(x, wp, sw, out, M, N, K):
    """The new entry point, called through the C ABI."""
    P = ctypes.c_void_p
    st = P(torch.cuda.current_stream().cuda_stream)
    return bn.lib().bitnet_linear_noalloc(P(out.data_ptr()), P(x.data_ptr()), bn.BF16,
                                          P(wp.data_ptr()), P(sw.data_ptr()), sw.numel(),
                                          M, N, K, st)


def inputs(seed, M, K, N):
    x = synth.act_bf16(synth.key(77, seed, synth.T_ACT), M, K)
    w = synth.ternary(synth.key(77, seed, synth.T_WEIGHT), N, K)
    sw = synth.uniform_f32(synth.key(77, seed, synth.T_SCALE_WT), N, 0.01, 0.1)
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
        d = bf16_ulp_diff(bf16_bits(out), bf16_bits(ref))
        assert d.max() <= 1, f"call {seed}: max ulp {d.max()}"
    bn.bitnet_device_status()


def test_noalloc_small_m_and_limit(cuda_ok):
    # M < 16 takes the fused GEMV (no scratch); a shape whose activations do
    # not fit the scratch is refused before anything is launched
    xd, wp, sw = inputs(5, 4, 1024, 256)
    ref = bn.bitnet_linear(xd, wp, sw)
    out = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(xd, wp, sw, out, 4, 256, 1024) == bn.OK
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(out), bf16_bits(ref))
    M, K = 4096, 8192
    assert bn.bitnet_linear_workspace_bytes(M, K) > SCRATCH_BYTES
    assert call_noalloc(xd, wp, sw, out, M, 256, K) == bn.ERR_WORKSPACE
    bn.bitnet_device_status()
