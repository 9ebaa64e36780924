"""Shared helpers for the tests: tensor conversion and bf16 ulp distance."""
import numpy as np
import torch


def to_dev(a, dtype=None):
    """numpy -> CUDA tensor (bf16 given as uint16 bits when dtype=bfloat16)."""
    if dtype == torch.bfloat16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_bits(t):
    """CUDA/CPU bf16 tensor -> numpy uint16 bits."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_ulp_diff(a_bits, b_bits):
    """Distance in bf16 ulps between two arrays of bf16 bit patterns."""
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + (b & 0x7FFF))
    return np.abs(ordered(a_bits) - ordered(b_bits))


def f32_to_bf16_bits(f):
    u = np.asarray(f, np.float32).view(np.uint32).astype(np.uint64)
    lower = u & 0xFFFF
    upper = u >> 16
    up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    return (upper + up.astype(np.uint64)).astype(np.uint16)
