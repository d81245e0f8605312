"""Helpers for the GPU tests: move numpy arrays (bf16 as uint16 bits) to
CUDA tensors and back, and the tolerance checks the tests share."""
import numpy as np
import torch

import workloads as W


def dev(a):
    """numpy -> CUDA tensor with the same bytes (uint16 travels as int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host(t, dtype=None):
    a = t.cpu().numpy()
    if dtype is not None:
        a = a.view(dtype)
    return a


def empty_bf16(*shape):
    return torch.zeros(*shape, dtype=torch.int16, device="cuda")


def maxnorm_err(got_bits, ref_bits):
    """max |got - ref| / max |ref| over bf16 bit arrays."""
    g = W.bf16_bits_to_f32(got_bits).astype(np.float64)
    r = W.bf16_bits_to_f32(ref_bits).astype(np.float64)
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-30))
