"""Helpers shared by the GPU parity tests (device transfer, error norms)."""
import numpy as np
import torch


def dev(a, dtype):
    """Host array -> CUDA tensor of `dtype` (bf16 by round-to-nearest-even from fp32)."""
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(dtype).cuda().contiguous()


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_f(got, want):
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def sv(x):
    return np.linalg.svd(np.asarray(x, np.float64), compute_uv=False)


def f32_ulp_diff(a, b):
    """Distance in fp32 units in the last place between two fp32-valued arrays."""
    ia = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    ib = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    ia = np.where(ia < 0, -(ia & 0x7FFFFFFF), ia)
    ib = np.where(ib < 0, -(ib & 0x7FFFFFFF), ib)
    return np.abs(ia - ib)


def bf16_ulp_diff(a, b):
    """Distance in bf16 ulps between two bf16-valued arrays."""
    ia = (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.int64)
    ib = (np.asarray(b, np.float32).view(np.uint32) >> 16).astype(np.int64)
    sa = np.where(ia & 0x8000, -(ia & 0x7FFF), ia)
    sb = np.where(ib & 0x8000, -(ib & 0x7FFF), ib)
    return np.abs(sa - sb)
