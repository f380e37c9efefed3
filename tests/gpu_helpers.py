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


def sv_gram(x):
    """Singular values of a large r x s matrix (r <= s or transposed) as the square roots of
    the eigenvalues of its r x r Gram matrix, in fp64: a 4096 x 11008 matrix takes seconds
    instead of the minutes of a full SVD.  An eigenvalue carries an absolute error of about
    eps * sigma_max^2, so a singular value sigma >= 1e-3 of a matrix with sigma_max <= 1.5 is
    off by less than 1e-12 -- far below the 0.05 bound it is checked against.  Returned in
    descending order, like np.linalg.svd."""
    a = np.asarray(x, np.float64)
    if a.shape[0] > a.shape[1]:
        a = a.T
    ev = np.linalg.eigvalsh(a @ a.T)
    return np.sqrt(np.clip(ev, 0.0, None))[::-1]


def assert_update_within_bound(W1, W0, O, lr, wd, s, bf16):
    """The updated weight against W1 = (1 - lr wd) W0 - lr s O evaluated exactly with the
    GPU's own O.  The kernel evaluates decay*W0 + step*O in fp32 (two roundings, each at most
    2^-23 of its term) and then stores the weight: every element lies within one storage ulp
    of the exact value plus that fp32 error, and more than 99% of the bf16 weights equal the
    exactly rounded value."""
    import oracle as orc
    W1_ref = orc.muon_update(W0, O, lr, wd, s)
    f32_err = 2.0 ** -23 * (np.abs((1 - lr * wd) * W0) + np.abs(lr * s * O))
    if bf16:
        R = orc.round_to_bf16(W1_ref)
        ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(R), 1e-38))) - 7), 2.0 ** -133)
        assert np.all(np.abs(W1 - R) <= ulp + f32_err)
        assert np.mean(bf16_ulp_diff(W1, R) == 0) > 0.99
    else:
        assert np.all(np.abs(W1 - W1_ref) <= 2.0 ** -23 * np.abs(W1_ref) + f32_err)


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
