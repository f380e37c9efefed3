"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module draws random numbers and lays out shapes; it holds none of the
Muon arithmetic (no momentum, no Newton-Schulz, no update, no projection).
Host draws use NumPy PCG64; large device-resident sets are drawn with a torch
CUDA generator (Philox) so that 6.5e9-element sets do not pass through the
host.  Shapes follow PyTorch's Linear layout: (rows, cols) = (d_out, d_in).
"""
from __future__ import annotations

import numpy as np

SEED_BASE = 1000

# Shapes of the parameter sets (rows x cols), in layer order.
GPT2_SMALL_LAYER = [(768, 2304), (768, 768), (768, 3072), (3072, 768)]
LLAMA7B_LAYER = [(4096, 4096)] * 4 + [(4096, 11008)] * 2 + [(11008, 4096)]


def gpt2_small_shapes(layers: int = 12):
    """12 layers x {768x2304 qkv, 768x768 attn-out, 768x3072 fc, 3072x768 proj}."""
    return GPT2_SMALL_LAYER * layers


def llama7b_shapes(layers: int = 32):
    """32 layers x {4 x 4096x4096 attention, 2 x 4096x11008 up/gate, 11008x4096 down}."""
    return LLAMA7B_LAYER * layers


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def single_fp32(seed: int = SEED_BASE + 1, rows: int = 256, cols: int = 128, std: float = 0.02):
    """One fp32 matrix: W, G ~ N(0, std^2), momentum zero."""
    r = rng(seed)
    W = (r.standard_normal((rows, cols)) * std).astype(np.float32)
    G = (r.standard_normal((rows, cols)) * std).astype(np.float32)
    M = np.zeros((rows, cols), dtype=np.float32)
    return W, G, M


def low_rank_plus_noise(seed: int = SEED_BASE + 2, batch: int = 64, n: int = 1024, rank: int = 32,
                        scale: float = 1e-2, noise_std: float = 1e-2):
    """Batch of n x n float32 gradients 1e-2 * P Q + N(0, 1e-4) noise with
    P (n x rank), Q (rank x n) of N(0, 1) entries -- extreme condition number.
    (The noise variance 1e-4 is standard deviation 1e-2.)  Returned in fp32;
    the caller rounds to bf16 storage."""
    r = rng(seed)
    out = np.empty((batch, n, n), dtype=np.float32)
    for i in range(batch):
        P = r.standard_normal((n, rank))
        Q = r.standard_normal((rank, n))
        E = r.standard_normal((n, n)) * noise_std
        out[i] = (scale * (P @ Q) + E).astype(np.float32)
    return out


def parameter_set_host(shapes, seed: int, w_std: float = 0.02, g_std: float = 1e-3):
    """Per-matrix (W, G) fp32 host arrays with W ~ N(0, w_std^2), G ~ N(0, g_std^2).
    The caller rounds to the storage dtype.  Momentum starts at zero."""
    r = rng(seed)
    out = []
    for (rows, cols) in shapes:
        W = (r.standard_normal((rows, cols)) * w_std).astype(np.float32)
        G = (r.standard_normal((rows, cols)) * g_std).astype(np.float32)
        out.append((W, G))
    return out


def stiefel_problem(seed: int = SEED_BASE + 4, batch: int = 16, n: int = 4096, k: int = 1024):
    """Column-orthonormal W (Q factor of the QR of an N(0,1) matrix), float64 on
    the host; the caller stores it as fp32."""
    r = rng(seed)
    Ws = np.empty((batch, n, k), dtype=np.float64)
    for i in range(batch):
        q, _ = np.linalg.qr(r.standard_normal((n, k)))
        Ws[i] = q
    return Ws


def stiefel_gradient(seed: int, step: int, batch: int, n: int, k: int):
    """A fresh N(0, 1) gradient batch for one step (seed = base + step)."""
    r = rng(seed + 7919 * (step + 1))
    return r.standard_normal((batch, n, k)).astype(np.float32)


def device_normal_(tensor, std: float, generator):
    """Fill a CUDA tensor in place with N(0, std^2) from a seeded torch generator."""
    tensor.normal_(mean=0.0, std=std, generator=generator)
    return tensor
