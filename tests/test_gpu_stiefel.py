"""GPU parity of stiefel_cayley_step (projection + Woodbury Cayley, fp32) against the oracle.

The fp32 path is compared with the fp64 oracle element by element (bound from fp32
rounding through a 2k x 2k solve: 2e-5 absolute on O(1/sqrt(n)) entries), and checked
against the method's invariant: ||W^T W - I||_max <= 1e-5, also after 100 steps on the
16 x 4096 x 1024 workload.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from matrix_orthogonalising_optimizer_02_b200 import binding as mb
from matrix_orthogonalising_optimizer_02_b200 import workloads
from gpu_helpers import host

pytestmark = pytest.mark.gpu


def orth_err_dev(W):
    k = W.shape[-1]
    Wd = W.double()
    E = Wd.transpose(-1, -2) @ Wd - torch.eye(k, dtype=torch.float64, device=W.device)
    return float(E.abs().max())


def stiefel_step(W, G, lr):
    b, n, k = W.shape
    ws = mb.workspace(mb.stiefel_workspace_size(b, n, k))
    mb.stiefel_cayley_step(W, G, lr, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    return ws


@pytest.mark.parametrize("n,k,lr", [(256, 64, 1e-2), (200, 72, 0.3), (130, 30, 1.0), (64, 16, 1e-2),
                                     (512, 128, 5e-2), (96, 96, 0.1),
                                     # 2k = 1280: the top block columns (over 1000 rows) factorise their
                                     # panels on 8-CTA clusters, the lower ones on one CTA per system
                                     (1536, 640, 1e-2),
                                     # odd k on the cluster path: no bf16 planes (n % 8 != 0), 3k odd, so
                                     # the fp64 updates with an odd N fall back to the FMA pipes
                                     (1100, 515, 1e-2)])
def test_stiefel_step_matches_oracle(n, k, lr):
    Ws = workloads.stiefel_problem(seed=900 + n, batch=2, n=n, k=k)
    Gs = workloads.stiefel_gradient(900 + n, 0, 2, n, k)
    W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    G = torch.tensor(Gs, dtype=torch.float32, device="cuda")
    W0 = host(W)
    stiefel_step(W, G, lr)
    got = host(W)
    for i in range(2):
        want = orc.stiefel_cayley_step(W0[i], Gs[i].astype(np.float64), lr)
        assert np.max(np.abs(got[i] - want)) <= 2e-5
        assert orc.orthogonality_error(got[i]) <= 1e-5


def test_stiefel_large_k_matches_oracle():
    """2k = 4096: panels of up to 4096 rows, 512 rows per CTA on the clusters, 22- and 32-column
    panels, and one-CTA panels below 1000 rows; one step against the oracle."""
    n, k, lr = 4096, 2048, 1e-2
    Ws = workloads.stiefel_problem(seed=990, batch=1, n=n, k=k)
    Gs = workloads.stiefel_gradient(990, 0, 1, n, k)
    W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    G = torch.tensor(Gs, dtype=torch.float32, device="cuda")
    W0 = host(W)
    stiefel_step(W, G, lr)
    got = host(W)
    want = orc.stiefel_cayley_step(W0[0], Gs[0].astype(np.float64), lr)
    assert np.max(np.abs(got[0] - want)) <= 2e-5
    assert orc.orthogonality_error(got[0]) <= 1e-5


def test_stiefel_more_systems_than_one_wave_of_clusters():
    """24 systems of 1200 x 520 (2k = 1040: the top block column's panels on 8-CTA clusters):
    192 cluster CTAs, more than the SMs hold at once, so clusters run in waves.  Two sampled
    systems against the oracle, the manifold invariant on all."""
    batch, n, k, lr = 24, 1200, 520, 1e-2
    Ws = workloads.stiefel_problem(seed=991, batch=batch, n=n, k=k)
    Gs = workloads.stiefel_gradient(991, 0, batch, n, k)
    W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    G = torch.tensor(Gs, dtype=torch.float32, device="cuda")
    W0 = host(W)
    stiefel_step(W, G, lr)
    got = host(W)
    for i in (0, 17):
        want = orc.stiefel_cayley_step(W0[i], Gs[i].astype(np.float64), lr)
        assert np.max(np.abs(got[i] - want)) <= 2e-5
    assert orth_err_dev(W) <= 1e-5


def test_stiefel_zero_lr_is_identity_map():
    Ws = workloads.stiefel_problem(seed=950, batch=1, n=128, k=32)
    W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    G = torch.randn(W.shape, device="cuda")
    W0 = W.clone()
    stiefel_step(W, G, 0.0)
    assert torch.allclose(W, W0, atol=1e-6)


def test_stiefel_workload_100_steps():
    batch, n, k, lr = 16, 4096, 1024, 1e-2
    Ws = workloads.stiefel_problem(batch=batch, n=n, k=k)
    W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1004)
    G = torch.empty_like(W)
    ws = mb.workspace(mb.stiefel_workspace_size(batch, n, k))
    # step 1 against the oracle on one matrix
    workloads.device_normal_(G, 1.0, gen)
    W0 = host(W[3])
    G0 = host(G[3])
    mb.stiefel_cayley_step(W, G, lr, ws)
    want = orc.stiefel_cayley_step(W0, G0, lr)
    assert np.max(np.abs(host(W[3]) - want)) <= 2e-5
    for _ in range(99):
        workloads.device_normal_(G, 1.0, gen)
        mb.stiefel_cayley_step(W, G, lr, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    assert orth_err_dev(W) <= 1e-5


@pytest.mark.parametrize("center", [True, False])
def test_muon_cayley_steps_match_oracle(center):
    """MuonCayley (EMA momentum, column centering, projection, Cayley) over 5 steps with
    the page's starting values lr = 3e-3, momentum 0.9."""
    batch, n, k, lr, beta = 2, 256, 64, 3e-3, 0.9
    Ws = workloads.stiefel_problem(seed=960, batch=batch, n=n, k=k)
    W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    M = torch.zeros_like(W)
    ws = mb.workspace(mb.muon_cayley_workspace_size(batch, n, k))
    Wr = [Ws[i].copy() for i in range(batch)]
    Mr = [np.zeros((n, k)) for _ in range(batch)]
    for step in range(5):
        Gs = workloads.stiefel_gradient(960, step, batch, n, k)
        G = torch.tensor(Gs, dtype=torch.float32, device="cuda")
        mb.muon_cayley_step(W, G, M, lr, beta, ws, center=center)
        for i in range(batch):
            Wr[i], Mr[i] = orc.muon_cayley_step(Wr[i], Gs[i].astype(np.float64), Mr[i], lr, float(np.float32(beta)),
                                                center=center)
    assert mb.device_status(ws) == mb.MUON_OK
    for i in range(batch):
        assert np.max(np.abs(host(W[i]) - Wr[i])) <= 2e-5
        assert np.max(np.abs(host(M[i]) - Mr[i])) <= 1e-5 * max(1.0, np.max(np.abs(Mr[i])))
        assert orc.orthogonality_error(host(W[i])) <= 1e-5


def test_muon_cayley_wide_batch_matches_transposed_oracle():
    """A wide batch (64 x 256: orthonormal rows) goes through the library's transpose
    branch; 3 steps against the oracle, which updates the transpose (page §4.4)."""
    batch, rows, cols, lr, beta = 2, 64, 256, 3e-3, 0.9
    Ws = np.ascontiguousarray(np.swapaxes(workloads.stiefel_problem(seed=970, batch=batch, n=cols, k=rows), 1, 2))
    W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    M = torch.zeros_like(W)
    ws = mb.workspace(mb.muon_cayley_workspace_size(batch, rows, cols))
    Wr = [Ws[i].copy() for i in range(batch)]
    Mr = [np.zeros((rows, cols)) for _ in range(batch)]
    for step in range(3):
        Gs = workloads.stiefel_gradient(970, step, batch, rows, cols)
        G = torch.tensor(Gs, dtype=torch.float32, device="cuda")
        mb.muon_cayley_step(W, G, M, lr, beta, ws, center=True)
        for i in range(batch):
            Wr[i], Mr[i] = orc.muon_cayley_step(Wr[i], Gs[i].astype(np.float64), Mr[i], lr, float(np.float32(beta)))
    assert mb.device_status(ws) == mb.MUON_OK
    for i in range(batch):
        got = host(W[i])
        assert np.max(np.abs(got - Wr[i])) <= 2e-5
        assert np.max(np.abs(host(M[i]) - Mr[i])) <= 1e-5 * max(1.0, np.max(np.abs(Mr[i])))
        assert np.max(np.abs(got @ got.T - np.eye(rows))) <= 1e-5


@pytest.mark.parametrize("n,k", [(256, 64), (300, 100), (1200, 520)])
def test_stiefel_nan_gradient_is_reported(n, k):
    """A NaN in G reaches every column of the 2k x 2k system, so the elimination meets columns
    with no finite entry: the step must still pick in-range pivots (row jj, as the textbook
    algorithm with a NaN-ignoring argmax would), report MUON_ERR_NONFINITE, and leave the
    device usable for the next call."""
    Ws = workloads.stiefel_problem(seed=970 + n, batch=2, n=n, k=k)
    W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    G = torch.randn(W.shape, device="cuda")
    G[1, 5, 7] = float("nan")
    ws = mb.workspace(mb.stiefel_workspace_size(2, n, k))
    mb.stiefel_cayley_step(W, G, 1e-2, ws)
    torch.cuda.synchronize()
    assert mb.device_status(ws) == mb.MUON_ERR_NONFINITE
    # the same workspace serves a clean step afterwards
    W2 = torch.tensor(Ws, dtype=torch.float32, device="cuda")
    G2 = torch.randn(W2.shape, device="cuda")
    mb.stiefel_cayley_step(W2, G2, 1e-2, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    assert orth_err_dev(W2) <= 1e-5
