"""Full-size parity: the parameter sets at their real sizes, in the launch configuration
the benchmark times (one muon_step_batched / ns_orthogonalize call over the whole set),
with sampled matrices checked against the fp64 oracle one by one and cheap invariants
checked on every matrix.

Sets: the Llama-7B-shaped set (224 matrices, 6.48e9 parameters, ~93 GB on the device),
the GPT-2-small set (48 matrices), and 64 low-rank 1024 x 1024 gradients under the fixed
and the hybrid schedule.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from matrix_orthogonalising_optimizer_02_b200 import binding as mb
from matrix_orthogonalising_optimizer_02_b200 import workloads
from gpu_helpers import assert_update_within_bound, dev, host, rel_f, sv, sv_gram

pytestmark = pytest.mark.gpu

LR, BETA, WD = 0.02, 0.95, 0.1


def _device_set(shapes, seed, sample):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    mats = []
    for i, (rows, cols) in enumerate(shapes):
        W = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda").normal_(0.0, 0.02, generator=gen)
        G = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda").normal_(0.0, 1e-3, generator=gen)
        M = torch.zeros((rows, cols), dtype=torch.float32, device="cuda")
        O = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda") if i in sample else None
        mats.append(mb.Matrix(W, G, M, O))
    return mats


def _check_set(shapes, seed, sample):
    mats = _device_set(shapes, seed, sample)
    before = {i: (host(mats[i].W), host(mats[i].G)) for i in sample}
    hp = mb.hyper(lr=LR, beta=BETA, weight_decay=WD)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    mb.muon_step_batched(mats, hp, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    for i in sample:
        W0, G = before[i]
        m = mats[i]
        M1 = host(m.M)
        assert np.array_equal(M1, G)                       # zero momentum: M1 = G exactly
        O = host(m.O_out)
        O_ref = orc.newton_schulz(orc.ns_input(M1), orc.fixed_schedule(5))
        assert rel_f(O, O_ref) <= 2e-2
        # the bf16 bound on every sampled shape, the 4096 x 11008 and 11008 x 4096 included
        assert np.max(np.abs(sv_gram(O) - sv_gram(O_ref))) <= 0.05
        s = orc.scale_factor(*W0.shape, "moonlight")
        assert_update_within_bound(host(m.W), W0, O, LR, WD, s, bf16=True)
    # every matrix of the set: finite weights and momentum after the step
    for m in mats:
        assert torch.isfinite(m.W.float()).all() and torch.isfinite(m.M).all()
    return mats


def test_llama7b_set_one_step():
    shapes = workloads.llama7b_shapes(32)
    # layer 0 q-projection (4096^2), layer 17 up (4096 x 11008, wide), layer 31 down (tall)
    sample = [0, 17 * 7 + 4, 31 * 7 + 6]
    _check_set(shapes, 1005, sample)


def test_gpt2_small_set_one_step():
    shapes = workloads.gpt2_small_shapes(12)
    sample = [0, 1, 2, 3, 45, 46, 47]
    _check_set(shapes, 1003, sample)


@pytest.mark.parametrize("sched,nsplit", [("kj5", 2), ("hybrid", 4)])
def test_low_rank_batch_full(sched, nsplit):
    G = workloads.low_rank_plus_noise(batch=64, n=1024)
    X = dev(G, torch.bfloat16)
    S = mb.Schedule.fixed(5, n_split_iters=nsplit) if sched == "kj5" else mb.Schedule.hybrid(n_split_iters=nsplit)
    ref = orc.fixed_schedule(5) if sched == "kj5" else orc.hybrid_schedule()
    Y = torch.empty_like(X)
    ws = mb.workspace(mb.ns_workspace_size(64, 1024, 1024, S))
    mb.ns_orthogonalize(X, Y, S, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    for i in [0, 21, 42, 63]:
        want = orc.newton_schulz(host(X[i]), ref)
        got = host(Y[i])
        assert rel_f(got, want) <= 2e-2
        assert np.max(np.abs(sv(got) - sv(want))) <= 0.05
    # all 64: every output singular value within the schedule's band around the oracle's range
    Yf = Y.float()
    s = torch.linalg.svdvals(Yf)
    assert torch.isfinite(s).all() and float(s.max()) < 1.6


@pytest.mark.parametrize("rows,cols", [(4096, 11008), (11008, 4096)])
def test_rank_one_input_maps_to_phi5_at_full_size(rows, cols):
    """A rank-1 input has one singular value, exactly 1 after the Frobenius pre-scale, so
    Newton-Schulz returns phi_5(1) u v^T: a closed form that holds at any size.  u and v have
    entries +-2^e, so u v^T is exact in bf16 and every later stage (Gram, polynomial, apply,
    each rounded to bf16 and accumulated in fp32) treats all entries alike up to a power of
    two: the device result stays exactly rank-1 and only its scalar carries rounding.  (A
    generic bf16-rounded u v^T is not rank-1: its rounding noise has tiny singular values,
    which the iteration lifts by design.)  phi_5(1) is the oracle's own iteration on 1 x 1."""
    r = workloads.rng(1201)
    u = np.where(r.random(rows) < 0.5, -1.0, 1.0) * 2.0 ** r.integers(-2, 3, rows)
    v = np.where(r.random(cols) < 0.5, -1.0, 1.0) * 2.0 ** r.integers(-2, 3, cols)
    X = torch.outer(torch.tensor(u, dtype=torch.float32), torch.tensor(v, dtype=torch.float32))
    X = X.to(torch.bfloat16).cuda().contiguous()
    Y = torch.empty_like(X)
    sch = mb.Schedule.fixed(5)
    ws = mb.workspace(mb.ns_workspace_size(1, rows, cols, sch))
    mb.ns_orthogonalize(X, Y, sch, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    phi = float(orc.newton_schulz(np.ones((1, 1)), orc.fixed_schedule(5))[0, 0])
    assert abs(phi - 0.69644) < 1e-4
    uh = u / np.linalg.norm(u)
    vh = v / np.linalg.norm(v)
    Yh = host(Y)
    # project onto u v^T and measure what is left, without forming another full matrix
    coef = float(uh @ Yh @ vh)
    resid2 = float(np.sum(Yh * Yh)) - coef * coef
    assert abs(coef - phi) <= 2e-2 * phi
    assert np.sqrt(max(resid2, 0.0)) <= 1e-3 * phi


def test_zero_gradient_from_zero_momentum_is_pure_decay():
    """M = 0 and G = 0 give X0 = 0, a zero Newton-Schulz output (0 / (0 + eps)), and the
    update reduces to W1 = bf16((1 - lr wd) W0) on every matrix of a mixed set."""
    shapes = [(4096, 4096), (4096, 11008), (11008, 4096), (136, 264), (264, 136)]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1202)
    mats = []
    for rows, cols in shapes:
        W = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda").normal_(0.0, 0.02, generator=gen)
        G = torch.zeros((rows, cols), dtype=torch.bfloat16, device="cuda")
        M = torch.zeros((rows, cols), dtype=torch.float32, device="cuda")
        mats.append(mb.Matrix(W, G, M, torch.empty_like(W)))
    before = [host(m.W) for m in mats]
    hp = mb.hyper(lr=LR, beta=BETA, weight_decay=WD)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    mb.muon_step_batched(mats, hp, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    decay = np.float32(1.0) - np.float32(LR) * np.float32(WD)
    for m, W0 in zip(mats, before):
        assert not torch.any(m.M) and not torch.any(m.O_out.float())
        want = orc.round_to_bf16((np.float32(W0) * decay).astype(np.float64))
        assert np.array_equal(host(m.W), want)


def test_muon_cayley_full_size_tall_and_wide():
    """MuonCayley at the 16 x 4096 x 1024 Stiefel workload size, and its wide transpose
    (16 x 1024 x 4096): two steps each, one sampled matrix against the oracle, the manifold
    invariant on every matrix."""
    for wide in (False, True):
        batch, n, k, lr, beta = 16, 4096, 1024, 3e-3, 0.9
        Ws = workloads.stiefel_problem(seed=1203, batch=batch, n=n, k=k)
        if wide:
            Ws = np.ascontiguousarray(np.swapaxes(Ws, 1, 2))
        W = torch.tensor(Ws, dtype=torch.float32, device="cuda")
        M = torch.zeros_like(W)
        rows, cols = W.shape[1], W.shape[2]
        ws = mb.workspace(mb.muon_cayley_workspace_size(batch, rows, cols))
        i = 5
        Wr, Mr = host(W[i]), np.zeros((rows, cols))
        gen = torch.Generator(device="cuda")
        gen.manual_seed(1204)
        G = torch.empty_like(W)
        for _ in range(2):
            workloads.device_normal_(G, 1.0, gen)
            Gi = host(G[i])
            mb.muon_cayley_step(W, G, M, lr, beta, ws, center=True)
            Wr, Mr = orc.muon_cayley_step(Wr, Gi, Mr, lr, float(np.float32(beta)))
        assert mb.device_status(ws) == mb.MUON_OK
        assert np.max(np.abs(host(W[i]) - Wr)) <= 2e-5
        Wd = W.double()
        gram = Wd @ Wd.transpose(1, 2) if wide else Wd.transpose(1, 2) @ Wd
        eye = torch.eye(gram.shape[-1], dtype=torch.float64, device="cuda")
        assert float((gram - eye).abs().max()) <= 1e-5
        del W, M, G, ws, Wd, gram
        torch.cuda.empty_cache()


def test_host_gradient_step_matches_device_step_on_eight_llama_layers():
    """The host-gradient path at scale: 8 Llama-7B layers (56 matrices, 3.2 GB of bf16
    gradients, 8 chunks) give bit-identical W and M to the device-resident step."""
    layer = [(4096, 4096)] * 4 + [(4096, 11008)] * 2 + [(11008, 4096)]
    shapes = layer * 8
    dev_set = _device_set(shapes, 1205, ())
    host_set = [mb.Matrix(m.W.clone(), m.G.cpu().pin_memory(), m.M.clone()) for m in dev_set]
    hp = mb.hyper(lr=LR, beta=BETA, weight_decay=WD)
    ws_d = mb.workspace(mb.muon_step_workspace_size(dev_set, hp))
    ws_h = mb.workspace(mb.muon_step_host_grad_workspace_size(host_set, hp))
    for _ in range(2):
        mb.muon_step_batched(dev_set, hp, ws_d)
        mb.muon_step_batched_host_grad(host_set, hp, ws_h)
    assert mb.device_status(ws_d) == mb.MUON_OK and mb.device_status(ws_h) == mb.MUON_OK
    for d, h in zip(dev_set, host_set):
        assert torch.equal(d.W, h.W) and torch.equal(d.M, h.M)
