"""torch.optim front-ends: argument checks on the CPU, and (GPU) two consecutive steps
against the oracle, momentum state carried between them."""
import numpy as np
import pytest
import torch

import oracle as orc
from matrix_orthogonalising_optimizer_02_b200 import workloads
from matrix_orthogonalising_optimizer_02_b200.optim import Muon, MuonCayley
from gpu_helpers import bf16_ulp_diff, host, rel_f


def test_muon_rejects_non_matrices():
    with pytest.raises(ValueError):
        Muon([torch.nn.Parameter(torch.zeros(8))])
    with pytest.raises(ValueError):
        Muon([torch.nn.Parameter(torch.zeros(8, 8))], scale_mode="bogus")
    MuonCayley([torch.nn.Parameter(torch.zeros(4, 8))])              # wide: updated as its transpose
    with pytest.raises(ValueError):
        MuonCayley([torch.nn.Parameter(torch.zeros(8, 4, dtype=torch.bfloat16))])


@pytest.mark.gpu
def test_muon_optimizer_two_steps_match_oracle():
    r = workloads.rng(80)
    shapes = [(128, 256), (256, 128), (64, 64)]
    params = [torch.nn.Parameter(torch.tensor(r.standard_normal(s) * 0.02, dtype=torch.float32)
                                 .to(torch.bfloat16).cuda()) for s in shapes]
    opt = Muon(params, lr=0.02, momentum=0.95, weight_decay=0.01, nesterov=True)
    W = [host(p) for p in params]
    M = [np.zeros(s) for s in shapes]
    beta = float(np.float32(0.95))
    for step in range(2):
        grads = [r.standard_normal(s) * 1e-3 for s in shapes]
        for p, g in zip(params, grads):
            p.grad = torch.tensor(g, dtype=torch.float32).to(torch.bfloat16).cuda()
        opt.step()
        for i, p in enumerate(params):
            G = orc.round_to_bf16(grads[i])
            M1, U = orc.momentum(M[i], G, beta, nesterov=True)
            M1_gpu = host(opt.state[p]["momentum_buffer"])
            assert np.max(np.abs(M1_gpu - M1)) <= 1e-6 * max(1.0, np.max(np.abs(M1)))
            O = orc.newton_schulz(orc.ns_input(beta * M1_gpu + G), orc.fixed_schedule(5))
            W1 = orc.round_to_bf16(orc.muon_update(W[i], O, 0.02, 0.01, orc.scale_factor(*shapes[i])))
            got = host(p)
            # O enters through the GPU's bf16 Newton-Schulz: bound the weight change by it
            d_ref, d_got = W1 - W[i], got - W[i]
            assert rel_f(d_got, d_ref) <= 3e-2
            W[i], M[i] = got, M1_gpu


@pytest.mark.gpu
def test_muon_cayley_optimizer_steps_stay_orthonormal():
    Ws = workloads.stiefel_problem(seed=81, batch=2, n=128, k=32)
    params = [torch.nn.Parameter(torch.tensor(w, dtype=torch.float32, device="cuda")) for w in Ws]
    opt = MuonCayley(params, lr=3e-3, momentum=0.9)
    ref = [w.copy() for w in Ws]
    Mr = [np.zeros_like(w) for w in Ws]
    r = workloads.rng(82)
    for _ in range(3):
        grads = [r.standard_normal(w.shape) for w in Ws]
        for p, g in zip(params, grads):
            p.grad = torch.tensor(g, dtype=torch.float32, device="cuda")
        opt.step()
        for i in range(2):
            ref[i], Mr[i] = orc.muon_cayley_step(ref[i], orc.round_to_f32(grads[i]), Mr[i], 3e-3,
                                                 float(np.float32(0.9)))
    for i, p in enumerate(params):
        assert np.max(np.abs(host(p) - ref[i])) <= 2e-5
        assert orc.orthogonality_error(host(p)) <= 1e-5
