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
from gpu_helpers import bf16_ulp_diff, dev, host, rel_f, sv

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
        if O.shape[0] == O.shape[1] or max(O.shape) <= 3072:
            assert np.max(np.abs(sv(O) - sv(O_ref))) <= 0.05
        s = orc.scale_factor(*W0.shape, "moonlight")
        R = orc.round_to_bf16(orc.muon_update(W0, O, LR, WD, s))
        assert np.mean(bf16_ulp_diff(host(m.W), R) <= 1) > 0.999
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
