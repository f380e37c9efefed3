"""GPU parity of the full Muon step (muon_step_batched through the C ABI) against the oracle.

Per element: the fp32 momentum within 1 ulp of the fp64 formula rounded to fp32; the
updated bf16 weight within 1 bf16 ulp of bf16((1 - lr wd) W0 - lr scale O) evaluated with
the GPU's own O; O itself against the oracle Newton-Schulz of the GPU's bf16(M1) within the
bf16 bound (2e-2 relative Frobenius).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from matrix_orthogonalising_optimizer_02_b200 import binding as mb
from matrix_orthogonalising_optimizer_02_b200 import workloads
from gpu_helpers import assert_update_within_bound, dev, f32_ulp_diff, host, rel_f

pytestmark = pytest.mark.gpu

SMALL_SET = [(96, 288), (96, 96), (96, 384), (384, 96), (136, 264)]


def make_set(shapes, seed, w_dtype=torch.bfloat16, g_dtype=torch.bfloat16, m_std=0.0):
    r = workloads.rng(seed)
    mats = []
    for (rows, cols) in shapes:
        W = dev(r.standard_normal((rows, cols)) * 0.02, w_dtype)
        G = dev(r.standard_normal((rows, cols)) * 1e-3, g_dtype)
        M = dev(r.standard_normal((rows, cols)) * m_std, torch.float32)
        O = torch.empty((rows, cols), dtype=torch.float32 if w_dtype == torch.float32 and g_dtype == torch.float32
                        else torch.bfloat16, device="cuda")
        mats.append(mb.Matrix(W, G, M, O))
    return mats


def snapshot(mats):
    return [(host(m.W), host(m.G), host(m.M)) for m in mats]


def check_step(mats, before, lr, wd, beta, nesterov, scale_mode, sched_host, fp32=False):
    # hyper-parameters cross the C ABI as fp32: the oracle takes the same beta
    beta = float(np.float32(beta))
    for m, (W0, G, M0) in zip(mats, before):
        rows, cols = W0.shape
        M1_ref, g_upd = orc.momentum(M0, G, beta, nesterov)
        M1 = host(m.M)
        assert np.max(f32_ulp_diff(M1, orc.round_to_f32(M1_ref))) <= 1
        O = host(m.O_out)
        X0 = orc.ns_input(beta * M1 + G if nesterov else M1, fp32)
        O_ref = orc.newton_schulz(X0, sched_host) if sched_host else orc.frobenius_prescale(X0)
        assert rel_f(O, O_ref) <= (1e-4 if fp32 else 2e-2)
        s = orc.scale_factor(rows, cols, scale_mode)
        assert_update_within_bound(host(m.W), W0, O, lr, wd, s, m.W.dtype == torch.bfloat16)


def test_step_single_fp32_matrix():
    W, G, M = workloads.single_fp32()
    mats = [mb.Matrix(dev(W, torch.float32), dev(G, torch.float32), dev(M, torch.float32),
                      torch.empty(W.shape, dtype=torch.float32, device="cuda"))]
    hp = mb.hyper(lr=0.02, beta=0.95, weight_decay=0.0, schedule=mb.Schedule.fixed(5, fp32_mode=True))
    before = snapshot(mats)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    mb.muon_step_batched(mats, hp, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    check_step(mats, before, 0.02, 0.0, 0.95, False, "moonlight", orc.fixed_schedule(5), fp32=True)
    # and the whole oracle step
    ref = orc.muon_step(W, G, M, lr=0.02, beta=0.95, fp32_mode=True, w_dtype="f32")
    assert rel_f(host(mats[0].O_out), ref["O"]) <= 1e-4


@pytest.mark.parametrize("nesterov", [False, True])
def test_step_fp32_small_fused_mixed_set(nesterov):
    """fp32 mode on a mixed set of small matrices (one fused launch): bf16 and fp32 weights
    and gradients, non-zero momentum, weight decay, tall, wide and ragged slabs."""
    shapes = [(256, 128), (128, 256), (64, 200), (200, 64), (8, 16)]
    mats = []
    r = workloads.rng(17)
    for i, (rows, cols) in enumerate(shapes):
        wd = torch.bfloat16 if i % 2 else torch.float32
        gd = torch.float32 if i % 3 else torch.bfloat16
        mats.append(mb.Matrix(dev(r.standard_normal((rows, cols)) * 0.02, wd),
                              dev(r.standard_normal((rows, cols)) * 1e-3, gd),
                              dev(r.standard_normal((rows, cols)) * 1e-3, torch.float32),
                              torch.empty((rows, cols), dtype=torch.float32, device="cuda")))
    hp = mb.hyper(lr=0.02, beta=0.95, weight_decay=0.1, nesterov=nesterov,
                  schedule=mb.Schedule.fixed(5, fp32_mode=True))
    before = snapshot(mats)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    mb.muon_step_batched(mats, hp, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    check_step(mats, before, 0.02, 0.1, 0.95, nesterov, "moonlight", orc.fixed_schedule(5), fp32=True)


@pytest.mark.parametrize("nesterov", [False, True])
@pytest.mark.parametrize("scale_mode", ["moonlight", "kellerjordan", "mup", "naive"])
def test_step_bf16_mixed_shapes(nesterov, scale_mode):
    mats = make_set(SMALL_SET, 11, m_std=1e-3)
    hp = mb.hyper(lr=0.02, beta=0.95, weight_decay=0.1, nesterov=nesterov, scale_mode=scale_mode)
    before = snapshot(mats)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    mb.muon_step_batched(mats, hp, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    check_step(mats, before, 0.02, 0.1, 0.95, nesterov, scale_mode, orc.fixed_schedule(5))


def test_step_zero_iterations_and_fp32_gradients():
    mats = make_set([(64, 128), (128, 64)], 12, g_dtype=torch.float32)
    hp = mb.hyper(lr=0.05, beta=0.9, weight_decay=0.01, schedule=mb.Schedule([]))
    before = snapshot(mats)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    mb.muon_step_batched(mats, hp, ws)
    check_step(mats, before, 0.05, 0.01, 0.9, False, "moonlight", [])


def test_step_grouped_workspace_is_bitwise_identical():
    a = make_set(SMALL_SET, 13)
    b = make_set(SMALL_SET, 13)
    hp = mb.hyper(lr=0.02, weight_decay=0.1)
    full = mb.workspace(mb.muon_step_workspace_size(a, hp))
    small = mb.workspace(mb.muon_step_workspace_min(b, hp))
    assert small.numel() < full.numel()
    for _ in range(2):
        mb.muon_step_batched(a, hp, full)
        mb.muon_step_batched(b, hp, small)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.W, y.W) and torch.equal(x.M, y.M)


def test_step_resume_matches_uninterrupted():
    """Checkpoint/resume: the library keeps no hidden state, so restoring (W, M) and
    stepping again gives bitwise the same result as an uninterrupted run."""
    a = make_set(SMALL_SET[:3], 14)
    hp = mb.hyper(lr=0.02, weight_decay=0.1)
    ws = mb.workspace(mb.muon_step_workspace_size(a, hp))
    mb.muon_step_batched(a, hp, ws)
    saved = [(m.W.clone(), m.M.clone()) for m in a]
    mb.muon_step_batched(a, hp, ws)
    b = [mb.Matrix(w.clone(), m.G, mm.clone(), torch.empty_like(m.O_out)) for m, (w, mm) in zip(a, saved)]
    ws2 = mb.workspace(mb.muon_step_workspace_size(b, hp))
    mb.muon_step_batched(b, hp, ws2)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.W, y.W) and torch.equal(x.M, y.M)


def test_step_gpt2_layer_shapes():
    mats = make_set(workloads.GPT2_SMALL_LAYER, 15)
    hp = mb.hyper(lr=0.02, weight_decay=0.1)
    before = snapshot(mats)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    mb.muon_step_batched(mats, hp, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    check_step(mats, before, 0.02, 0.1, 0.95, False, "moonlight", orc.fixed_schedule(5))


def test_nonfinite_gradient_is_reported():
    mats = make_set([(64, 64)], 16)
    mats[0].G[3, 5] = float("nan")
    hp = mb.hyper(lr=0.02)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    mb.muon_step_batched(mats, hp, ws)
    assert mb.device_status(ws) == mb.MUON_ERR_NONFINITE
