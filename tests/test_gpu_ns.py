"""GPU parity of ns_orthogonalize (through the C ABI) against the fp64 oracle.

Tolerances are the ones the method's target fixes: bf16 Newton-Schulz within 2e-2 relative
Frobenius error and output singular values within +-0.05 of the oracle's; fp32 mode within
1e-4.  Single-product schedules (T = 1 with one non-zero coefficient) isolate each of the
three grouped GEMM stages; their bound is a few bf16 roundings (1e-2).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from matrix_orthogonalising_optimizer_02_b200 import binding as mb
from matrix_orthogonalising_optimizer_02_b200 import workloads
from gpu_helpers import dev, host, rel_f, sv

pytestmark = pytest.mark.gpu

BF16_TOL, BF16_SV_TOL, FP32_TOL = 2e-2, 0.05, 1e-4


def run_ns(X, schedule, out_dtype=torch.bfloat16):
    Xo = torch.empty(X.shape, dtype=out_dtype, device="cuda")
    b, r, c = (1, *X.shape) if X.dim() == 2 else X.shape
    ws = mb.workspace(mb.ns_workspace_size(b, r, c, schedule))
    mb.ns_orthogonalize(X, Xo, schedule, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    return Xo


SHAPES = [(128, 256), (256, 128), (384, 640), (640, 384), (136, 264), (264, 136), (256, 256), (8, 16),
          (16, 8), (1024, 1024), (768, 2304), (3072, 768)]


@pytest.mark.parametrize("shape", SHAPES)
def test_ns_bf16_fixed_schedule(shape):
    r = workloads.rng(100 + shape[0] + 7 * shape[1])
    X = dev(r.standard_normal(shape), torch.bfloat16)
    got = host(run_ns(X, mb.Schedule.fixed(5)))
    want = orc.newton_schulz(host(X), orc.fixed_schedule(5))
    assert rel_f(got, want) <= BF16_TOL
    assert np.max(np.abs(sv(got) - sv(want))) <= BF16_SV_TOL


@pytest.mark.parametrize("abc", [(1.0, 0.0, 0.0), (0.0, 1.0, 0.0), (0.0, 0.0, 1.0), (0.5, -0.25, 0.125)])
@pytest.mark.parametrize("shape", [(384, 640), (640, 384), (136, 264)])
def test_ns_single_iteration_stages(abc, shape):
    r = workloads.rng(200 + shape[0])
    X = dev(r.standard_normal(shape), torch.bfloat16)
    got = host(run_ns(X, mb.Schedule([abc]), out_dtype=torch.float32))
    want = orc.newton_schulz(host(X), [abc])
    assert rel_f(got, want) <= 1e-2


def test_ns_zero_iterations_is_prescale():
    r = workloads.rng(300)
    X = dev(r.standard_normal((200, 96)), torch.float32)
    got = host(run_ns(X, mb.Schedule([]), out_dtype=torch.float32))
    want = orc.frobenius_prescale(orc.round_to_bf16(host(X)))
    assert rel_f(got, want) <= 1e-6


def test_ns_batched_matches_per_matrix():
    r = workloads.rng(301)
    X = dev(r.standard_normal((3, 256, 384)), torch.bfloat16)
    got = run_ns(X, mb.Schedule.fixed(5))
    for i in range(3):
        one = run_ns(X[i].contiguous(), mb.Schedule.fixed(5))
        assert torch.equal(got[i], one)
        want = orc.newton_schulz(host(X[i]), orc.fixed_schedule(5))
        assert rel_f(host(got[i]), want) <= BF16_TOL


@pytest.mark.parametrize("shape", [(256, 128), (130, 70), (64, 200), (33, 33)])
def test_ns_fp32_mode(shape):
    r = workloads.rng(400 + shape[0])
    X = dev(r.standard_normal(shape) * 0.02, torch.float32)
    got = host(run_ns(X, mb.Schedule.fixed(5, fp32_mode=True), out_dtype=torch.float32))
    want = orc.newton_schulz(host(X), orc.fixed_schedule(5))
    assert rel_f(got, want) <= FP32_TOL


@pytest.mark.parametrize("shape", [(128, 1024), (1024, 128), (96, 40), (40, 96), (8, 16), (120, 120)])
def test_ns_fp32_small_fused(shape):
    """fp32 mode with min(rows, cols) <= 128 runs as one cluster per matrix: the largest long
    side (1024 = 8 slabs of 128), tall and wide, slabs of 5 columns, a tiny matrix and a
    square one, batched, each against the oracle."""
    r = workloads.rng(410 + shape[0] + 3 * shape[1])
    X = dev(r.standard_normal((3, *shape)) * 0.02, torch.float32)
    got = run_ns(X, mb.Schedule.fixed(5, fp32_mode=True), out_dtype=torch.float32)
    for i in range(3):
        want = orc.newton_schulz(host(X[i]), orc.fixed_schedule(5))
        assert rel_f(host(got[i]), want) <= FP32_TOL
    one = run_ns(X[1].contiguous(), mb.Schedule.fixed(5, fp32_mode=True), out_dtype=torch.float32)
    assert torch.equal(one, got[1])


def test_ns_fp32_small_fused_bf16_io_and_hybrid():
    """bf16 input and output around the fp32 iteration, under the 10-iteration hybrid
    schedule."""
    r = workloads.rng(420)
    X = dev(r.standard_normal((2, 64, 200)), torch.bfloat16)
    got = run_ns(X, mb.Schedule.hybrid(fp32_mode=True), out_dtype=torch.bfloat16)
    for i in range(2):
        want = orc.newton_schulz(host(X[i]), orc.hybrid_schedule())
        assert rel_f(host(got[i]), want) <= 4e-3       # one bf16 rounding of the output


@pytest.mark.parametrize("sched,nsplit", [("kj5", 2), ("hybrid", 4)])
def test_ns_low_rank_split(sched, nsplit):
    G = workloads.low_rank_plus_noise(batch=2, n=1024)
    X = dev(G, torch.bfloat16)
    S = mb.Schedule.fixed(5, n_split_iters=nsplit) if sched == "kj5" else mb.Schedule.hybrid(n_split_iters=nsplit)
    ref_sched = orc.fixed_schedule(5) if sched == "kj5" else orc.hybrid_schedule()
    got = run_ns(X, S)
    for i in range(2):
        want = orc.newton_schulz(host(X[i]), ref_sched)
        g = host(got[i])
        assert rel_f(g, want) <= BF16_TOL
        assert np.max(np.abs(sv(g) - sv(want))) <= BF16_SV_TOL


def test_ns_deterministic():
    r = workloads.rng(500)
    X = dev(r.standard_normal((512, 768)), torch.bfloat16)
    a = run_ns(X, mb.Schedule.fixed(5))
    b = run_ns(X, mb.Schedule.fixed(5))
    assert torch.equal(a, b)
