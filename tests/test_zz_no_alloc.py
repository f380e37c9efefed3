"""The workspace-free Frobenius pre-scaling entry point, for callers that cannot allocate
device memory at the call site (its scratch is a fixed array inside the library).

Checked through the C ABI against the workspace-based path (ns_orthogonalize with zero
iterations) on two calls in a row with different shapes and dtypes, so a second call that
reused stale scratch from the first would show up.  This file is collected last on
purpose: it must pass both alone in a fresh process and after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as orc
from matrix_orthogonalising_optimizer_02_b200 import binding as mb
from matrix_orthogonalising_optimizer_02_b200 import workloads

pytestmark = pytest.mark.gpu

CASES = [
    # batch, rows, cols, input dtype, output dtype, fp32 mode
    (3, 256, 384, torch.bfloat16, torch.bfloat16, False),
    (2, 136, 264, torch.float32, torch.float32, False),
    (1, 130, 70, torch.float32, torch.float32, True),
]


def _reference(X, out_dtype, fp32_mode):
    Y = torch.empty(X.shape, dtype=out_dtype, device="cuda")
    sch = mb.Schedule([], fp32_mode=fp32_mode)
    b, r, c = X.shape
    ws = mb.workspace(mb.ns_workspace_size(b, r, c, sch))
    mb.ns_orthogonalize(X, Y, sch, ws)
    assert mb.device_status(ws) == mb.MUON_OK
    return Y


def _dt(t):
    return mb.MUON_F32 if t == torch.float32 else mb.MUON_BF16


def _call(lib, x_ptr, din, y_ptr, dout, batch, rows, cols, fp32, scale=None):
    return lib.muon_frobenius_prescale_static(
        x_ptr, _dt(din), y_ptr, _dt(dout), batch, rows, cols, int(fp32), ctypes.c_float(1e-7),
        ctypes.c_void_p(scale.data_ptr() if scale is not None else None),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_prescale_two_calls_match_workspace_path():
    lib = mb.load()
    for i, (batch, rows, cols, din, dout, fp32) in enumerate(CASES):
        r = workloads.rng(700 + i)
        X = torch.tensor(r.standard_normal((batch, rows, cols)) * (i + 1), dtype=torch.float32).to(din).cuda()
        Y = torch.full(X.shape, float("nan"), dtype=dout, device="cuda")
        scale = torch.zeros(batch, dtype=torch.float32, device="cuda")
        st = lib.muon_frobenius_prescale_static(
            X.data_ptr(), mb.MUON_F32 if din == torch.float32 else mb.MUON_BF16, Y.data_ptr(),
            mb.MUON_F32 if dout == torch.float32 else mb.MUON_BF16, batch, rows, cols, int(fp32), ctypes.c_float(1e-7),
            ctypes.c_void_p(scale.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == mb.MUON_OK
        ref = _reference(X, dout, fp32)
        torch.cuda.synchronize()
        # same arithmetic in the same order: the tolerance of the zero-iteration parity test
        assert torch.allclose(Y.double(), ref.double(), rtol=1e-6, atol=0.0)
        x0 = X.double() if fp32 else X.to(torch.bfloat16).double()
        norms = x0.flatten(1).norm(dim=1)
        assert torch.allclose(scale.double(), 1.0 / (norms + 1e-7), rtol=1e-6)


def test_static_prescale_rejects_sizes_beyond_the_scratch():
    lib = mb.load()
    X = torch.zeros((1, 8, 8), dtype=torch.float32, device="cuda")
    big_rows = 8192 * 65  # 65 blocks per matrix x 1024 matrices > 65536 blocks
    st = lib.muon_frobenius_prescale_static(X.data_ptr(), mb.MUON_F32, X.data_ptr(), mb.MUON_F32, 1024, big_rows, 1,
                                            0, ctypes.c_float(1e-7), None, None)
    assert st == mb.MUON_ERR_UNSUPPORTED_SHAPE
    st = lib.muon_frobenius_prescale_static(X.data_ptr(), mb.MUON_F32, X.data_ptr(), mb.MUON_F32, 5000, 8, 8,
                                            0, ctypes.c_float(1e-7), None, None)
    assert st == mb.MUON_ERR_UNSUPPORTED_SHAPE


def test_static_prescale_matches_the_oracle():
    """One bf16 case against the oracle's Frobenius pre-scale of the rounded input."""
    lib = mb.load()
    r = workloads.rng(710)
    X = torch.tensor(r.standard_normal((2, 96, 160)), dtype=torch.float32).to(torch.bfloat16).cuda()
    Y = torch.empty(X.shape, dtype=torch.float32, device="cuda")
    assert _call(lib, X.data_ptr(), torch.bfloat16, Y.data_ptr(), torch.float32, 2, 96, 160, False) == mb.MUON_OK
    torch.cuda.synchronize()
    for i in range(2):
        want = orc.frobenius_prescale(X[i].double().cpu().numpy())
        got = Y[i].double().cpu().numpy()
        # fp32 partial sums of 32 squares per thread (relative error below 2^-19 in the squared
        # norm), one rounding of the fp32 scale and one of the product
        assert np.max(np.abs(got - want)) <= 1e-5 * np.max(np.abs(want))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_prescale_unaligned_and_in_place(dtype):
    """Pointers one element past an aligned base, and X_out == X_in, against the workspace
    path on an aligned copy of the same values."""
    lib = mb.load()
    batch, rows, cols = 2, 72, 136
    r = workloads.rng(711)
    n = batch * rows * cols
    base_in = torch.tensor(r.standard_normal(n + 1), dtype=torch.float32).to(dtype).cuda()
    X = base_in[1:].view(batch, rows, cols)                     # one element off the allocation
    ref = _reference(X.contiguous().clone(), dtype, False)
    base_out = torch.full((n + 1,), float("nan"), dtype=dtype, device="cuda")
    Y = base_out[1:].view(batch, rows, cols)
    assert _call(lib, X.data_ptr(), dtype, Y.data_ptr(), dtype, batch, rows, cols, False) == mb.MUON_OK
    torch.cuda.synchronize()
    assert torch.allclose(Y.double(), ref.double(), rtol=1e-6, atol=0.0)
    Z = X.clone()
    assert _call(lib, Z.data_ptr(), dtype, Z.data_ptr(), dtype, batch, rows, cols, False) == mb.MUON_OK
    torch.cuda.synchronize()
    assert torch.allclose(Z.double(), ref.double(), rtol=1e-6, atol=0.0)


def test_static_prescale_nonfinite_input_shows_in_the_scale():
    """No status word: an infinite element gives scale 0 (and NaN at that element), a NaN
    gives a NaN scale; the other matrix of the batch is unaffected."""
    lib = mb.load()
    r = workloads.rng(712)
    for bad, want_scale in ((float("inf"), 0.0), (float("nan"), None)):
        X = torch.tensor(r.standard_normal((2, 64, 64)), dtype=torch.float32).cuda()
        X[0, 3, 5] = bad
        Y = torch.empty_like(X)
        scale = torch.full((2,), 7.0, dtype=torch.float32, device="cuda")
        assert _call(lib, X.data_ptr(), torch.float32, Y.data_ptr(), torch.float32, 2, 64, 64, False,
                     scale) == mb.MUON_OK
        torch.cuda.synchronize()
        s0 = float(scale[0])
        if want_scale is None:
            assert np.isnan(s0) and torch.isnan(Y[0]).all()
        else:
            assert s0 == want_scale and torch.isnan(Y[0, 3, 5]) and int(torch.isnan(Y[0]).sum()) == 1
        x1 = X[1].to(torch.bfloat16).double()
        assert abs(float(scale[1]) - 1.0 / (float(x1.norm()) + 1e-7)) <= 1e-6 * float(scale[1])
