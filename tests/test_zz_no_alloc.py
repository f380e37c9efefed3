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
