"""CPU checks of the C ABI: the library loads, exports every entry point that
include/muon_b200.h declares, and its host-side argument checks reject bad input before
touching the GPU (these calls return before any CUDA call, so they run without a device).
"""
import ctypes
import os
import re

import pytest

from matrix_orthogonalising_optimizer_02_b200 import binding as mb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon_b200.h")


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MUON_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = header_functions()
    for must in ["muon_step_batched", "ns_orthogonalize", "stiefel_cayley_step", "muon_step_workspace_size",
                 "ns_workspace_size", "stiefel_workspace_size", "muon_status_string"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = mb.load()
    missing = [n for n in header_functions() if not hasattr(lib, n)]
    assert missing == []
    assert sorted(mb.EXPORTED) == header_functions()


def test_status_strings():
    lib = mb.load()
    for s in range(9):
        assert lib.muon_status_string(s) != b"unknown status"
    assert lib.muon_status_string(9) == b"unknown status"
    assert b"sm_100a" in lib.muon_build_info()


def test_workspace_queries_are_host_only():
    s = mb.Schedule.fixed(5)
    a = mb.ns_workspace_size(1, 1024, 1024, s)
    b = mb.ns_workspace_size(2, 1024, 1024, s)
    assert a > 0 and b > a
    split = mb.Schedule.fixed(5, n_split_iters=2)
    assert mb.ns_workspace_size(1, 1024, 1024, split) > a
    assert mb.ns_workspace_size(1, 1000, 1001, s) == 0          # bf16 path needs multiples of 8
    assert mb.ns_workspace_size(1, 1000, 1001, mb.Schedule.fixed(5, fp32_mode=True)) > 0
    assert mb.stiefel_workspace_size(16, 4096, 1024) > 16 * 4096 * 1024 * 8
    assert mb.stiefel_workspace_size(1, 10, 20) == 0            # n < k
    # MuonCayley takes wide batches: the transposed plan plus the transposes of W and M
    assert mb.muon_cayley_workspace_size(2, 64, 256) >= mb.stiefel_workspace_size(2, 256, 64) + 2 * 2 * 64 * 256 * 4
    assert mb.muon_cayley_workspace_size(2, 256, 64) == mb.stiefel_workspace_size(2, 256, 64)
    assert mb.muon_cayley_workspace_size(1, 5000, 4100) == 0     # min(n, k) > 4096


def _descs(shapes, ptr=1 << 20):
    arr = (mb.MatrixDesc * len(shapes))()
    for i, (r, c) in enumerate(shapes):
        arr[i] = mb.MatrixDesc(ptr, ptr, ptr, None, r, c, mb.MUON_BF16, mb.MUON_BF16)
    return arr


def test_step_workspace_grouping_bounds():
    lib = mb.load()
    hp, _keep = mb.hyper(0.02)
    shapes = [(4096, 4096)] * 4 + [(4096, 11008)] * 3
    d = _descs(shapes)
    full = lib.muon_step_workspace_size(d, len(shapes), ctypes.byref(hp))
    small = lib.muon_step_workspace_min(d, len(shapes), ctypes.byref(hp))
    assert 0 < small < full
    # the 7-matrix Llama layer: X ping/pong + A, B per matrix, bf16
    data = sum(2 * r * c * 2 + 2 * min(r, c) ** 2 * 2 for r, c in shapes)
    assert full >= data


def test_step_argument_errors():
    lib = mb.load()
    hp, _keep = mb.hyper(0.02)
    ws = ctypes.c_void_p(1 << 24)
    assert lib.muon_step_batched(None, 1, ctypes.byref(hp), ws, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG
    d = _descs([(64, 64)])
    assert lib.muon_step_batched(d, 0, ctypes.byref(hp), ws, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG
    d = _descs([(60, 64)])
    assert lib.muon_step_batched(d, 1, ctypes.byref(hp), ws, 1 << 30, None) == mb.MUON_ERR_UNSUPPORTED_SHAPE
    d = _descs([(64, 64)], ptr=(1 << 20) + 4)
    assert lib.muon_step_batched(d, 1, ctypes.byref(hp), ws, 1 << 30, None) == mb.MUON_ERR_ALIGNMENT
    d = _descs([(64, 64)])
    assert lib.muon_step_batched(d, 1, ctypes.byref(hp), ws, 100, None) == mb.MUON_ERR_WORKSPACE_TOO_SMALL
    bad = mb.hyper(0.02, schedule=mb.Schedule.fixed(5, n_split_iters=6))
    assert lib.muon_step_batched(d, 1, ctypes.byref(bad[0]), ws, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG
    bad = mb.hyper(float("nan"))
    assert lib.muon_step_batched(d, 1, ctypes.byref(bad[0]), ws, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG
    bad = mb.hyper(0.02, schedule=mb.Schedule.fixed(5, eps=0.0))
    assert lib.muon_step_batched(d, 1, ctypes.byref(bad[0]), ws, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG
    too_many = mb.Schedule([(1.0, 0.0, 0.0)] * (mb.MUON_MAX_NS_ITERS + 1))
    bad = mb.hyper(0.02, schedule=too_many)
    assert lib.muon_step_batched(d, 1, ctypes.byref(bad[0]), ws, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG


def test_ns_and_stiefel_argument_errors():
    lib = mb.load()
    s = mb.Schedule.fixed(5)
    p = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 24)
    assert lib.ns_orthogonalize(None, 0, p, 0, 1, 64, 64, ctypes.byref(s.c), ws, 1 << 30, None) == \
        mb.MUON_ERR_INVALID_ARG
    assert lib.ns_orthogonalize(p, 7, p, 0, 1, 64, 64, ctypes.byref(s.c), ws, 1 << 30, None) == \
        mb.MUON_ERR_INVALID_ARG
    assert lib.ns_orthogonalize(p, 0, p, 0, 1, 64, 68, ctypes.byref(s.c), ws, 1 << 30, None) == \
        mb.MUON_ERR_UNSUPPORTED_SHAPE
    assert lib.ns_orthogonalize(p, 0, p, 0, 1, 64, 64, ctypes.byref(s.c), ctypes.c_void_p((1 << 24) + 16),
                                1 << 30, None) == mb.MUON_ERR_ALIGNMENT
    assert lib.ns_orthogonalize(p, 0, p, 0, 1, 64, 64, ctypes.byref(s.c), ws, 1000, None) == \
        mb.MUON_ERR_WORKSPACE_TOO_SMALL
    assert lib.stiefel_cayley_step(p, p, 1, 16, 32, ctypes.c_float(0.01), ws, 1 << 30, None) == \
        mb.MUON_ERR_UNSUPPORTED_SHAPE
    assert lib.stiefel_cayley_step(None, p, 1, 64, 32, ctypes.c_float(0.01), ws, 1 << 30, None) == \
        mb.MUON_ERR_INVALID_ARG
    assert lib.stiefel_cayley_step(p, p, 1, 64, 32, ctypes.c_float(float("inf")), ws, 1 << 30, None) == \
        mb.MUON_ERR_INVALID_ARG
    assert lib.stiefel_cayley_step(p, p, 1, 64, 32, ctypes.c_float(0.01), ws, 10, None) == \
        mb.MUON_ERR_WORKSPACE_TOO_SMALL


def test_timing_api_is_host_only():
    mb.timing_enable(False)
    mb.timing_reset()
    for kind in mb.KERNEL_KINDS:
        ms, n, work = mb.timing_read(kind)
        assert ms == 0 and n == 0 and work == 0
    with pytest.raises(mb.MuonError):
        mb._check(mb.load().muon_timing_read(99, None, None, None), "timing_read")


def test_host_gradient_workspace_is_host_only_and_bounded():
    lib = mb.load()
    hp, _keep = mb.hyper(0.02)
    shapes = [(4096, 4096)] * 4 + [(4096, 11008)] * 2 + [(11008, 4096)]
    d = _descs(shapes * 4)
    n = len(shapes) * 4
    full = lib.muon_step_workspace_size(d, n, ctypes.byref(hp))
    host = lib.muon_step_host_grad_workspace_size(d, n, ctypes.byref(hp))
    # one chunk's step workspace plus two staging slots: well below the whole set's workspace
    # plus its gradients, and at least two slots of the largest chunk's bf16 gradients
    grads = sum(r * c * 2 for r, c in shapes * 4)
    assert 2 * grads / 8 <= host < full
    assert lib.muon_step_host_grad_workspace_size(d, 0, ctypes.byref(hp)) == 0


def test_host_gradient_step_argument_errors_are_host_side():
    """Validation of the host-gradient step happens before any CUDA call."""
    lib = mb.load()
    hp, _keep = mb.hyper(0.02)
    ws = ctypes.c_void_p(1 << 24)
    d = _descs([(64, 64)])
    assert lib.muon_step_batched_host_grad(None, 1, ctypes.byref(hp), ws, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_step_batched_host_grad(d, 0, ctypes.byref(hp), ws, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_step_batched_host_grad(d, 1, ctypes.byref(hp), None, 1 << 30, None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_step_batched_host_grad(d, 1, ctypes.byref(hp), ctypes.c_void_p((1 << 24) + 16), 1 << 30,
                                           None) == mb.MUON_ERR_ALIGNMENT
    d = _descs([(60, 64)])
    assert lib.muon_step_batched_host_grad(d, 1, ctypes.byref(hp), ws, 1 << 30, None) == \
        mb.MUON_ERR_UNSUPPORTED_SHAPE


def test_last_error_is_a_string_and_grouping_bounds_the_step_workspace():
    lib = mb.load()
    assert isinstance(lib.muon_last_error(), bytes)
    hp, _keep = mb.hyper(0.02)
    layer = [(4096, 4096)] * 4 + [(4096, 11008)] * 2 + [(11008, 4096)]
    d = _descs(layer * 32)
    full = lib.muon_step_workspace_size(d, len(layer) * 32, ctypes.byref(hp))
    # the 224-matrix set runs in groups whose NS buffers share at most 5 GiB
    per_layer = sum(2 * r * c * 2 + 2 * min(r, c) ** 2 * 2 for r, c in layer)
    assert 4 * per_layer < full < (5 << 30) + (64 << 20)


def test_binding_rejects_tensors_it_cannot_pass_by_pointer():
    """The binding hands the library raw data pointers, so it refuses strided views, a
    non-fp32 momentum buffer and tensors off the GPU before any library call."""
    import torch
    W = torch.zeros((8, 16), dtype=torch.bfloat16)
    M = torch.zeros((8, 16), dtype=torch.float32)
    hp = mb.hyper(0.02)
    with pytest.raises(ValueError, match="contiguous"):
        mb.muon_step_workspace_size([mb.Matrix(torch.zeros((16, 8), dtype=torch.bfloat16).t(), W, M)], hp)
    with pytest.raises(TypeError, match="fp32"):
        mb.muon_step_workspace_size([mb.Matrix(W, W, M.to(torch.bfloat16))], hp)
    with pytest.raises(ValueError, match="CUDA"):
        mb.muon_step_workspace_size([mb.Matrix(W, W, M)], hp)
    with pytest.raises(ValueError, match="contiguous"):
        mb.ns_orthogonalize(torch.zeros((16, 8)).t(), torch.zeros((8, 16)), mb.Schedule.fixed(1), torch.zeros(1))
    with pytest.raises(ValueError, match="CUDA"):
        mb.stiefel_cayley_step(torch.zeros((16, 8)), torch.zeros((16, 8)), 0.01, torch.zeros(1))


def test_wait_selftest_argument_errors_are_host_side():
    lib = mb.load()
    assert lib.muon_selftest_wait_timeout(None, 4096, None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_selftest_wait_timeout(ctypes.c_void_p(1 << 24), 100, None) == mb.MUON_ERR_INVALID_ARG
    assert lib.muon_selftest_wait_timeout(ctypes.c_void_p((1 << 24) + 16), 4096, None) == mb.MUON_ERR_ALIGNMENT
