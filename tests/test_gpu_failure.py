"""Failure detection without a GPU fault: a bounded device wait that runs out (on an
mbarrier nothing completes) must end its kernel, report MUON_ERR_DEVICE_TIMEOUT through the
workspace status word and leave the context usable for the next call."""
import time

import pytest
import torch

from matrix_orthogonalising_optimizer_02_b200 import binding as mb

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_reports_status_and_leaves_the_context_usable():
    lib = mb.load()
    ws = mb.workspace(4096)
    t0 = time.time()
    st = lib.muon_selftest_wait_timeout(ws.data_ptr(), 4096, mb._stream(None))
    assert st == mb.MUON_OK
    assert mb.device_status(ws) == mb.MUON_ERR_DEVICE_TIMEOUT
    assert 3.5 < time.time() - t0 < 60          # the wait's 4 s limit, not a hang
    assert mb.device_status(ws) == mb.MUON_OK    # reading the status clears it
    # the context still runs the library
    X = torch.randn(64, 128, device="cuda").to(torch.bfloat16)
    Y = torch.empty_like(X)
    sch = mb.Schedule.fixed(5)
    ws2 = mb.workspace(mb.ns_workspace_size(1, 64, 128, sch))
    mb.ns_orthogonalize(X, Y, sch, ws2)
    assert mb.device_status(ws2) == mb.MUON_OK
    assert torch.isfinite(Y.float()).all()
