"""CUDA graphs: after one eager call (which builds and caches the plan), a step issues
only a memset, a pinned-host table copy and kernel launches, so it can be captured once
and replayed.  Replays must equal eager steps bitwise."""
import pytest
import torch

from matrix_orthogonalising_optimizer_02_b200 import binding as mb
from matrix_orthogonalising_optimizer_02_b200 import workloads
from gpu_helpers import dev

pytestmark = pytest.mark.gpu


def _set(seed):
    r = workloads.rng(seed)
    mats = []
    for (rows, cols) in [(256, 768), (768, 256), (256, 256)]:
        mats.append(mb.Matrix(dev(r.standard_normal((rows, cols)) * 0.02, torch.bfloat16),
                              dev(r.standard_normal((rows, cols)) * 1e-3, torch.bfloat16),
                              torch.zeros((rows, cols), dtype=torch.float32, device="cuda")))
    return mats


def test_step_graph_replay_matches_eager():
    eager, graphed = _set(90), _set(90)
    hp = mb.hyper(lr=0.02, weight_decay=0.1)
    ws_e = mb.workspace(mb.muon_step_workspace_size(eager, hp))
    ws_g = mb.workspace(mb.muon_step_workspace_size(graphed, hp))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        mb.muon_step_batched(graphed, hp, ws_g, stream=s)     # builds and caches the plan
    torch.cuda.current_stream().wait_stream(s)
    mb.muon_step_batched(eager, hp, ws_e)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        mb.muon_step_batched(graphed, hp, ws_g)
    for _ in range(3):
        g.replay()
        mb.muon_step_batched(eager, hp, ws_e)
    torch.cuda.synchronize()
    for a, b in zip(eager, graphed):
        assert torch.equal(a.W, b.W) and torch.equal(a.M, b.M)


def test_captured_plan_survives_plan_cache_churn():
    """A captured graph's table copy reads the plan's pinned host tables, so a plan used under
    capture must outlive any number of later plans: replaying after 40 other plans (more than
    the cache holds) still equals the eager steps, and no call reports an error."""
    eager, graphed = _set(91), _set(91)
    hp = mb.hyper(lr=0.02, weight_decay=0.1)
    ws_e = mb.workspace(mb.muon_step_workspace_size(eager, hp))
    ws_g = mb.workspace(mb.muon_step_workspace_size(graphed, hp))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        mb.muon_step_batched(graphed, hp, ws_g, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    mb.muon_step_batched(eager, hp, ws_e)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        mb.muon_step_batched(graphed, hp, ws_g)
    # 40 distinct plans: ns_orthogonalize over 40 shapes
    sch = mb.Schedule.fixed(1)
    for i in range(40):
        rows, cols = 64 + 8 * i, 96
        X = torch.ones((rows, cols), dtype=torch.bfloat16, device="cuda")
        Y = torch.empty_like(X)
        ws = mb.workspace(mb.ns_workspace_size(1, rows, cols, sch))
        mb.ns_orthogonalize(X, Y, sch, ws)
        assert mb.device_status(ws) == mb.MUON_OK
    for _ in range(2):
        g.replay()
        mb.muon_step_batched(eager, hp, ws_e)
    torch.cuda.synchronize()
    for a, b in zip(eager, graphed):
        assert torch.equal(a.W, b.W) and torch.equal(a.M, b.M)
