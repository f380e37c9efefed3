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
