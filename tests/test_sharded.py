"""Matrix-ownership sharding: the assignment (host logic) and the owner-computes /
broadcast exchange on CPU (gloo) with world sizes 2 and 4, and within a subgroup.  The
stand-in step marks each owned matrix with its owner's rank, so after the exchange every
rank must hold the same weights, each changed exactly once, by its owner."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from matrix_orthogonalising_optimizer_02_b200 import workloads
from matrix_orthogonalising_optimizer_02_b200.sharded import ShardedMuonStep, lpt_assign, ns_cost


def test_lpt_assignment_balances_the_llama_set():
    shapes = workloads.llama7b_shapes(32)
    for world in (1, 2, 4, 8):
        owner = lpt_assign(shapes, world)
        assert sorted(set(owner)) == list(range(world))
        load = [0.0] * world
        for i, s in enumerate(shapes):
            load[owner[i]] += ns_cost(*s)
        bound = sum(load) / world + max(ns_cost(*s) for s in shapes)
        assert max(load) <= bound
        assert max(load) / (sum(load) / world) < 1.02         # 224 matrices: near-perfect balance
        assert owner == lpt_assign(shapes, world)             # deterministic


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q, members=None):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # every rank takes part in creating the subgroup, only its members in the exchange
        group = dist.new_group(members) if members is not None else None
        if members is not None and rank not in members:
            q.put((rank, "ok"))
            return
        shapes = [(64, 32), (32, 64), (48, 48), (16, 80), (80, 16), (8, 8), (24, 24), (40, 8)]
        g = torch.Generator().manual_seed(5)
        weights = [torch.randn(s, generator=g) for s in shapes]     # identical on every rank
        before = [w.clone() for w in weights]
        my = dist.get_rank(group) if group is not None else rank

        def step_owned(indices):
            for i in indices:
                weights[i].add_(float(my + 1))

        sh = ShardedMuonStep(weights, step_owned, group=group)
        sh.step()
        for i, w in enumerate(weights):
            assert torch.equal(w, before[i] + float(sh.owner[i] + 1))   # changed once, by its owner
        size = dist.get_world_size(group)
        sums = torch.tensor([float(sum(w.sum() for w in weights))])
        gathered = [torch.zeros(1) for _ in range(size)]
        dist.all_gather(gathered, sums, group=group)
        assert all(torch.equal(x, gathered[0]) for x in gathered)
        q.put((rank, "ok"))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


def _run(world, members=None):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, members)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    results = dict(q.get(timeout=5) for _ in procs)
    assert results == {r: "ok" for r in range(world)}


@pytest.mark.parametrize("world", [2, 4])
def test_owner_computes_then_broadcast_gloo(world):
    _run(world)


def test_owner_computes_then_broadcast_within_a_subgroup():
    """Ranks 1 and 3 of 4 shard among themselves: owners are group ranks, broadcasts use
    their global ranks."""
    _run(4, members=[1, 3])
