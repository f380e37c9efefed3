"""Matrix-ownership sharding of the Muon step over data-parallel ranks.

Muon needs whole matrices, so the optimizer state is sharded by matrix, not by element
(prism.simon-ai.net/article/8795: a ZeRO-like scheme that gathers each matrix instead of
chopping it, with a knapsack-style assignment of matrices to GPUs).  Each rank owns a
subset of the matrices, chosen greedily by longest-processing-time on the Newton-Schulz
FLOPs, keeps their momentum, runs one grouped step over them, and then every updated
weight is broadcast from its owner so that all ranks hold the same parameters again.
The exchange goes through torch.distributed (NCCL on GPUs, gloo on CPUs).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def ns_cost(rows: int, cols: int) -> float:
    """Newton-Schulz FLOPs per iteration for one matrix (symmetric Gram and square counted
    once): 3 r^2 s + r^3 with r = min, s = max."""
    r, s = min(rows, cols), max(rows, cols)
    return 3.0 * r * r * s + float(r) ** 3


def lpt_assign(shapes: Sequence[Tuple[int, int]], world: int) -> List[int]:
    """Owner rank of every matrix: largest cost first, each to the least-loaded rank (ties
    to the lowest rank).  Deterministic, so every rank computes the same assignment."""
    order = sorted(range(len(shapes)), key=lambda i: (-ns_cost(*shapes[i]), i))
    load = [0.0] * world
    owner = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda q: (load[q], q))
        owner[i] = r
        load[r] += ns_cost(*shapes[i])
    return owner


class ShardedMuonStep:
    """Owner-computes Muon step for one parameter set replicated on every rank.

    ``weights`` are the replicated parameter tensors (same order on every rank).
    ``step_owned(indices)`` performs the optimizer step for the matrices at `indices`
    (those this rank owns); by default the caller passes a closure around
    ``binding.muon_step_batched``.  ``step()`` runs it and then broadcasts each matrix from
    its owner (one broadcast per matrix, issued in the same order on every rank).
    """

    def __init__(self, weights: Sequence[torch.Tensor], step_owned: Callable[[List[int]], None],
                 group: Optional[dist.ProcessGroup] = None):
        self.weights = list(weights)
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.owner = lpt_assign([tuple(w.shape) for w in self.weights], self.world)
        self.owned = [i for i, o in enumerate(self.owner) if o == self.rank]
        self.step_owned = step_owned

    def step(self):
        if self.owned:
            self.step_owned(self.owned)
        for i, w in enumerate(self.weights):
            src = dist.get_global_rank(self.group, self.owner[i]) if self.group is not None else self.owner[i]
            dist.broadcast(w, src=src, group=self.group)
