"""Multi-GPU host logic for the block-sparse path (one process per GPU).

The path needs no data exchange between GPUs: scoring, both selection scopes
and attention are independent per (batch, head).  Ranks therefore either run
independent layers (weak scaling, what ``bench.py --gpus N`` does) or split
the (batch, head) units of one layer.  For a frozen blockset the cost of a
unit is its kept-pair count, which varies several-fold between heads, so the
split is a longest-processing-time assignment on those counts; every rank
computes the same assignment from the same counts, so no collective is needed
to agree on it.  The only collectives are host-side timing helpers.
"""
from __future__ import annotations

import heapq

import torch
import torch.distributed as dist


def lpt_shards(weights, world: int):
    """Deterministic longest-processing-time split of units into `world` shards.

    Units are taken heaviest first (ties: lower index first) and each goes to
    the currently lightest shard (ties: lower rank).  Returns a list of
    ascending unit-index lists, one per rank.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(weights)), key=lambda i: (-float(weights[i]), i))
    heap = [(0.0, r) for r in range(world)]
    shards = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        shards[r].append(i)
        heapq.heappush(heap, (load + float(weights[i]), r))
    return [sorted(s) for s in shards]


def shard_loads(weights, shards):
    return [sum(float(weights[i]) for i in s) for s in shards]


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (e.g. a device-timed duration) over all ranks."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and torch.device(device).type == "cuda":
            dist.barrier(device_ids=[torch.device(device).index])
        else:
            dist.barrier()
