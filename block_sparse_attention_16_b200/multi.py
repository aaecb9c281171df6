"""Multi-GPU host logic for the block-sparse path (one process per GPU).

The path needs no data exchange between GPUs: scoring, both selection scopes
and attention are independent per (batch, head).  Ranks therefore either run
independent layers (weak scaling, what ``bench.py --gpus N`` does) or split
the (batch, head) units of one layer (``run_sharded_layer``: each rank attends
its units, then one all_gather of the outputs when every rank needs the whole
layer).  For a frozen blockset the cost of a
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


# ---------------------------------------------------------------- one layer split over ranks
def layer_shards(weights, world: int | None = None):
    """The LPT split of a layer's (batch, head) units over the ranks of the
    current process group (or `world` ranks); units are flat b*H + h."""
    if world is None:
        world = dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1
    return lpt_shards(weights, world)


def gather_units(out_local, shards, rank: int, n_units: int):
    """Every rank's unit outputs ([len(shards[r]), ...], rows in the order of
    shards[r]) into the full [n_units, ...] tensor on every rank: one
    all_gather of the shard outputs padded to the largest shard."""
    rest = tuple(out_local.shape[1:])
    full = torch.empty((n_units,) + rest, dtype=out_local.dtype, device=out_local.device)
    world = len(shards)
    if world == 1:
        full[shards[0]] = out_local
        return full
    m = max(len(s) for s in shards)
    pad = torch.zeros((m,) + rest, dtype=out_local.dtype, device=out_local.device)
    pad[:len(shards[rank])] = out_local
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad)
    for r, s in enumerate(shards):
        if s:
            full[s] = bufs[r][:len(s)]
    return full


def run_sharded_layer(q, k, v, weights, compute, gather: bool = True):
    """One layer split over the ranks by (batch, head) unit: this rank runs
    compute(q_units, k_units, v_units, units) on its units (tensors [U', N, d]
    gathered from [B, H, N, d]) and, with `gather`, every rank returns the full
    [B, H, N, d] output (one all_gather; the attention itself exchanges
    nothing).  Without `gather` it returns (units, its outputs)."""
    B, H, N, d = q.shape
    rank = dist.get_rank() if dist.is_available() and dist.is_initialized() else 0
    shards = layer_shards(weights)
    units = shards[rank]
    idx = torch.tensor(units, dtype=torch.long, device=q.device)
    flat = [x.reshape(B * H, N, d).index_select(0, idx) for x in (q, k, v)]
    out = compute(*flat, units)
    if not gather:
        return units, out
    return gather_units(out, shards, rank, B * H).reshape(B, H, N, d)


def attend_units(lbsa, bs, units):
    """The GPU compute of run_sharded_layer: the library's attention on a subset
    of a blockset's (batch, head) units, through a blockset holding only their
    rows (exported and re-imported as CSR).  A rank left without units (more
    ranks than units) computes nothing and returns an empty [0, N, d] tensor."""
    if len(units) == 0:
        return lambda qu, ku, vu, _units: qu[:0]
    row_ptr, col = lbsa.lbsa_blockset_export(bs)
    nB = bs.nB
    rp = row_ptr.to(torch.int64)
    parts, starts = [], [0]
    for u in units:
        a, b = int(rp[u * nB]), int(rp[(u + 1) * nB])
        seg = rp[u * nB:(u + 1) * nB + 1] - a
        parts.append(col[a:b])
        starts.extend((seg[1:] + starts[-1]).tolist())
    sub_rp = torch.tensor(starts, dtype=torch.int32, device=col.device)
    sub_col = torch.cat(parts) if parts else col[:0]
    sub = lbsa.lbsa_blockset_from_csr(sub_rp, sub_col, 1, len(units), nB, bs.block)

    def compute(qu, ku, vu, _units):
        return lbsa.lbsa_attend(qu[None], ku[None], vu[None], sub)[0]
    return compute
