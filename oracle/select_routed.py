"""Entropy-routed competition domains (oracle; test infrastructure).

EG-Sparse abstract (readsearch.ai page of arXiv 2610.14672, "Competition
Domains Matter: Selective Head Globalization for Training-Free Sparse
Attention in Video Diffusion Transformers"): the usual block selection lets
the key blocks of one query row of one head compete; EG-Sparse routes the
heads whose scores have low entropy to a pool shared by a group of heads,
keeps per-row selection for the other heads, and needs nothing beyond the block
scores the sparse path computes anyway.

The abstract fixes neither the entropy, the routing rule, the grouping nor
the rule inside a pool.  Readings taken here, each the plainest one the rest
of the pages support:
  * Entropy of a head: each query-block row of its materialised block scores
    x[i, :] is normalised to a distribution pi_ij = x_ij / sum_j x_ij; the row
    entropy is H_i = -sum_j pi_ij ln pi_ij (0 ln 0 = 0; a row summing to 0
    has H_i = 0); the head entropy is the mean of H_i over the nQ rows divided
    by ln(nB), so it lies in [0, 1] (nB = 1 gives 0).
  * Routing: a head is low-entropy when its entropy is < the threshold e.
  * Grouping: the low-entropy heads of one batch element, in ascending head
    order, form consecutive groups of g heads (the last may be smaller).
    g >= H gives one pool for all of them; e > 1 with g >= H is the
    "all-head" pool of the abstract's diagnostic.
  * Competition domain of a pool: for query block i, the (member, key block)
    pairs of its member heads' row i, flat index m*nB + j with m the member's
    rank in the pool.  The materialised scores compete unnormalised (with
    exact block masses every member row sums to 1).  The threshold rule of
    select.py applies unchanged: exact fixed-point weights, score bits
    descending then flat index ascending, the shortest prefix reaching
    ceil(P*W/2^24), at least one pair per domain; p >= 1 keeps all.  A member
    head's row i keeps the pairs of the prefix that are its own, so it may be
    empty (as under head scope; its output is then 0).
  * High-entropy heads: the row-scope threshold rule with the same p.

head_entropy, route_heads and select_routed follow these steps in order.
select_routed takes an optional `entropy` so that the routing decision (a
floating-point comparison deciding integers) can be taken on the same values
the CUDA path computed.
"""
from __future__ import annotations

import math

import numpy as np

from .select import _segment_keep, _weights, csr_from_rows


def head_entropy(scores) -> np.ndarray:
    """Normalised mean row entropy of every head: fp64 [B, H] in [0, 1]."""
    x = np.asarray(scores, dtype=np.float64)
    B, H, nQ, nB = x.shape
    out = np.zeros((B, H), dtype=np.float64)
    if nB == 1:
        return out
    for b in range(B):
        for h in range(H):
            total = 0.0
            for i in range(nQ):
                row = x[b, h, i]
                s = row.sum()
                if s <= 0.0:
                    continue
                pi = row[row > 0.0] / s
                total += float(-(pi * np.log(pi)).sum())
            out[b, h] = total / nQ / math.log(nB)
    return out


def route_heads(entropy, threshold: float, group: int) -> np.ndarray:
    """Pool id of every head, -1 for heads selected per row: int64 [B, H]."""
    e = np.asarray(entropy, dtype=np.float64)
    if group < 1:
        raise ValueError("group must be >= 1")
    B, H = e.shape
    pool = np.full((B, H), -1, dtype=np.int64)
    for b in range(B):
        low = [h for h in range(H) if e[b, h] < threshold]
        for rank, h in enumerate(low):
            pool[b, h] = rank // group
    return pool


def select_routed(scores, p: float, threshold: float, group: int, entropy=None):
    """Entropy-routed selection on fp32 scores [B, H, nB, nB] -> CSR over rows (b*H + h)*nB + i."""
    x = np.ascontiguousarray(np.asarray(scores, dtype=np.float32))
    B, H, nQ, nB = x.shape
    if not (p > 0.0) or math.isnan(p) or p > 1.0:
        raise ValueError("p must lie in (0, 1]")
    bits, w = _weights(x)
    ent = head_entropy(x) if entropy is None else np.asarray(entropy, dtype=np.float64).reshape(B, H)
    pool = route_heads(ent, threshold, group)
    rows = {}
    for b in range(B):
        for h in range(H):
            if pool[b, h] < 0:
                for i in range(nQ):
                    rows[(b, h, i)] = _segment_keep(bits[b, h, i], w[b, h, i], p)
        for k in range(int(pool[b].max()) + 1 if (pool[b] >= 0).any() else 0):
            members = [h for h in range(H) if pool[b, h] == k]
            for i in range(nQ):
                seg_bits = np.concatenate([bits[b, h, i] for h in members])
                seg_w = np.concatenate([w[b, h, i] for h in members])
                kept = _segment_keep(seg_bits, seg_w, p)
                for m, h in enumerate(members):
                    mine = kept[(kept // nB) == m] % nB
                    rows[(b, h, i)] = np.sort(mine)
    ordered = [rows[(b, h, i)] for b in range(B) for h in range(H) for i in range(nQ)]
    return csr_from_rows(ordered)
