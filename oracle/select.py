"""Mass-threshold block selection (oracle; test infrastructure).

Rule (LoSA abstract, scholarbro.com author page): per head and query block,
keep as few key/value blocks as retain at least the share p of the attention
mass (0.99 by default).  Rule (VMoBA review on pith.science,
circularity check and referee report): sort the normalized similarities of a
head's query-key block pairs, keep the smallest count k' whose cumulative sum
reaches tau (0.25), rows may end up empty.

Readings taken where the pages are silent:
  * "meets"/"reaches" means >=.
  * Ties in the sort: higher score first, then lower flat index first.
  * The cumulative sum is taken in exact integer fixed point so that the
    result does not depend on summation order (a GPU scan and this loop must
    agree bit for bit):
        w_i = floor(x_i * 2^32)             (x_i fp32 score, 0 <= x_i < 2)
        W   = sum_i w_i
        P   = round_half_even(p * 2^24)
        T   = ceil(P * W / 2^24)
    keep the shortest prefix of the sorted order whose sum of w is >= T, and
    at least one element.  p >= 1 keeps every element (the dense path).
  * Scores that are NaN, negative (sign bit set, -0.0 included) or >= 2 are
    rejected.
  * Scope "row": one segment per (b, h, query block); scope "head": one
    segment per (b, h) over all nQ*nB pairs, flat index i*nB + j, where the
    nQ rows are query blocks (block-mean proxy) or query tokens (per-token
    proxy).  Kept columns are emitted per row in ascending order (CSR).

select_fp64 is the same rule on fp64 masses with a plain sequential fp64
cumulative sum compared against p * total; it serves invariant checks, not
bit-exact parity.
"""
from __future__ import annotations

import math

import numpy as np


class InvalidScores(ValueError):
    pass


def threshold_fixed_point(p: float, W: int) -> int:
    """T = ceil(round_half_even(p*2^24) * W / 2^24) in exact integer arithmetic."""
    P = round(float(p) * (1 << 24))          # Python round(): half to even; p*2^24 is exact
    num = P * int(W)
    return -((-num) >> 24)


def _segment_keep(bits: np.ndarray, w: np.ndarray, p: float) -> np.ndarray:
    """Indices (into the segment) kept by the fixed-point rule."""
    n = bits.shape[0]
    if p >= 1.0:
        return np.arange(n)
    W = int(w.sum())
    T = threshold_fixed_point(p, W)
    idx = np.arange(n)
    # order: bits descending, then index ascending (lexsort's last key is primary)
    order = np.lexsort((idx, -bits.astype(np.int64)))
    csum = np.cumsum(w[order])              # int64, exact: n * 2^33 < 2^63
    hit = np.nonzero(csum >= T)[0]
    k = int(hit[0]) + 1 if len(hit) else n
    k = max(k, 1)
    return np.sort(order[:k])


def _weights(x32: np.ndarray):
    bits = x32.view(np.uint32)
    if np.any(bits >= np.uint32(0x40000000)):
        raise InvalidScores("scores must be finite, non-negative and < 2")
    w = np.floor(x32.astype(np.float64) * 4294967296.0).astype(np.int64)
    return bits, w


def select_contract(scores, p: float, scope: str = "row"):
    """Fixed-point selection on fp32 scores [B, H, nQ, nB] -> CSR (row_ptr, col).

    Rows of the CSR are r = (b*H + h)*nQ + i; col holds key-block ids.
    """
    x = np.ascontiguousarray(np.asarray(scores, dtype=np.float32))
    B, H, nQ, nK = x.shape
    if not (p > 0.0) or math.isnan(p) or p > 1.0:
        raise ValueError("p must lie in (0, 1]")
    bits, w = _weights(x)
    rows = []
    for b in range(B):
        for h in range(H):
            if scope == "row":
                for i in range(nQ):
                    rows.append(_segment_keep(bits[b, h, i], w[b, h, i], p))
            elif scope == "head":
                kept = _segment_keep(bits[b, h].reshape(-1), w[b, h].reshape(-1), p)
                per = [[] for _ in range(nQ)]
                for f in kept:
                    per[int(f) // nK].append(int(f) % nK)
                rows.extend(np.asarray(sorted(c), dtype=np.int64) for c in per)
            else:
                raise ValueError(scope)
    return csr_from_rows(rows)


def select_fp64(masses, p: float, scope: str = "row"):
    """Same rule on fp64 values with a sequential fp64 cumulative sum (>= p*total)."""
    x = np.asarray(masses, dtype=np.float64)
    B, H, nQ, nK = x.shape

    def keep(seg):
        n = seg.shape[0]
        if p >= 1.0:
            return np.arange(n)
        order = np.lexsort((np.arange(n), -seg))
        total = float(seg.sum())
        c = 0.0
        k = n
        for pos in range(n):
            c += seg[order[pos]]
            if c >= p * total:
                k = pos + 1
                break
        return np.sort(order[:max(k, 1)])

    rows = []
    for b in range(B):
        for h in range(H):
            if scope == "row":
                rows.extend(keep(x[b, h, i]) for i in range(nQ))
            else:
                kept = keep(x[b, h].reshape(-1))
                per = [[] for _ in range(nQ)]
                for f in kept:
                    per[int(f) // nK].append(int(f) % nK)
                rows.extend(np.asarray(sorted(c), dtype=np.int64) for c in per)
    return csr_from_rows(rows)


def csr_from_rows(rows):
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int64)
    for r, c in enumerate(rows):
        row_ptr[r + 1] = row_ptr[r] + len(c)
    col = (np.concatenate([np.asarray(c, dtype=np.int64) for c in rows])
           if row_ptr[-1] else np.zeros(0, dtype=np.int64))
    return row_ptr, col


def csr_rows(row_ptr, col):
    return [np.asarray(col[row_ptr[r]:row_ptr[r + 1]]) for r in range(len(row_ptr) - 1)]
