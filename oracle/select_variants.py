"""Two further block-selection rules (oracle; test infrastructure).

Local + top-k (VMoBA review on pith.science, referee report major comment 2
and "free parameters": the training-free experiments select query-key blocks
by "Local + TopK" with k = 2, 6 or 18).  The pages do not define "local";
reading taken here: the query block's own key block (the diagonal j = i of the
block grid, both in the same token order), plus the k highest-scoring other
key blocks of the row.  Ordering as in the threshold rule: fp32 score bits
descending, then lower key-block index first.  Rows keep min(k + 1, nB)
blocks.

Top-p with a per-head floor (SCOPE abstract on mlsift.com: hybrid Top-p /
Top-k selection whose Top-k is set per head while running, as the mean of the
key counts the first pass kept in that head, each weighted by the size of its
query cluster; only clusters that kept fewer than that receive more keys).  Block-level reading taken here:
  * initial counts c_i: the row-scope threshold rule of select.py (p);
  * weights: the valid tokens of query block i, v_i = min(block, n_valid - i*block);
  * floor K_h = ceil(sum_i v_i c_i / sum_i v_i), exact integer arithmetic;
  * row i keeps the first max(c_i, min(K_h, nB)) blocks of its sorted order
    (the threshold prefix extended by the next-ranked blocks).
p >= 1 keeps every block, as in the threshold rule.
"""
from __future__ import annotations

import numpy as np

from .select import _segment_keep, _weights, csr_from_rows


def _order(bits_row: np.ndarray) -> np.ndarray:
    """Key-block ids by score bits descending, then id ascending."""
    n = bits_row.shape[0]
    return np.lexsort((np.arange(n), -bits_row.astype(np.int64)))


def select_local_topk(scores, k: int):
    """Per (b, h, i): {i} plus the k top-ranked key blocks j != i -> CSR."""
    x = np.ascontiguousarray(np.asarray(scores, dtype=np.float32))
    B, H, nQ, nK = x.shape
    if nQ != nK:
        raise ValueError("scores must be square per head")
    if k < 0:
        raise ValueError("k must be >= 0")
    bits, _ = _weights(x)
    rows = []
    for b in range(B):
        for h in range(H):
            for i in range(nQ):
                order = [j for j in _order(bits[b, h, i]) if j != i]
                rows.append(np.sort(np.asarray([i] + order[:k], dtype=np.int64)))
    return csr_from_rows(rows)


def floor_of_head(counts, n_valid: int, block: int) -> int:
    """ceil(sum_i v_i c_i / sum_i v_i) with v_i the valid tokens of query block i."""
    nQ = len(counts)
    v = [min(block, n_valid - i * block) for i in range(nQ)]
    num = sum(int(vi) * int(ci) for vi, ci in zip(v, counts))
    den = sum(v)
    return -((-num) // den)


def select_topp_floor(scores, p: float, n_valid: int, block: int):
    """Row-scope threshold rule, then each row raised to the head's floor -> CSR."""
    x = np.ascontiguousarray(np.asarray(scores, dtype=np.float32))
    B, H, nQ, nK = x.shape
    if nQ != nK:
        raise ValueError("scores must be square per head")
    if not (nQ - 1) * block < n_valid <= nQ * block:
        raise ValueError("n_valid does not match the block grid")
    bits, w = _weights(x)
    rows = []
    for b in range(B):
        for h in range(H):
            init = [_segment_keep(bits[b, h, i], w[b, h, i], p) for i in range(nQ)]
            counts = [len(r) for r in init]
            K = floor_of_head(counts, n_valid, block)
            for i in range(nQ):
                n = max(counts[i], min(K, nK))
                rows.append(np.sort(_order(bits[b, h, i])[:n]).astype(np.int64))
    return csr_from_rows(rows)
