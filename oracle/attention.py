"""Dense and block-sparse softmax attention in fp64 (oracle; test infrastructure).

Dense attention is the "dense step" of LoSA (abstract, scholarbro.com author
page): plain bidirectional softmax attention over the whole 3D token sequence,
scale 1/sqrt(d) (the pages never state the scale; the mean-pooled proxy
workload writes 1/sqrt(d), and it is the standard choice).

Sparse attention follows the VMoBA review ("What carries the argument"):
attention runs on the true keys and values of the kept blocks and nothing else,
and the softmax is renormalised over the union of their valid keys.  A query row whose
list is empty (possible under VMoBA's global selection, referee report major
comment 1) attends to nothing: its output is 0 and its log-sum-exp is -inf.

token_sparse_attention is the same with one list per query token (VMoBA's
per-token selection): token r attends to the valid keys of its own kept
blocks.

Arrays are [B, H, S, d] with S >= n_valid; rows >= n_valid are padding that
is never read.  Everything is upcast to float64 (bf16/fp32 inputs convert
exactly).
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def dense_attention(q, k, v, n_valid: int, rows=None):
    """Softmax attention over all valid keys.

    Returns (O, lse): O [B, H, R, d], lse [B, H, R] for the query rows ``rows``
    (default: all valid rows 0..n_valid-1).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, _, d = q.shape
    rows = np.arange(n_valid) if rows is None else np.asarray(rows)
    O = np.zeros((B, H, len(rows), d))
    lse = np.zeros((B, H, len(rows)))
    scale = 1.0 / np.sqrt(d)
    for b in range(B):
        for h in range(H):
            z = (q[b, h, rows] @ k[b, h, :n_valid].T) * scale
            m = z.max(axis=1, keepdims=True)
            e = np.exp(z - m)
            l = e.sum(axis=1, keepdims=True)
            O[b, h] = (e / l) @ v[b, h, :n_valid]
            lse[b, h] = (m + np.log(l))[:, 0]
    return O, lse


def sparse_attention(q, k, v, n_valid: int, block: int, row_ptr, col, qblocks=None):
    """Attention of each query block over the valid keys of its kept key blocks.

    ``row_ptr``/``col`` is a CSR over rows r = (b*H + h)*nB + i (query block i
    of head h, batch b); ``col`` holds key-block ids.  Returns (O, lse) for the
    query blocks ``qblocks`` (default all): O [B, H, len(qblocks)*block, d] with
    rows of a partial last block beyond n_valid left at 0, lse likewise (-inf
    for padded or empty rows).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, _, d = q.shape
    nB = -(-n_valid // block)
    qblocks = np.arange(nB) if qblocks is None else np.asarray(qblocks)
    O = np.zeros((B, H, len(qblocks) * block, d))
    lse = np.full((B, H, len(qblocks) * block), -np.inf)
    scale = 1.0 / np.sqrt(d)
    for b in range(B):
        for h in range(H):
            for n, i in enumerate(qblocks):
                r = (b * H + h) * nB + int(i)
                blocks = np.asarray(col[row_ptr[r]:row_ptr[r + 1]], dtype=np.int64)
                r0, r1 = int(i) * block, min((int(i) + 1) * block, n_valid)
                if len(blocks) == 0:
                    continue
                keys = np.concatenate([np.arange(j * block, min((j + 1) * block, n_valid))
                                       for j in blocks])
                z = (q[b, h, r0:r1] @ k[b, h, keys].T) * scale
                m = z.max(axis=1, keepdims=True)
                e = np.exp(z - m)
                l = e.sum(axis=1, keepdims=True)
                o0 = n * block
                O[b, h, o0:o0 + (r1 - r0)] = (e / l) @ v[b, h, keys]
                lse[b, h, o0:o0 + (r1 - r0)] = (m + np.log(l))[:, 0]
    return O, lse


def token_sparse_attention(q, k, v, n_valid: int, block: int, row_ptr, col, tokens=None):
    """Attention of each query token over the valid keys of its own kept key blocks.

    ``row_ptr``/``col`` is a CSR over rows r = (b*H + h)*n_valid + t (query
    token t of head h, batch b); ``col`` holds key-block ids.  Returns (O, lse)
    for the tokens ``tokens`` (default all valid): O [B, H, len(tokens), d],
    lse [B, H, len(tokens)]; an empty list gives O = 0 and lse = -inf.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, _, d = q.shape
    tokens = np.arange(n_valid) if tokens is None else np.asarray(tokens)
    O = np.zeros((B, H, len(tokens), d))
    lse = np.full((B, H, len(tokens)), -np.inf)
    scale = 1.0 / np.sqrt(d)
    for b in range(B):
        for h in range(H):
            for n, t in enumerate(tokens):
                r = (b * H + h) * n_valid + int(t)
                blocks = np.asarray(col[row_ptr[r]:row_ptr[r + 1]], dtype=np.int64)
                if len(blocks) == 0:
                    continue
                keys = np.concatenate([np.arange(j * block, min((j + 1) * block, n_valid))
                                       for j in blocks])
                z = (k[b, h, keys] @ q[b, h, int(t)]) * scale
                m = z.max()
                e = np.exp(z - m)
                l = e.sum()
                O[b, h, n] = (e / l) @ v[b, h, keys]
                lse[b, h, n] = m + np.log(l)
    return O, lse
