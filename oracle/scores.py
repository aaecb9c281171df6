"""Block scores in fp64 (oracle; test infrastructure).

block_mass -- LoSA's exact block attention mass (abstract, scholarbro.com
author page): from the dense softmax P of one attention step, the mass that
query block i sends to key block j.  The page does not say how the rows of a
query block are combined; the reading used here is the mean over the block's
valid query rows of each row's mass on the key block, so every query-block
row of the score matrix sums to 1:

    mass[b,h,i,j] = (1/|I_i|) * sum_{r in I_i} sum_{c in J_j} P[r, c]

where I_i, J_j are the valid tokens (index < n_valid) of blocks i and j.

meanpool_scores -- VMoBA's block-mean proxy (pith.science review of arXiv
2506.23858, "What carries the argument"): each key block stands in as the
mean of its keys.  The pages score per-token queries against block means; the
block-granular reading used here scores the query-block mean instead:

    qbar_i = mean_{r in I_i} q_r,  kbar_j = mean_{c in J_j} k_c,
    s_ij   = qbar_i . kbar_j / sqrt(d),
    score[b,h,i,j] = exp(s_ij) / sum_{i',j'} exp(s_i'j')   (over the head)

"normalized similarity" (review, circularity check) is read as this softmax
over all query-block x key-block pairs of the head.

token_meanpool_scores -- the same proxy in the pages' own granularity: every
query token scores every key-block mean (the complete token-by-block score
table of referee report major comment 1), and the similarities of one head
are normalised by a softmax over all of its (query token, key block) pairs:

    s_rj = q_r . kbar_j / sqrt(d)      for valid tokens r < n_valid
    score[b,h,r,j] = exp(s_rj) / sum_{r',j'} exp(s_r'j')   (over the head)
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def block_mass(q, k, n_valid: int, block: int, qblocks=None):
    """Exact mean-row block mass [B, H, len(qblocks), nB] (default: all query blocks)."""
    q, k = _f64(q), _f64(k)
    B, H, _, d = q.shape
    nB = -(-n_valid // block)
    qblocks = np.arange(nB) if qblocks is None else np.asarray(qblocks)
    scale = 1.0 / np.sqrt(d)
    out = np.zeros((B, H, len(qblocks), nB))
    for b in range(B):
        for h in range(H):
            kk = k[b, h, :n_valid]
            for n, i in enumerate(qblocks):
                r0, r1 = int(i) * block, min((int(i) + 1) * block, n_valid)
                z = (q[b, h, r0:r1] @ kk.T) * scale
                e = np.exp(z - z.max(axis=1, keepdims=True))
                P = e / e.sum(axis=1, keepdims=True)
                for j in range(nB):
                    c0, c1 = j * block, min((j + 1) * block, n_valid)
                    out[b, h, n, j] = P[:, c0:c1].sum(axis=1).mean()
    return out


def meanpool_scores(q, k, n_valid: int, block: int):
    """Block-mean proxy scores [B, H, nB, nB], softmax-normalised over each head."""
    q, k = _f64(q), _f64(k)
    B, H, _, d = q.shape
    nB = -(-n_valid // block)
    out = np.zeros((B, H, nB, nB))
    for b in range(B):
        for h in range(H):
            qbar = np.stack([q[b, h, i * block:min((i + 1) * block, n_valid)].mean(axis=0)
                             for i in range(nB)])
            kbar = np.stack([k[b, h, j * block:min((j + 1) * block, n_valid)].mean(axis=0)
                             for j in range(nB)])
            s = (qbar @ kbar.T) / np.sqrt(d)
            e = np.exp(s - s.max())
            out[b, h] = e / e.sum()
    return out


def token_meanpool_scores(q, k, n_valid: int, block: int):
    """Per-token proxy scores [B, H, n_valid, nB], softmax-normalised over each head."""
    q, k = _f64(q), _f64(k)
    B, H, _, d = q.shape
    nB = -(-n_valid // block)
    out = np.zeros((B, H, n_valid, nB))
    for b in range(B):
        for h in range(H):
            kbar = np.stack([k[b, h, j * block:min((j + 1) * block, n_valid)].mean(axis=0)
                             for j in range(nB)])
            s = (q[b, h, :n_valid] @ kbar.T) / np.sqrt(d)
            e = np.exp(s - s.max())
            out[b, h] = e / e.sum()
    return out
