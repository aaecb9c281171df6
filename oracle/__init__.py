"""CPU oracle for block-sparse video attention -- TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 NumPy restatement of what the block-sparse attention path
computes, written from the pages' prose:

  * LoSA (abstract, scholarbro.com author page of C. Sun): block masses
    measured exactly during one dense step; per head and query block as few
    key/value blocks as keep 99% of the mass; the same block indices
    reused, frozen, at later steps.
  * VMoBA (pith.science review of arXiv 2506.23858, "What carries the
    argument", referee report major comments 1-2, circularity check, free
    parameters): each key block stands in as its mean key, scored by
    query-block means or by every query token; one selection over all
    query-key block (or query-token, key-block) pairs of a head; the least
    count of pairs whose running sum of normalised similarity gets to tau; a
    1D / 2D / 3D block partition that changes from layer to layer; empty query
    rows; the "Local + TopK" selection of the training-free experiments.
  * SCOPE (abstract, mlsift.com): hybrid Top-p with a per-head Top-k floor,
    the size-weighted mean of the counts the first pass kept.
  * EG-Sparse (abstract, readsearch.ai page of arXiv 2610.14672): heads whose
    scores have low entropy select jointly with a group of other heads, the
    rest per row, using only the block scores computed anyway.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It imports nothing from the CUDA library or its
Python binding and shares no helper with them.

Modules
  attention   dense_attention, sparse_attention, token_sparse_attention   (pinned)
  scores      block_mass, meanpool_scores, token_meanpool_scores      (pinned)
  select      select_contract, select_fp64, csr tools  (pinned)
  select_variants  select_local_topk (VMoBA "Local + TopK"), select_topp_floor
              (SCOPE-style per-head floor over row top-p)   (pinned)
  select_routed  head_entropy, route_heads, select_routed (EG-Sparse
              entropy-routed competition domains)    (pinned)
  partition   raster / 1D / 2D / 3D token orders       (pinned)

Every function is pinned by a ``-m "not gpu"`` test against something other
than itself (library routines, closed forms, brute force, hand-worked
examples under ``tests/golden/``); none is "parity unpinned".
"""
from .attention import dense_attention, sparse_attention, token_sparse_attention
from .scores import block_mass, meanpool_scores, token_meanpool_scores
from .select import (select_contract, select_fp64, InvalidScores, threshold_fixed_point,
                     csr_rows, csr_from_rows)
from .select_variants import select_local_topk, select_topp_floor, floor_of_head
from .select_routed import head_entropy, route_heads, select_routed
from .partition import (perm_raster, perm_1d_temporal, perm_2d_frame_tiles, perm_3d_tiles,
                        perm_for_call, PARTITION_CYCLE)

__all__ = [
    "dense_attention", "sparse_attention", "token_sparse_attention", "block_mass", "meanpool_scores",
    "token_meanpool_scores",
    "select_contract", "select_fp64", "InvalidScores", "threshold_fixed_point",
    "csr_rows", "csr_from_rows", "select_local_topk", "select_topp_floor", "floor_of_head",
    "head_entropy", "route_heads", "select_routed",
    "perm_raster", "perm_1d_temporal", "perm_2d_frame_tiles", "perm_3d_tiles",
    "perm_for_call", "PARTITION_CYCLE",
]
