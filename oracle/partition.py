"""Token orders that turn a (T, H, W) video grid into key/query blocks (oracle).

VMoBA (pith.science review of arXiv 2506.23858: "What carries the argument",
"Load-bearing premise", free parameters) partitions tokens into blocks along
one, two or three axes and cycles 1D -> 2D -> 3D across layers with a fixed
mod-3 schedule.  The pages give block sizes per resolution but no exact
ordering; the readings used here (all return ``perm`` with
``blocked[slot] = raster[perm[slot]]``, raster index (t*H + h)*W + w):

  raster          identity
  1D temporal     tokens ordered with t fastest: slot = (h*W + w)*T + t
  2D frame tiles  frame by frame; inside a frame, th x tw spatial tiles in
                  raster tile order, tokens raster inside a tile; edge tiles
                  truncated
  3D tiles        tt x th x tw tiles in raster tile order, tokens raster inside
                  a tile, edge tiles truncated

Consecutive ``block`` slots then form one block; the tail is padding.
Plain Python loops: obviously correct, O(T*H*W).
"""
from __future__ import annotations

import numpy as np

PARTITION_CYCLE = ("1d", "2d", "3d")


def perm_raster(T, H, W):
    return np.arange(T * H * W, dtype=np.int64)


def perm_1d_temporal(T, H, W):
    out = []
    for h in range(H):
        for w in range(W):
            for t in range(T):
                out.append((t * H + h) * W + w)
    return np.asarray(out, dtype=np.int64)


def perm_2d_frame_tiles(T, H, W, th=8, tw=8):
    out = []
    for t in range(T):
        for h0 in range(0, H, th):
            for w0 in range(0, W, tw):
                for h in range(h0, min(h0 + th, H)):
                    for w in range(w0, min(w0 + tw, W)):
                        out.append((t * H + h) * W + w)
    return np.asarray(out, dtype=np.int64)


def perm_3d_tiles(T, H, W, tt=4, th=4, tw=4):
    out = []
    for t0 in range(0, T, tt):
        for h0 in range(0, H, th):
            for w0 in range(0, W, tw):
                for t in range(t0, min(t0 + tt, T)):
                    for h in range(h0, min(h0 + th, H)):
                        for w in range(w0, min(w0 + tw, W)):
                            out.append((t * H + h) * W + w)
    return np.asarray(out, dtype=np.int64)


def perm_for_call(call: int, T, H, W, tile=(4, 4, 4), frame_tile=(8, 8)):
    """VMoBA's cyclic schedule: call c uses PARTITION_CYCLE[c mod 3]."""
    kind = PARTITION_CYCLE[call % 3]
    if kind == "1d":
        return perm_1d_temporal(T, H, W)
    if kind == "2d":
        return perm_2d_frame_tiles(T, H, W, *frame_tile)
    return perm_3d_tiles(T, H, W, *tile)
