"""Pins for oracle.partition (CPU): bijection, library rearranges on divisible grids."""
import numpy as np
import pytest
from einops import rearrange

import oracle


@pytest.mark.parametrize("grid", [(4, 8, 8), (21, 30, 52), (5, 7, 9)])
def test_perms_are_bijections(grid):
    T, H, W = grid
    for perm in (oracle.perm_raster(T, H, W), oracle.perm_1d_temporal(T, H, W),
                 oracle.perm_2d_frame_tiles(T, H, W, 8, 8), oracle.perm_3d_tiles(T, H, W, 4, 4, 4)):
        assert np.array_equal(np.sort(perm), np.arange(T * H * W))


def test_3d_tiles_divisible_grid_matches_einops():
    T, H, W = 8, 12, 16
    raster = np.arange(T * H * W).reshape(T, H, W)
    ref = rearrange(raster, "(nt a) (nh b) (nw c) -> (nt nh nw a b c)", a=4, b=4, c=4)
    assert np.array_equal(oracle.perm_3d_tiles(T, H, W, 4, 4, 4), ref)


def test_2d_frame_tiles_divisible_grid_matches_einops():
    T, H, W = 3, 16, 24
    raster = np.arange(T * H * W).reshape(T, H, W)
    ref = rearrange(raster, "t (nh a) (nw b) -> (t nh nw a b)", a=8, b=8)
    assert np.array_equal(oracle.perm_2d_frame_tiles(T, H, W, 8, 8), ref)


def test_1d_temporal_matches_transpose():
    T, H, W = 21, 30, 52
    ref = np.arange(T * H * W).reshape(T, H, W).transpose(1, 2, 0).reshape(-1)
    assert np.array_equal(oracle.perm_1d_temporal(T, H, W), ref)


def test_3d_tiles_truncated_edges_wan_grid():
    T, H, W = 21, 30, 52
    perm = oracle.perm_3d_tiles(T, H, W)
    t, h, w = np.unravel_index(perm, (T, H, W))
    # first tile: the 4x4x4 corner, raster inside
    assert np.array_equal(perm[:64], rearrange(np.arange(T * H * W).reshape(T, H, W)[:4, :4, :4],
                                               "a b c -> (a b c)"))
    # the last tile of the first slab of tiles is the (0, 7, 12) tile: 4 x 2 x 4 tokens
    slab = 4 * H * W
    assert np.all(t[:slab] < 4) and np.all(t[slab:] >= 4)
    assert np.array_equal(np.unique(h[slab - 32:slab]), [28, 29])
    # the final slab has one frame (t = 20)
    assert np.all(t[20 * H * W:] == 20)


def test_cycle_schedule():
    T, H, W = 4, 8, 8
    assert np.array_equal(oracle.perm_for_call(0, T, H, W), oracle.perm_1d_temporal(T, H, W))
    assert np.array_equal(oracle.perm_for_call(4, T, H, W), oracle.perm_2d_frame_tiles(T, H, W))
    assert np.array_equal(oracle.perm_for_call(5, T, H, W), oracle.perm_3d_tiles(T, H, W))
