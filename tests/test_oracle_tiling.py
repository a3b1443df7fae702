"""Pins for the oracle's tiling and pooling (CPU only)."""
import json
import os

import numpy as np
import pytest

from oracle import tiling
from block_sparse_attention_reorder_b200.datagen import WORKLOADS


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_counts_match_workload_definitions(name, golden_dir):
    g = json.load(open(os.path.join(golden_dir, "workload_counts.json")))[name]
    wl = WORKLOADS[name]
    assert [wl.T, wl.H, wl.W] == g["grid"]
    assert list(wl.tile) == g.get("tile", [4, 4, 4])
    assert list(tiling.padded_dims(wl.T, wl.H, wl.W, wl.tile)) == g["padded"]
    assert tiling.n_blocks(wl.T, wl.H, wl.W, wl.tile) == g["Nblk"]
    if "tiles" in g:
        assert list(tiling.tile_grid(wl.T, wl.H, wl.W, wl.tile)) == g["tiles"]


TILE_CASES = [((5, 6, 7), (4, 4, 4)), ((8, 16, 16), (4, 4, 4)), ((1, 1, 1), (4, 4, 4)),
              ((4, 9, 4), (4, 4, 4)), ((7, 10, 9), (6, 8, 8)), ((5, 6, 11), (2, 4, 8)),
              ((3, 5, 70), (1, 1, 128)), ((7, 10, 13), (3, 4, 4))]


@pytest.mark.parametrize("grid,tile", TILE_CASES)
def test_index_map_by_forward_enumeration(grid, tile):
    """Walk tiles and in-tile slots forwards and check the oracle's inverse map."""
    T, H, W = grid
    tt, th, tw = tile
    nT, nH, nW = tiling.tile_grid(T, H, W, tile)
    assert (nT, nH, nW) == (-(-T // tt), -(-H // th), -(-W // tw))
    tid, row = tiling.token_tile_and_row(T, H, W, tile)
    seen = 0
    for bt in range(nT):
        for bh in range(nH):
            for bw in range(nW):
                j = (bt * nH + bh) * nW + bw
                for dt in range(tt):
                    for dh in range(th):
                        for dw in range(tw):
                            t, h, w = tt * bt + dt, th * bh + dh, tw * bw + dw
                            if t < T and h < H and w < W:
                                n = (t * H + h) * W + w
                                assert tid[n] == j
                                assert row[n] == (dt * th + dh) * tw + dw
                                seen += 1
    assert seen == T * H * W


def test_reorder_round_trip_and_zero_pads():
    rng = np.random.default_rng(0)
    T, H, W = 5, 6, 7
    x = rng.standard_normal((2, T * H * W, 3, 8))
    xt = tiling.reorder(x, T, H, W)
    valid = tiling.tile_valid_rows(T, H, W)
    assert xt.shape == (2, 3, tiling.n_blocks(T, H, W), 64, 8)
    assert np.all(xt[:, :, ~valid, :] == 0)
    assert valid.sum() == T * H * W
    np.testing.assert_array_equal(tiling.unreorder(xt, T, H, W), x)


def test_pool_is_valid_token_mean():
    """Constant input pools to the constant even in partial tiles (pads excluded)."""
    T, H, W = 5, 6, 7
    x = np.full((1, T * H * W, 2, 4), 3.25)
    np.testing.assert_array_equal(tiling.pool_mean(x, T, H, W), 3.25)


@pytest.mark.parametrize("grid,tile", [((6, 5, 9), (4, 4, 4)), ((7, 10, 9), (6, 8, 8)),
                                       ((5, 6, 11), (2, 4, 8)), ((7, 10, 13), (3, 4, 4))])
def test_pool_against_coordinate_masks(grid, tile):
    rng = np.random.default_rng(1)
    T, H, W = grid
    tt, th, tw = tile
    x = rng.standard_normal((1, T * H * W, 2, 3))
    pooled = tiling.pool_mean(x, T, H, W, tile)
    g = x.reshape(1, T, H, W, 2, 3)
    nT, nH, nW = tiling.tile_grid(T, H, W, tile)
    for bt in range(nT):
        for bh in range(nH):
            for bw in range(nW):
                blk = g[0, tt * bt:tt * bt + tt, th * bh:th * bh + th, tw * bw:tw * bw + tw]
                ref = blk.reshape(-1, 2, 3).mean(axis=0)
                np.testing.assert_allclose(pooled[0, :, (bt * nH + bh) * nW + bw], ref,
                                           rtol=1e-13, atol=1e-15)


def test_reorder_round_trip_large_tile():
    rng = np.random.default_rng(2)
    T, H, W, tile = 7, 10, 9, (6, 8, 8)
    x = rng.standard_normal((1, T * H * W, 2, 4))
    xt = tiling.reorder(x, T, H, W, tile)
    assert xt.shape == (1, 2, 2 * 2 * 2, 384, 4)
    valid = tiling.tile_valid_rows(T, H, W, tile)
    assert np.all(xt[:, :, ~valid, :] == 0) and valid.sum() == T * H * W
    np.testing.assert_array_equal(tiling.unreorder(xt, T, H, W, tile), x)
