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
    assert list(tiling.padded_dims(wl.T, wl.H, wl.W)) == g["padded"]
    assert tiling.n_blocks(wl.T, wl.H, wl.W) == g["Nblk"]


@pytest.mark.parametrize("grid", [(5, 6, 7), (8, 16, 16), (1, 1, 1), (4, 9, 4)])
def test_index_map_by_forward_enumeration(grid):
    """Walk tiles and in-tile slots forwards and check the oracle's inverse map."""
    T, H, W = grid
    nT, nH, nW = tiling.tile_grid(T, H, W)
    tid, row = tiling.token_tile_and_row(T, H, W)
    seen = 0
    for bt in range(nT):
        for bh in range(nH):
            for bw in range(nW):
                j = (bt * nH + bh) * nW + bw
                for dt in range(4):
                    for dh in range(4):
                        for dw in range(4):
                            t, h, w = 4 * bt + dt, 4 * bh + dh, 4 * bw + dw
                            if t < T and h < H and w < W:
                                n = (t * H + h) * W + w
                                assert tid[n] == j
                                assert row[n] == (dt * 4 + dh) * 4 + dw
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


def test_pool_against_coordinate_masks():
    rng = np.random.default_rng(1)
    T, H, W = 6, 5, 9
    x = rng.standard_normal((1, T * H * W, 2, 3))
    pooled = tiling.pool_mean(x, T, H, W)
    g = x.reshape(1, T, H, W, 2, 3)
    nT, nH, nW = tiling.tile_grid(T, H, W)
    for bt in range(nT):
        for bh in range(nH):
            for bw in range(nW):
                blk = g[0, 4 * bt:4 * bt + 4, 4 * bh:4 * bh + 4, 4 * bw:4 * bw + 4]
                ref = blk.reshape(-1, 2, 3).mean(axis=0)
                np.testing.assert_allclose(pooled[0, :, (bt * nH + bh) * nW + bw], ref,
                                           rtol=1e-13, atol=1e-15)
