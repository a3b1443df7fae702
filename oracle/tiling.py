"""Oracle: token tiling of the (T, H, W) latent grid and tile-mean pooling.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Follows the video-aware block organisation of the FVAttn summary page
(Summary, Abstract) and the shared 3D tile granularity of the FPSAttention
page (Approach). The pages give no formula, so this module fixes one:

* the grid is zero-padded up to a multiple of the tile along each axis;
* tile id of token (t, h, w) = ((t // tt) * nH + h // th) * nW + w // tw with
  nT, nH, nW the tile counts per axis;
* row of the token inside its tile = ((t % tt) * th + h % th) * tw + w % tw;
* a token is valid iff t < T, h < H and w < W; padded tokens are zeros and
  never appear in pooling or as keys.

Pooling (a reading, the pages are silent): the mean over the VALID tokens of
a tile. Padding to the next multiple guarantees at least one valid token per
tile.

Parity: pinned by closed-form index maps, the reorder/unreorder round trip,
and constant-tile pooling (tests/test_oracle_tiling.py).
"""

from __future__ import annotations

import numpy as np


def padded_dims(T: int, H: int, W: int, tile=(4, 4, 4)):
    """(Tp, Hp, Wp): each axis rounded up to a multiple of the tile."""
    tt, th, tw = tile
    return (-(-T // tt) * tt, -(-H // th) * th, -(-W // tw) * tw)


def tile_grid(T: int, H: int, W: int, tile=(4, 4, 4)):
    """(nT, nH, nW) tile counts per axis."""
    Tp, Hp, Wp = padded_dims(T, H, W, tile)
    return (Tp // tile[0], Hp // tile[1], Wp // tile[2])


def n_blocks(T, H, W, tile=(4, 4, 4)) -> int:
    nT, nH, nW = tile_grid(T, H, W, tile)
    return nT * nH * nW


def token_tile_and_row(T: int, H: int, W: int, tile=(4, 4, 4)):
    """For every natural token n = (t*H + h)*W + w: its tile id and in-tile row."""
    tt, th, tw = tile
    _, nH, nW = tile_grid(T, H, W, tile)
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    t, h, w = t.ravel(), h.ravel(), w.ravel()
    tid = ((t // tt) * nH + h // th) * nW + w // tw
    row = ((t % tt) * th + h % th) * tw + w % tw
    return tid.astype(np.int64), row.astype(np.int64)


def tile_valid_rows(T: int, H: int, W: int, tile=(4, 4, 4)) -> np.ndarray:
    """Boolean [Nblk, tile volume]: whether each tile slot holds a real token."""
    nb = n_blocks(T, H, W, tile)
    vol = tile[0] * tile[1] * tile[2]
    valid = np.zeros((nb, vol), dtype=bool)
    tid, row = token_tile_and_row(T, H, W, tile)
    valid[tid, row] = True
    return valid


def reorder(x_nat: np.ndarray, T: int, H: int, W: int, tile=(4, 4, 4)) -> np.ndarray:
    """Natural [B, L, heads, D] -> tiled [B, heads, Nblk, vol, D], pads zero."""
    B, L, Hh, D = x_nat.shape
    assert L == T * H * W
    nb = n_blocks(T, H, W, tile)
    vol = tile[0] * tile[1] * tile[2]
    out = np.zeros((B, Hh, nb, vol, D), dtype=x_nat.dtype)
    tid, row = token_tile_and_row(T, H, W, tile)
    for n in range(L):
        out[:, :, tid[n], row[n], :] = x_nat[:, n, :, :]
    return out


def unreorder(x_tiled: np.ndarray, T: int, H: int, W: int, tile=(4, 4, 4)) -> np.ndarray:
    """Tiled [B, heads, Nblk, vol, D] -> natural [B, L, heads, D] (valid tokens)."""
    B, Hh, nb, vol, D = x_tiled.shape
    L = T * H * W
    out = np.zeros((B, L, Hh, D), dtype=x_tiled.dtype)
    tid, row = token_tile_and_row(T, H, W, tile)
    for n in range(L):
        out[:, n, :, :] = x_tiled[:, :, tid[n], row[n], :]
    return out


def pool_mean(x_nat: np.ndarray, T: int, H: int, W: int, tile=(4, 4, 4)) -> np.ndarray:
    """Tile mean over valid tokens, fp64: natural [B, L, heads, D] -> [B, heads, Nblk, D]."""
    B, L, Hh, D = x_nat.shape
    nb = n_blocks(T, H, W, tile)
    tid, _ = token_tile_and_row(T, H, W, tile)
    x = x_nat.astype(np.float64)
    sums = np.zeros((B, Hh, nb, D), dtype=np.float64)
    counts = np.zeros((nb,), dtype=np.float64)
    for n in range(L):
        sums[:, :, tid[n], :] += x[:, n, :, :]
        counts[tid[n]] += 1.0
    assert (counts > 0).all(), "every tile holds at least one valid token"
    return sums / counts[None, None, :, None]
