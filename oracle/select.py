"""Oracle: coarse block scores and key-tile selection rules.

TEST INFRASTRUCTURE ONLY (see the package docstring).

* Block scores: S[i, j] = scale * qbar_i . kbar_j with qbar, kbar the tile
  means of Q and K and scale = 1/sqrt(D) (a reading: the pages name routing
  on pooled scores but give no score function; the softmax scale is the
  plainest choice, and top-k and the window rule do not depend on it).
* Top-k: keep the k key tiles with the largest score; equal scores are
  ordered by the lower tile index first. The Wan-14B fine-tuning row of the
  trainable-sparse-attention record (Dataset Splits) fixes the final
  sparsity at 0.9, i.e. k = 0.1 * Nblk.
* Top-p with a top-k floor (FVAttn summary page, Summary and Abstract): in
  the same order, keep the shortest prefix whose softmax mass over the row
  reaches p, and never fewer than k tiles.
* Fixed window (FPSAttention page, ablation rows on the (6,6,1), (6,6,6)
  and (3,3,1) sparsity windows): keep the key tiles whose tile coordinates
  differ from the query tile's by at most the half-widths along (t, h, w);
  the window is clipped at the grid edge.

Kept sets are reported as ascending tile-index lists.

Parity: top-k pinned by the brute-force rank rule and scale invariance;
top-p by exhaustive subset enumeration on small rows and closed-form special
cases; window by its closed-form count; scores by a hand-computed case
(tests/test_oracle_select.py).
"""

from __future__ import annotations

import numpy as np


def block_scores(pq: np.ndarray, pk: np.ndarray, scale: float) -> np.ndarray:
    """[..., N, D] x [..., N, D] -> [..., N, N] fp64, S = scale * pq @ pk^T."""
    return scale * np.matmul(pq.astype(np.float64), np.swapaxes(pk.astype(np.float64), -1, -2))


def _check_row(s: np.ndarray):
    if np.isnan(s).any():
        raise ValueError("NaN block score: selection is undefined")


def rank_order(s_row: np.ndarray) -> np.ndarray:
    """Tile indices ordered by (score descending, index ascending).

    -0.0 and +0.0 compare equal, so they tie and the lower index goes first.
    """
    _check_row(s_row)
    j = np.arange(s_row.shape[0])
    key = -(s_row.astype(np.float64)) + 0.0  # +0.0 folds -0.0 into +0.0
    return np.lexsort((j, key))


def topk_row(s_row: np.ndarray, k: int) -> np.ndarray:
    """Ascending list of the k top-ranked tiles of one score row."""
    n = s_row.shape[0]
    k = min(k, n)
    return np.sort(rank_order(s_row)[:k])


def topp_count(s_row: np.ndarray, p: float, k: int):
    """Number of tiles top-p keeps, plus the prefix masses (for tie windows).

    pi = softmax(s_row) in fp64; c_m = sum of the m top-ranked pi;
    m* = min{m : c_m >= p}; kept = min(N, max(m*, k)).
    """
    n = s_row.shape[0]
    order = rank_order(s_row)
    s = s_row.astype(np.float64)
    e = np.exp(s - s.max())
    pi = e / e.sum()
    c = np.cumsum(pi[order])
    hit = np.nonzero(c >= p)[0]
    m_star = int(hit[0]) + 1 if hit.size else n
    return min(n, max(m_star, k)), c


def topp_row(s_row: np.ndarray, p: float, k: int) -> np.ndarray:
    cnt, _ = topp_count(s_row, p, k)
    return np.sort(rank_order(s_row)[:cnt])


def window_row(i: int, grid_tiles, half) -> np.ndarray:
    """Ascending key tiles within the (t, h, w) half-widths of query tile i."""
    nT, nH, nW = grid_tiles
    a, b, c = half
    ti, hi, wi = i // (nH * nW), (i // nW) % nH, i % nW
    out = []
    for j in range(nT * nH * nW):
        tj, hj, wj = j // (nH * nW), (j // nW) % nH, j % nW
        if abs(tj - ti) <= a and abs(hj - hi) <= b and abs(wj - wi) <= c:
            out.append(j)
    return np.array(out, dtype=np.int64)


def select_rows(S: np.ndarray, rule: str, *, k: int = 0, p: float = 0.0,
                grid_tiles=None, half=None):
    """Apply a rule to every row of S [..., N, N] -> list of ascending lists.

    Returns (lists, shape) where lists is a flat Python list over S's leading
    dims and query tiles in C order.
    """
    N = S.shape[-1]
    flat = S.reshape(-1, N)
    lists = []
    for r in range(flat.shape[0]):
        i = r % N
        if rule == "topk":
            lists.append(topk_row(flat[r], k))
        elif rule == "topp":
            lists.append(topp_row(flat[r], p, k))
        elif rule == "window":
            lists.append(window_row(i, grid_tiles, half))
        else:
            raise ValueError(rule)
    return lists


def lists_to_mask(lists, N: int) -> np.ndarray:
    """Flat list of per-row kept lists -> boolean block mask [rows, N]."""
    m = np.zeros((len(lists), N), dtype=bool)
    for r, lst in enumerate(lists):
        m[r, lst] = True
    return m
