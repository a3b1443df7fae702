"""Oracle: dense softmax attention under a block mask, in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Block-sparse attention reaches exactly (up to rounding order) the plain
definition "softmax attention in which query token n may attend key token m
iff the tile pair (tile(n), tile(m)) is kept and m is a real (unpadded)
token". This module writes that definition out:

    O_n = sum_m softmax_m(scale * q_n . k_m | allowed(n, m)) * v_m

with scale = 1/sqrt(D) by default. Where the method keeps tile pairs
(FPSAttention page, Approach: tile-wise structured sparse attention; FVAttn
summary page, Summary: routing then a materialised mask; trainable sparse
attention record, Research Type: the block-sparse attention that replaces
full attention), masked pairs contribute exp(-inf) = 0 exactly, so
`attention_rows` may skip them without changing the value; it is pinned
equal to `dense_masked` on small cases.

The e4m3 variant replaces Q and K by their per-tile quantised-dequantised
values (see ``e4m3``) and keeps V as given.

Parity: pinned against torch's scaled_dot_product_attention in fp64 on CPU
for the all-kept mask, a pure-Python triple loop on tiny inputs, softmax
normalisation, the single-key closed form and in-tile permutation
invariance (tests/test_oracle_attention.py). The backward
(``dense_masked_backward``) is pinned by central finite differences of the
forward on tiny masked cases and by torch autograd of fp64 SDPA for the
all-kept mask.
"""

from __future__ import annotations

import math

import numpy as np

from . import e4m3, select, tiling


def dense_masked(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray,
                 scale: float):
    """q [Lq, D], k/v [Lk, D], allowed bool [Lq, Lk] -> (o [Lq, D], lse [Lq]) fp64.

    A row with no allowed key returns o = 0 and lse = -inf.
    """
    s = scale * (q.astype(np.float64) @ k.astype(np.float64).T)
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ v.astype(np.float64)) / np.where(l > 0, l, 1.0)
    lse = np.where(l[:, 0] > 0, m_safe[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)),
                   -np.inf)
    return o, lse


def token_mask(lists_bh, T, H, W, tile=(4, 4, 4)) -> np.ndarray:
    """Kept lists of one (batch, head) [Nblk lists] -> allowed [L, L] token mask."""
    nb = tiling.n_blocks(T, H, W, tile)
    bm = select.lists_to_mask(lists_bh, nb)
    tid, _ = tiling.token_tile_and_row(T, H, W, tile)
    return bm[tid][:, tid]  # natural tokens are all valid keys


def attention_full(q_nat, k_nat, v_nat, lists, T, H, W, tile=(4, 4, 4), scale=None):
    """Whole layer through the materialised [L, L] mask (small grids only).

    q/k/v natural [B, L, heads, D]; lists: flat list over (b, head, tile).
    Returns (o [B, L, heads, D], lse [B, heads, L]).
    """
    B, L, Hh, D = q_nat.shape
    nb = tiling.n_blocks(T, H, W, tile)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = np.zeros((B, L, Hh, D), dtype=np.float64)
    lse = np.zeros((B, Hh, L), dtype=np.float64)
    for b in range(B):
        for h in range(Hh):
            r0 = (b * Hh + h) * nb
            mask = token_mask(lists[r0:r0 + nb], T, H, W, tile)
            o[b, :, h, :], lse[b, h] = dense_masked(q_nat[b, :, h], k_nat[b, :, h],
                                                    v_nat[b, :, h], mask, scale)
    return o, lse


def attention_rows(q_nat, k_nat, v_nat, lists, T, H, W, tile=(4, 4, 4), scale=None,
                   rows=None):
    """Selected query tiles only: for each (b, head, i) in `rows` the outputs of
    the valid tokens of query tile i, attending the valid tokens of its kept
    key tiles. Returns {(b, h, i): (token ids, o [n, D], lse [n])}.
    """
    B, L, Hh, D = q_nat.shape
    nb = tiling.n_blocks(T, H, W, tile)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    tid, _ = tiling.token_tile_and_row(T, H, W, tile)
    members = [np.nonzero(tid == j)[0] for j in range(nb)]
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(Hh) for i in range(nb)]
    out = {}
    for (b, h, i) in rows:
        lst = lists[(b * Hh + h) * nb + i]
        qi = members[i]
        kj = np.concatenate([members[j] for j in lst]) if len(lst) else np.zeros(0, int)
        allowed = np.ones((qi.size, kj.size), dtype=bool)
        o, lse = dense_masked(q_nat[b, qi, h], k_nat[b, kj, h], v_nat[b, kj, h], allowed,
                              scale)
        out[(b, h, i)] = (qi, o, lse)
    return out


def dense_masked_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray,
                          scale: float, do: np.ndarray):
    """Gradients of L = sum(do * o) for o = dense_masked(q, k, v, allowed, scale)[0].

    Plain differentiation of softmax attention (the trainable block-sparse
    attention that "Faster Video Diffusion with Trainable Sparse Attention"
    trains with, reproducibility record, Research Type row): with P the masked
    softmax, dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dO * O)),
    dQ = scale dS K, dK = scale dS^T Q. A row with no allowed key has P = 0 and
    contributes nothing. Returns (dq [Lq, D], dk [Lk, D], dv [Lk, D]) in fp64.
    """
    q, k, v, do = (x.astype(np.float64) for x in (q, k, v, do))
    s = scale * (q @ k.T)
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    l = e.sum(axis=1, keepdims=True)
    p = e / np.where(l > 0, l, 1.0)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - (do * o).sum(axis=1, keepdims=True))
    return scale * (ds @ k), scale * (ds.T @ q), dv


def attention_backward_full(q_nat, k_nat, v_nat, do_nat, lists, T, H, W, tile=(4, 4, 4), scale=None):
    """Gradients of the whole layer through the materialised [L, L] mask (small
    grids only): natural [B, L, heads, D] in, (dq, dk, dv) natural fp64 out."""
    B, L, Hh, D = q_nat.shape
    nb = tiling.n_blocks(T, H, W, tile)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    dq, dk, dv = (np.zeros((B, L, Hh, D), dtype=np.float64) for _ in range(3))
    for b in range(B):
        for h in range(Hh):
            r0 = (b * Hh + h) * nb
            mask = token_mask(lists[r0:r0 + nb], T, H, W, tile)
            dq[b, :, h], dk[b, :, h], dv[b, :, h] = dense_masked_backward(
                q_nat[b, :, h], k_nat[b, :, h], v_nat[b, :, h], mask, scale, do_nat[b, :, h])
    return dq, dk, dv


def attention_backward_tiles(q_nat, k_nat, v_nat, do_nat, lists, T, H, W, tile=(4, 4, 4), scale=None,
                             b=0, h=0, qtiles=(), ktiles=()):
    """Gradients for selected tiles of one (batch, head), without the [L, L]
    mask (large grids): dQ of the valid tokens of each query tile in
    `qtiles`, and dK, dV of the valid tokens of each key tile in `ktiles`.

    dQ_i needs only query tile i and its kept key tiles. dK_j and dV_j sum
    over the query tiles that keep j; each such query row's softmax is taken
    over all of its own kept keys (as the full layer does). Returns
    ({i: (token ids, dq)}, {j: (token ids, dk, dv)}) in fp64.
    """
    B, L, Hh, D = q_nat.shape
    nb = tiling.n_blocks(T, H, W, tile)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    tid, _ = tiling.token_tile_and_row(T, H, W, tile)
    members = [np.nonzero(tid == t)[0] for t in range(nb)]
    rows = lists[(b * Hh + h) * nb:(b * Hh + h + 1) * nb]
    q, k, v, do = (x[b, :, h].astype(np.float64) for x in (q_nat, k_nat, v_nat, do_nat))

    def row_softmax(i):
        """P over query tile i's kept keys, the key token ids, and Delta."""
        qi = members[i]
        kj = np.concatenate([members[j] for j in rows[i]]) if len(rows[i]) else np.zeros(0, int)
        s = scale * (q[qi] @ k[kj].T)
        m = s.max(axis=1, keepdims=True) if kj.size else np.zeros((qi.size, 1))
        e = np.exp(s - m)
        p = e / e.sum(axis=1, keepdims=True) if kj.size else e
        o = p @ v[kj]
        delta = (do[qi] * o).sum(axis=1)
        return qi, kj, p, delta

    dq_out = {}
    for i in qtiles:
        qi, kj, p, delta = row_softmax(i)
        ds = p * (do[qi] @ v[kj].T - delta[:, None])
        dq_out[i] = (qi, scale * (ds @ k[kj]))
    dkv_out = {}
    for j in ktiles:
        kj_tokens = members[j]
        dk = np.zeros((kj_tokens.size, D))
        dv = np.zeros((kj_tokens.size, D))
        for i in range(nb):
            if j not in set(int(x) for x in rows[i]):
                continue
            qi, kj, p, delta = row_softmax(i)
            cols = np.isin(kj, kj_tokens)  # this key tile's columns, in token order
            pj = p[:, cols]
            dsj = pj * (do[qi] @ v[kj[cols]].T - delta[:, None])
            dv += pj.T @ do[qi]
            dk += scale * (dsj.T @ q[qi])
        dkv_out[j] = (kj_tokens, dk, dv)
    return dq_out, dkv_out


def fp8_qk(q_nat, k_nat, T, H, W, tile=(4, 4, 4)):
    """Per-tile e4m3 quantise-dequantise of Q and K.

    Returns (q_deq, k_deq) natural fp64, and (codes, scales) of each in the
    tiled layout.
    """
    res = []
    for x in (q_nat, k_nat):
        xt = tiling.reorder(x.astype(np.float32), T, H, W, tile)
        codes, scales = e4m3.quantize_tiled(xt)
        deq = e4m3.dequantize_tiled(codes, scales)
        res.append((tiling.unreorder(deq, T, H, W, tile), codes, scales))
    return res[0][0], res[1][0], (res[0][1], res[0][2]), (res[1][1], res[1][2])


def route(q_nat, k_nat, T, H, W, rule, *, k=0, p=0.0, half=(0, 0, 0), tile=(4, 4, 4),
          scale=None, score_dtype=np.float64):
    """Pool, score and select: -> (pooled q, pooled k, S, flat kept lists).

    `score_dtype` rounds S before selection (np.float32 mirrors a library that
    stores fp32 scores); the selection itself is exact on whatever S it gets.
    """
    D = q_nat.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    pq = tiling.pool_mean(q_nat, T, H, W, tile)
    pk = tiling.pool_mean(k_nat, T, H, W, tile)
    S = select.block_scores(pq, pk, scale).astype(score_dtype)
    lists = select.select_rows(S, rule, k=k, p=p, grid_tiles=tiling.tile_grid(T, H, W, tile),
                               half=half)
    return pq, pk, S, lists
