"""Pins for the oracle's masked attention (CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import attention, select, tiling


def test_all_kept_equals_torch_sdpa_fp64():
    rng = np.random.default_rng(0)
    L, D = 96, 16
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    o, lse = attention.dense_masked(q, k, v, np.ones((L, L), bool), 1 / math.sqrt(D))
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(t)[None, None] for t in (q, k, v)))[0, 0].numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)
    mask = rng.random((L, L)) < 0.3
    mask[np.arange(L), np.arange(L)] = True
    o2, _ = attention.dense_masked(q, k, v, mask, 0.25)
    ref2 = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(t)[None, None] for t in (q, k, v)),
        attn_mask=torch.from_numpy(mask)[None, None], scale=0.25)[0, 0].numpy()
    np.testing.assert_allclose(o2, ref2, rtol=1e-12, atol=1e-13)


def test_brute_force_triple_loop():
    rng = np.random.default_rng(1)
    Lq, Lk, D = 5, 7, 3
    q, k, v = rng.standard_normal((Lq, D)), rng.standard_normal((Lk, D)), rng.standard_normal((Lk, D))
    mask = rng.random((Lq, Lk)) < 0.6
    mask[:, 0] = True
    o, lse = attention.dense_masked(q, k, v, mask, 0.7)
    for n in range(Lq):
        w = [math.exp(0.7 * sum(q[n, d] * k[m, d] for d in range(D))) if mask[n, m] else 0.0
             for m in range(Lk)]
        z = sum(w)
        assert lse[n] == pytest.approx(math.log(z), rel=1e-13)
        for d in range(D):
            assert o[n, d] == pytest.approx(sum(w[m] * v[m, d] for m in range(Lk)) / z,
                                            rel=1e-12, abs=1e-14)


def test_rows_normalised():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal((40, 8)) * 3, rng.standard_normal((40, 8)) * 3
    mask = rng.random((40, 40)) < 0.5
    mask[:, 3] = True
    o, _ = attention.dense_masked(q, k, np.ones((40, 8)), mask, 1.0)
    np.testing.assert_allclose(o, 1.0, rtol=1e-14)


def test_single_valid_key_returns_its_value():
    """Grid 5x1x1: tile 1 holds only token t=4; attending only tile 1 copies v[4]."""
    T, H, W = 5, 1, 1
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((1, 5, 1, 4)) for _ in range(3))
    lists = [np.array([1]), np.array([1])]
    o, lse = attention.attention_full(q, k, v, lists, T, H, W)
    np.testing.assert_array_equal(o[0, :, 0], np.repeat(v[0, 4:5, 0], 5, axis=0))
    np.testing.assert_allclose(lse[0, 0], 0.5 * q[0, :, 0] @ k[0, 4, 0], rtol=1e-14)


def test_in_tile_permutation_invariance():
    T, H, W = 8, 4, 8
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, T * H * W, 2, 8)) for _ in range(3))
    nb = tiling.n_blocks(T, H, W)
    lists = [np.sort(rng.choice(nb, 2, replace=False)) for _ in range(2 * nb)]
    o, _ = attention.attention_full(q, k, v, lists, T, H, W)
    tid, _ = tiling.token_tile_and_row(T, H, W)
    perm = np.arange(T * H * W)
    for j in range(nb):
        mem = np.nonzero(tid == j)[0]
        perm[mem] = rng.permutation(mem)
    o2, _ = attention.attention_full(q[:, perm], k[:, perm], v[:, perm], lists, T, H, W)
    np.testing.assert_allclose(o2, o[:, perm], rtol=1e-12, atol=1e-13)


def test_rows_form_equals_full_mask_form():
    T, H, W = 6, 5, 9
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((2, T * H * W, 2, 8)) for _ in range(3))
    nb = tiling.n_blocks(T, H, W)
    lists = [np.sort(rng.choice(nb, rng.integers(1, nb + 1), replace=False)) for _ in range(4 * nb)]
    o, lse = attention.attention_full(q, k, v, lists, T, H, W)
    rows = attention.attention_rows(q, k, v, lists, T, H, W)
    for (b, h, i), (tok, oi, li) in rows.items():
        np.testing.assert_allclose(oi, o[b, tok, h], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(li, lse[b, h, tok], rtol=1e-13)


def test_all_tiles_kept_is_dense_attention_over_valid_tokens():
    T, H, W = 5, 6, 7
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((1, T * H * W, 1, 8)) for _ in range(3))
    nb = tiling.n_blocks(T, H, W)
    lists = [np.arange(nb)] * nb
    o, _ = attention.attention_full(q, k, v, lists, T, H, W)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(t[0, :, 0])[None, None] for t in (q, k, v)))[0, 0].numpy()
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=1e-12, atol=1e-13)


def test_fp8_qk_uses_tile_scales():
    T, H, W = 4, 4, 8
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, T * H * W, 1, 16)).astype(np.float32)
    k = q * 3
    qd, kd, (qc, qs), (kc, ks) = attention.fp8_qk(q, k, T, H, W)
    np.testing.assert_array_equal(qc, kc)  # scaling by 3 scales amax and scale alike
    assert qs.shape == (1, 1, 2)
    np.testing.assert_allclose(qd, q, rtol=2 ** -4, atol=float(qs.max()) * 2 ** -9)


@pytest.mark.parametrize("tile", [(2, 4, 8), (6, 8, 8)])
def test_self_tile_lists_match_coordinate_blocks(tile):
    """Each query tile keeping only itself is attention within the coordinate
    block (t // tile_t, h // tile_h, w // tile_w), written out per token."""
    T, H, W = 7, 10, 9
    tt, th, tw = tile
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((1, T * H * W, 1, 4)) for _ in range(3))
    nb = tiling.n_blocks(T, H, W, tile)
    o, _ = attention.attention_full(q, k, v, [np.array([j]) for j in range(nb)], T, H, W, tile)
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    blk = np.stack([t.ravel() // tt, h.ravel() // th, w.ravel() // tw], axis=1)
    for n in range(0, T * H * W, 7):
        keys = np.nonzero((blk == blk[n]).all(axis=1))[0]
        s = np.array([q[0, n, 0] @ k[0, m, 0] for m in keys]) / 2.0
        p = np.exp(s - s.max())
        ref = (p[:, None] * v[0, keys, 0]).sum(axis=0) / p.sum()
        np.testing.assert_allclose(o[0, n, 0], ref, rtol=1e-12, atol=1e-13)


def test_backward_matches_central_differences():
    """dq, dk, dv of L = sum(do * o) against central differences of the
    forward, on a masked case (some rows attend nothing, some partially)."""
    rng = np.random.default_rng(9)
    q, do = rng.standard_normal((6, 5)), rng.standard_normal((6, 5))  # 6 queries, D = 5
    k, v = rng.standard_normal((5, 5)), rng.standard_normal((5, 5))    # 5 keys
    allowed = rng.random((6, 5)) < 0.6
    allowed[2] = False  # a row with no key
    scale = 0.37
    dq, dk, dv = attention.dense_masked_backward(q, k, v, allowed, scale, do)

    def loss(qq, kk, vv):
        return float((attention.dense_masked(qq, kk, vv, allowed, scale)[0] * do).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)
    assert np.all(dq[2] == 0)


def test_backward_all_kept_equals_torch_autograd():
    """All tiles kept: the layer backward is dense attention's, as torch
    autograd of fp64 scaled_dot_product_attention computes it."""
    T, H, W = 5, 6, 7
    rng = np.random.default_rng(10)
    q, k, v, do = (rng.standard_normal((1, T * H * W, 2, 8)) for _ in range(4))
    nb = tiling.n_blocks(T, H, W)
    dq, dk, dv = attention.attention_backward_full(q, k, v, do, [np.arange(nb)] * (2 * nb), T, H, W)
    for h in range(2):
        tq, tk, tv = (torch.from_numpy(x[0, :, h].copy()).requires_grad_(True) for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None])
        o.backward(torch.from_numpy(do[0, :, h])[None, None])
        np.testing.assert_allclose(dq[0, :, h], tq.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dk[0, :, h], tk.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dv[0, :, h], tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_tiles_form_equals_full_mask_form():
    """The per-tile backward (for large grids) equals the [L, L]-mask form."""
    T, H, W = 5, 6, 9
    rng = np.random.default_rng(11)
    q, k, v, do = (rng.standard_normal((1, T * H * W, 2, 8)) for _ in range(4))
    nb = tiling.n_blocks(T, H, W)
    lists = [np.sort(rng.choice(nb, size=3, replace=False)) for _ in range(2 * nb)]
    lists[5] = np.array([], dtype=np.int64)  # a query tile that keeps nothing
    dq, dk, dv = attention.attention_backward_full(q, k, v, do, lists, T, H, W)
    for h in range(2):
        dq_t, dkv_t = attention.attention_backward_tiles(q, k, v, do, lists, T, H, W, h=h,
                                                         qtiles=range(nb), ktiles=range(nb))
        for i, (tok, g) in dq_t.items():
            np.testing.assert_allclose(g, dq[0, tok, h], rtol=1e-12, atol=1e-13)
        for j, (tok, gk, gv) in dkv_t.items():
            np.testing.assert_allclose(gk, dk[0, tok, h], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(gv, dv[0, tok, h], rtol=1e-12, atol=1e-13)


def test_layer_gradient_through_routing_is_the_fixed_mask_gradient():
    """The routing (pool -> score -> select) is piecewise constant in Q and
    K: away from score ties, a small change of Q or K leaves every kept list
    as it is, so the derivative of the whole layer (routing included) is the
    gradient with the kept mask held fixed, and nothing flows back through
    the pooled scores. Central differences of the routed layer, with the
    lists checked unchanged at every probe, against attention_backward_full
    on the routed lists."""
    rng = np.random.default_rng(21)
    T, H, W, D = 4, 8, 12, 8  # 1 x 2 x 3 = 6 tiles of (4,4,4)
    shape = (1, T * H * W, 1, D)
    q, k, v, do = (rng.standard_normal(shape) for _ in range(4))

    def routed(qq, kk):
        return attention.route(qq, kk, T, H, W, "topk", k=2)[3]

    lists = routed(q, k)
    dq, dk, dv = attention.attention_backward_full(q, k, v, do, lists, T, H, W)

    def loss(qq, kk, vv):
        lst = routed(qq, kk)
        assert all(np.array_equal(a, b) for a, b in zip(lst, lists)), "probe crossed a score tie"
        return float((attention.attention_full(qq, kk, vv, lst, T, H, W)[0] * do).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for flat in rng.choice(x.size, size=12, replace=False):
            idx = np.unravel_index(flat, x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(g[idx] - num) <= 1e-6 * max(1.0, abs(num)), (name, idx, g[idx], num)
