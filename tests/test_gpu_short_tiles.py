"""Tiles of fewer than 64 tokens (the (3,4,4) tile of the FPSAttention tile
ablation): each tile is stored as 64 rows whose last 64 - V are padding. The
kernels must treat those rows like the padded slots at the grid's edge: never
pooled, never keys, never written back to the natural layout.

Checked against the oracle, which tiles with V = 48 rows: the GPU's tiled
tensors are compared on their first V rows (the rest must be zero), the
natural-layout outputs directly.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_reorder_b200.datagen import Workload, make_qkv
from oracle import attention, tiling
from tests.helpers import lists_from_device, lists_to_device, to64

pytestmark = pytest.mark.gpu

CASES = {
    # keys-on-M kernel (head_dim 128), top-k and top-p
    "tile344_topk": Workload("tile344_topk", 1, 2, 128, 7, 10, 13, "topk", k=5, seed=31, tile=(3, 4, 4)),
    "tile344_topp": Workload("tile344_topp", 1, 2, 128, 8, 9, 11, "topp", k=2, p=0.9, seed=32,
                             temperature=(0.3, 3.0), tile=(3, 4, 4)),
    # e4m3 window on the keys-on-M kernel
    "tile344_window_fp8": Workload("tile344_window_fp8", 1, 2, 128, 9, 10, 13, "window", win=(1, 1, 0),
                                   qk_fp8=True, seed=33, tile=(3, 4, 4)),
    # paired-tile kernel (head_dim 64)
    "tile344_d64_window": Workload("tile344_d64_window", 1, 2, 64, 7, 9, 10, "window", win=(1, 1, 1),
                                   seed=34, tile=(3, 4, 4)),
}


@pytest.fixture(scope="module")
def bs():
    from block_sparse_attention_reorder_b200 import bsattn
    return bsattn


def _vol(wl):
    return wl.tile[0] * wl.tile[1] * wl.tile[2]


def _to_oracle_tiles(x, wl):
    """GPU tiled [B, Hh, N, 64, D] -> the oracle's [B, Hh, N, V, D]; the padding rows must be zero."""
    a = to64(x)
    assert np.all(a[..., _vol(wl):, :] == 0)
    return a[..., :_vol(wl), :]


@pytest.mark.parametrize("name", list(CASES))
def test_short_tile_reorder_pool_unreorder(bs, name):
    wl = CASES[name]
    plan = bs.Plan.for_workload(wl)
    assert plan.V == 64
    q, _, _ = make_qkv(wl, "cuda")
    xt = torch.full(plan.tiled_shape(), 7.0, dtype=torch.bfloat16, device="cuda")
    pooled = torch.empty((wl.B, wl.heads, plan.N, wl.head_dim), dtype=torch.float32, device="cuda")
    bs.attn_reorder(plan, q, xt, pooled)
    qn = to64(q)
    np.testing.assert_array_equal(_to_oracle_tiles(xt, wl), tiling.reorder(qn, wl.T, wl.H, wl.W, wl.tile))
    np.testing.assert_allclose(to64(pooled), tiling.pool_mean(qn, wl.T, wl.H, wl.W, wl.tile), rtol=1e-5, atol=2e-6)
    back = torch.empty_like(q)
    bs.attn_unreorder(plan, xt, back)
    assert torch.equal(back, q)
    assert bs.attn_check_device_status(plan) == 0


@pytest.mark.parametrize("name", list(CASES))
def test_short_tile_layer_against_oracle(bs, name):
    """attn_layer (natural layout) against the oracle; the natural attention
    equals reorder -> attn_forward -> unreorder bit for bit."""
    wl = CASES[name]
    plan = bs.Plan.for_workload(wl)
    q, k, v = make_qkv(wl, "cuda")
    o = torch.full_like(q, float("nan"))
    lse = torch.full((wl.B, wl.heads, wl.L), float("nan"), dtype=torch.float32, device="cuda")
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    bs.attn_layer(plan, q, k, v, o, plan.workspace("layer"), lse_nat=lse, idx=idx, cnt=cnt)
    assert bs.attn_check_device_status(plan) == 0
    qn, kn, vn = to64(q), to64(k), to64(v)
    qa, ka = qn, kn
    if wl.qk_fp8:
        qa, ka, _, _ = attention.fp8_qk(qn, kn, wl.T, wl.H, wl.W, wl.tile)
    _, _, _, lists = attention.route(qn, kn, wl.T, wl.H, wl.W, wl.rule, tile=wl.tile, k=wl.k, p=wl.p,
                                     half=wl.win)
    got = lists_from_device(idx, cnt)
    agree = [np.array_equal(a, b) for a, b in zip(got, lists)]
    assert np.mean(agree) >= 0.9
    # The attention is checked on the lists the layer used (valid selections).
    o_ref, lse_ref = attention.attention_full(qa, ka, vn, got, wl.T, wl.H, wl.W, wl.tile)
    on = to64(o)
    assert np.isfinite(on).all()
    if wl.qk_fp8:
        assert np.linalg.norm(on - o_ref) / np.linalg.norm(o_ref) <= 1e-2
    else:
        err = np.abs(on - o_ref)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
        np.testing.assert_allclose(to64(lse), lse_ref, rtol=0, atol=2e-2)
    # Natural attention = tiled attention, bit for bit.
    if not wl.qk_fp8:
        ts = plan.tiled_shape()
        tq, tk, tv = (torch.empty(ts, dtype=torch.bfloat16, device="cuda") for _ in range(3))
        for x, t in zip((q, k, v), (tq, tk, tv)):
            bs.attn_reorder(plan, x, t)
        ot = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
        bs.attn_forward(plan, tq, tk, tv, idx, cnt, ot)
        back = torch.empty_like(q)
        bs.attn_unreorder(plan, ot, back)
        o2 = torch.empty_like(q)
        bs.attn_forward_natural(plan, q, k, v, idx, cnt, o2)
        assert bs.attn_check_device_status(plan) == 0
        assert torch.equal(o2, back)


@pytest.mark.parametrize("name", ["tile344_topk", "tile344_d64_window"])
def test_short_tile_backward_against_oracle(bs, name):
    wl = CASES[name]
    plan = bs.Plan.for_workload(wl)
    q, k, v = make_qkv(wl, "cpu")
    g = torch.Generator(device="cpu").manual_seed(200 + wl.seed)
    d_o = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qn, kn, vn, don = (to64(x) for x in (q, k, v, d_o))
    _, _, _, lists = attention.route(qn, kn, wl.T, wl.H, wl.W, wl.rule, tile=wl.tile, k=wl.k, p=wl.p,
                                     half=wl.win, score_dtype=np.float32)
    idx, cnt = lists_to_device(lists, plan.kmax)
    si, sc = plan.list_shapes()
    idx, cnt = idx.view(si), cnt.view(sc)
    ts = plan.tiled_shape()
    tiled = []
    for x in (q, k, v, d_o):
        t = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
        bs.attn_reorder(plan, x.cuda(), t)
        tiled.append(t)
    qt, kt, vt, dot = tiled
    ot = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    bs.attn_forward(plan, qt, kt, vt, idx, cnt, ot, lse)
    dq, dk, dv = (torch.full(ts, float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    bs.attn_backward(plan, qt, kt, vt, ot, dot, lse, idx, cnt, dq, dk, dv, plan.workspace("backward"))
    assert bs.attn_check_device_status(plan) == 0
    ref = attention.attention_backward_full(qn, kn, vn, don, lists, wl.T, wl.H, wl.W, wl.tile)
    for name_, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        nat = tiling.unreorder(_to_oracle_tiles(got, wl), wl.T, wl.H, wl.W, wl.tile)
        err = nat - r
        rel = np.linalg.norm(err) / max(np.linalg.norm(r), 1e-30)
        assert rel <= 1e-2, (name_, rel)
        assert np.abs(err).max() <= 3e-2 * np.abs(r).max(), (name_, np.abs(err).max())
