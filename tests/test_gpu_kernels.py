"""Kernel-level parity: each C-ABI step against the oracle on the same inputs."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_reorder_b200.datagen import make_qkv, random_scores
from oracle import attention, e4m3, select, tiling
from tests.helpers import (SMALL, assert_topp_equal, assert_valid_selection, lists_from_device,
                           lists_to_device, to64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bs():
    from block_sparse_attention_reorder_b200 import bsattn
    assert torch.cuda.is_available()
    return bsattn


def _plan(bs, wl, **over):
    args = dict(rule=wl.rule, k=wl.k, p=wl.p, win=wl.win, tile=wl.tile, qk_fp8=wl.qk_fp8)
    args.update(over)
    return bs.Plan(wl.B, wl.heads, wl.head_dim, wl.T, wl.H, wl.W, **args)


@pytest.mark.parametrize("name", list(SMALL))
def test_reorder_pool_unreorder(bs, name):
    wl = SMALL[name]
    plan = _plan(bs, wl)
    q, _, _ = make_qkv(wl, "cuda")
    xt = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
    pooled = torch.empty((wl.B, wl.heads, plan.N, wl.head_dim), dtype=torch.float32, device="cuda")
    bs.attn_reorder(plan, q, xt, pooled)
    qn = to64(q)
    np.testing.assert_array_equal(to64(xt), tiling.reorder(qn, wl.T, wl.H, wl.W, wl.tile))
    ref = tiling.pool_mean(qn, wl.T, wl.H, wl.W, wl.tile)
    np.testing.assert_allclose(to64(pooled), ref, rtol=1e-5, atol=2e-6)
    pooled2 = torch.zeros_like(pooled)
    bs.attn_pool(plan, q, pooled2)
    torch.testing.assert_close(pooled2, pooled, rtol=0, atol=0)
    back = torch.empty_like(q)
    bs.attn_unreorder(plan, xt, back)
    assert torch.equal(back, q)
    assert bs.attn_check_device_status(plan) == 0


@pytest.mark.parametrize("name", ["ragged_topk", "tiny_d64"])
def test_block_scores(bs, name):
    wl = SMALL[name]
    plan = _plan(bs, wl)
    q, k, _ = make_qkv(wl, "cuda")
    pq = tiling.pool_mean(to64(q), wl.T, wl.H, wl.W).astype(np.float32)
    pk = tiling.pool_mean(to64(k), wl.T, wl.H, wl.W).astype(np.float32)
    S = torch.empty((wl.B, wl.heads, plan.N, plan.N), dtype=torch.float32, device="cuda")
    bs.attn_block_scores(plan, torch.from_numpy(pq).cuda(), torch.from_numpy(pk).cuda(), S)
    scale = 1 / math.sqrt(wl.head_dim)
    ref = select.block_scores(pq, pk, scale)
    bound = 1e-5 * scale * np.matmul(np.abs(pq).astype(np.float64),
                                     np.swapaxes(np.abs(pk).astype(np.float64), -1, -2)) + 1e-30
    assert np.all(np.abs(to64(S) - ref) <= bound)


@pytest.mark.parametrize("grid,heads,D", [((24, 48, 80), 5, 128), ((20, 44, 84), 6, 64)])
def test_block_scores_large(bs, grid, heads, D):
    """Large rows take the 128-wide block kernel (ragged N in the second case)."""
    T, H, W = grid
    plan = bs.Plan(1, heads, D, T, H, W, rule="topk", k=8)
    N = plan.N
    g = torch.Generator(device="cpu").manual_seed(N)
    pq = torch.randn((1, heads, N, D), generator=g, dtype=torch.float32)
    pk = torch.randn((1, heads, N, D), generator=g, dtype=torch.float32)
    S = torch.empty((1, heads, N, N), dtype=torch.float32, device="cuda")
    bs.attn_block_scores(plan, pq.cuda(), pk.cuda(), S)
    scale = 1 / math.sqrt(D)
    ref = select.block_scores(pq.numpy(), pk.numpy(), scale)
    bound = 1e-5 * scale * np.matmul(np.abs(pq.numpy()).astype(np.float64),
                                     np.swapaxes(np.abs(pk.numpy()).astype(np.float64), -1, -2)) + 1e-30
    assert np.all(np.abs(to64(S) - ref) <= bound)


@pytest.mark.parametrize("N,k", [(32, 8), (364, 46), (1440, 144), (37, 37), (2048, 1),
                                 (100, 99), (5, 2), (1000, 500)])
def test_select_topk_bit_exact(bs, N, k):
    rows = 2 * 3 * N if N <= 400 else 2 * N
    S = random_scores(rows, N, seed=N * 7 + k)
    # A plan whose N matches: grid of N tiles along w (4 x 4 x 4N)
    plan = bs.Plan(1, rows // N, 64, 4, 4, 4 * N, rule="topk", k=k)
    assert plan.N == N
    idx = torch.empty((1, rows // N, N, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, rows // N, N), dtype=torch.int32, device="cuda")
    bs.attn_select_from_scores(plan, S.view(1, rows // N, N, N).cuda(), idx, cnt)
    got = lists_from_device(idx, cnt)
    Sn = S.numpy()
    for r in range(rows):
        np.testing.assert_array_equal(got[r], select.topk_row(Sn[r], k))


@pytest.mark.parametrize("N,k,p", [(32, 8, 0.9), (364, 16, 0.9), (1440, 16, 0.9), (50, 0, 0.5),
                                   (700, 3, 0.99), (2048, 16, 0.9), (17, 17, 0.3), (9, 1, 1.0),
                                   (128, 4, 0.9), (256, 0, 0.95), (364, 200, 0.5), (1440, 16, 1.0)])
@pytest.mark.parametrize("sharp", [1.0, 8.0])
def test_select_topp_bit_exact(bs, N, k, p, sharp):
    rows = 2 * N if N <= 400 else N
    S = random_scores(rows, N, seed=N * 13 + k) * sharp
    plan = bs.Plan(1, rows // N, 64, 4, 4, 4 * N, rule="topp", k=k, p=p)
    idx = torch.empty((1, rows // N, N, N), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, rows // N, N), dtype=torch.int32, device="cuda")
    bs.attn_select_from_scores(plan, S.view(1, rows // N, N, N).cuda(), idx, cnt)
    got = lists_from_device(idx, cnt)
    Sn = S.numpy()
    for r in range(rows):
        assert_topp_equal(got[r], Sn[r], p, k)


def _degenerate_rows(N, seed):
    """Rows that defeat value binning: ties, outliers, ulp clusters, denormals."""
    rng = np.random.default_rng(seed)
    base = rng.standard_normal(N).astype(np.float32)
    rows = [np.full(N, 0.5, np.float32),                                   # one value
            np.where(rng.random(N) < 0.5, 0.0, -0.0).astype(np.float32),   # +0 / -0
            np.where(rng.random(N) < 0.5, 1.0, 2.0).astype(np.float32),    # two values
            np.where(np.arange(N) == N // 3, 1e30, base).astype(np.float32),
            np.where(np.arange(N) == N // 2, -1e30, base).astype(np.float32),
            (base * 1e-42).astype(np.float32),                              # denormals
            1.0 + rng.integers(0, 40, N).astype(np.float32) * np.finfo(np.float32).eps,  # ulps
            np.where(rng.random(N) < 0.1, -np.inf, base).astype(np.float32),
            np.round(base, 1).astype(np.float32),                           # many ties
            np.where(np.arange(N) < N // 4, base.max(), base).astype(np.float32)]
    return np.stack([r.astype(np.float32) for r in rows])


@pytest.mark.parametrize("N", [37, 300, 1440, 2048])
@pytest.mark.parametrize("rule", ["topk", "topp"])
def test_select_degenerate_rows(bs, N, rule):
    S = _degenerate_rows(N, seed=N)
    rows = S.shape[0]
    k = max(1, N // 10)
    pad = np.tile(S, (N // rows + 1, 1))[:N]  # one head: N rows
    plan = bs.Plan(1, 1, 64, 4, 4, 4 * N, rule=rule, k=k, p=0.9)
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    bs.attn_select_from_scores(plan, torch.from_numpy(pad).view(1, 1, N, N).cuda(), idx, cnt)
    got = lists_from_device(idx, cnt)
    for r in range(N):
        if rule == "topk":
            np.testing.assert_array_equal(got[r], select.topk_row(pad[r], k))
        else:
            assert_topp_equal(got[r], pad[r], 0.9, k)


@pytest.mark.parametrize("name", ["ragged_window_fp8", "ragged_bf16_window", "tile248_window_fp8",
                                  "tile688_window_fp8"])
def test_window_lists(bs, name):
    wl = SMALL[name]
    plan = _plan(bs, wl)
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    bs.attn_select_from_scores(plan, None, idx, cnt)
    got = lists_from_device(idx, cnt)
    grid = tiling.tile_grid(wl.T, wl.H, wl.W, wl.tile)
    for r, l in enumerate(got):
        np.testing.assert_array_equal(l, select.window_row(r % plan.N, grid, wl.win))


@pytest.mark.parametrize("name", ["ragged_window_fp8", "ragged_d64_fp8", "tiny_d64", "tile688_window_fp8",
                                  "tile11x128_d64"])
def test_quantize_e4m3_bytes(bs, name):
    wl = SMALL[name]
    plan = _plan(bs, wl)
    q, _, _ = make_qkv(wl, "cuda")
    q = q * 37.0  # exercise larger magnitudes too
    q = q.to(torch.bfloat16)
    xt = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
    bs.attn_reorder(plan, q, xt)
    codes = torch.empty(plan.tiled_shape(), dtype=torch.uint8, device="cuda")
    scales = torch.empty((wl.B, wl.heads, plan.N), dtype=torch.float32, device="cuda")
    bs.attn_quantize_e4m3(plan, xt, codes, scales)
    rc, rs = e4m3.quantize_tiled(tiling.reorder(to64(q).astype(np.float32), wl.T, wl.H, wl.W, wl.tile))
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)


def _bf16(x):
    return (np.array([x], np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32)[0]


def _bf16_step(x, n):
    """The bf16 value n representable steps above (n > 0) or below x > 0."""
    return (np.array([x], np.float32).view(np.uint32) + np.uint32(n << 16) if n > 0 else
            np.array([x], np.float32).view(np.uint32) - np.uint32((-n) << 16)).view(np.float32)[0]


# Tile amax values away from the common range: the exact-division fallback of
# the quantiser (scale below 2^-92, or infinite) and the values next to that
# bound, the bf16 extremes, and ordinary ones; 24 tiles.
_GUARD = np.float32(448.0) * np.float32(2.0) ** -92  # scale exactly 2^-92
_BF16_MAX = np.array([0x7F7F0000], np.uint32).view(np.float32)[0]
_EDGE_AMAX = [_GUARD, _bf16_step(_GUARD, -1), _bf16_step(_GUARD, 1), _bf16_step(_GUARD, -2),
              np.float32(2.0) ** -100, _bf16(1e-30), _bf16(1e-35), _bf16(1.2e-38), _bf16(9.2e-41),
              _BF16_MAX, _bf16(1e38), np.float32(2.0) ** 100, np.float32(1.0), np.float32(448.0),
              np.float32(0.5), _bf16(3e-20), _bf16(7e15), np.float32(np.inf), np.float32(np.inf), _bf16(5e-3),
              _bf16(123.0), _bf16(2e-27), _bf16(6e-26), _bf16(1e-24)]


@pytest.mark.parametrize("amax_set", ["random", "edges"])
def test_quantize_e4m3_every_bf16_magnitude(bs, amax_set):
    """Tiles holding every bf16 magnitude of the 32 binades up to the tile's
    amax (both signs, +0 and -0 filling the 64 x 128 tile), under 24 amax
    values (random ones between 5e-5 and 2e4, or the edge set above, where a
    tile with an infinite amax holds +inf and -inf): e4m3 codes byte-identical
    to the oracle's fp32-division quantisation. Many of these quotients fall
    exactly on, or next to, e4m3 rounding midpoints (bf16 ratios have short
    binary expansions), and the smallest ones in the e4m3 subnormal range and
    below it."""
    T, H, W = 4, 4, 4 * 12  # 12 tiles of 64 tokens
    heads = 2
    plan = bs.Plan(1, heads, 128, T, H, W, rule="window", win=(0, 0, 1), qk_fp8=True)
    rng = np.random.default_rng(5)
    tiles = np.zeros((1, heads, plan.N, 64, 128), dtype=np.float32)
    for h in range(heads):
        for t in range(plan.N):
            if amax_set == "random":
                amax = _bf16(np.float32(rng.uniform(0.5, 2.0) * 10.0 ** rng.uniform(-4, 4)))
            else:
                amax = _EDGE_AMAX[h * plan.N + t]
            top = amax if np.isfinite(amax) else _BF16_MAX
            e = int(np.frexp(top)[1]) - 1
            # binade bases as bf16 (those below the smallest bf16 subnormal are 0)
            base = (np.float32(2.0) ** np.arange(e - 31, e + 1, dtype=np.float32)).view(np.uint32) & 0xFFFF0000
            mags = (base[:, None] + (np.arange(128, dtype=np.uint32) << 16)[None, :]).reshape(-1).view(np.float32)
            mags = np.unique(mags[mags < amax])
            vals = np.concatenate([[amax, -amax], mags, -mags])[:8192].astype(np.float32)
            flat = np.zeros(8192, np.float32)
            flat[:vals.size] = vals
            flat[vals.size::2] = -0.0
            tiles[0, h, t] = rng.permutation(flat).reshape(64, 128)
    xt = torch.from_numpy(tiles).to(torch.bfloat16).cuda()
    assert torch.equal(xt.float().cpu(), torch.from_numpy(tiles))  # every value is a bf16 value
    codes = torch.empty(plan.tiled_shape(), dtype=torch.uint8, device="cuda")
    scales = torch.empty((1, heads, plan.N), dtype=torch.float32, device="cuda")
    bs.attn_quantize_e4m3(plan, xt, codes, scales)
    with np.errstate(invalid="ignore"):  # inf / inf in the tiles with an infinite amax: NaN, code 0x7F
        rc, rs = e4m3.quantize_tiled(tiles)
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    # attn_layer quantises while it reorders (natural source): its output is
    # bit-identical to attn_forward on the codes above.
    x_nat = torch.from_numpy(tiling.unreorder(tiles, T, H, W, (4, 4, 4))).to(torch.bfloat16).cuda()
    v_nat = torch.randn(x_nat.shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    bs.attn_select_from_scores(plan, None, idx, cnt)
    o_layer = torch.empty_like(x_nat)
    bs.attn_layer(plan, x_nat, x_nat, v_nat, o_layer, plan.workspace("layer"))
    vt = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
    bs.attn_reorder(plan, v_nat, vt)
    ot = torch.empty_like(vt)
    bs.attn_forward(plan, codes, codes, vt, idx, cnt, ot, q_scale=scales, k_scale=scales)
    o_chain = torch.empty_like(x_nat)
    bs.attn_unreorder(plan, ot, o_chain)
    assert bs.attn_check_device_status(plan) == 0
    assert torch.equal(o_layer.view(torch.int16), o_chain.view(torch.int16))  # bitwise: NaN rows included


def _oracle_inputs(wl):
    q, k, v = make_qkv(wl, "cpu")
    return q, k, v, to64(q), to64(k), to64(v)


@pytest.mark.parametrize("name", ["tiny_d64", "ragged_topk", "ragged_topp", "ragged_bf16_window",
                                  "tile688_topk", "tile488_topp", "tile11x128_d64"])
def test_forward_bf16_against_oracle(bs, name):
    wl = SMALL[name]
    plan = _plan(bs, wl, qk_fp8=False)
    q, k, v, qn, kn, vn = _oracle_inputs(wl)
    _, _, _, lists = attention.route(qn, kn, wl.T, wl.H, wl.W, wl.rule, tile=wl.tile, k=wl.k, p=wl.p,
                                     half=wl.win, score_dtype=np.float32)
    idx, cnt = lists_to_device(lists, plan.kmax)
    tiled = []
    for x in (q, k, v):
        t = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
        bs.attn_reorder(plan, x.cuda(), t)
        tiled.append(t)
    o = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    si, sc = plan.list_shapes()
    bs.attn_forward(plan, tiled[0], tiled[1], tiled[2], idx.view(si), cnt.view(sc), o, lse)
    assert bs.attn_check_device_status(plan) == 0
    o_ref, lse_ref = attention.attention_full(qn, kn, vn, lists, wl.T, wl.H, wl.W, wl.tile)
    o_nat = tiling.unreorder(to64(o), wl.T, wl.H, wl.W, wl.tile)
    err = np.abs(o_nat - o_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    lse_nat = np.stack([tiling.unreorder(to64(lse)[:, h:h + 1, :, :, None], wl.T, wl.H, wl.W, wl.tile)[..., 0, 0]
                        for h in range(wl.heads)], axis=1)
    np.testing.assert_allclose(lse_nat, lse_ref, rtol=0, atol=2e-2)


@pytest.mark.parametrize("name", ["ragged_window_fp8", "ragged_d64_fp8", "tile248_window_fp8",
                                  "tile688_window_fp8"])
def test_forward_fp8_against_oracle(bs, name):
    wl = SMALL[name]
    plan = _plan(bs, wl)
    q, k, v, qn, kn, vn = _oracle_inputs(wl)
    qd, kd, (qc, qs), (kc, ks) = attention.fp8_qk(qn, kn, wl.T, wl.H, wl.W, wl.tile)
    _, _, _, lists = attention.route(qn, kn, wl.T, wl.H, wl.W, wl.rule, tile=wl.tile, k=wl.k, p=wl.p,
                                     half=wl.win, score_dtype=np.float32)
    idx, cnt = lists_to_device(lists, plan.kmax)
    vt = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
    bs.attn_reorder(plan, v.cuda(), vt)
    o = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
    si, sc = plan.list_shapes()
    bs.attn_forward(plan, torch.from_numpy(qc).cuda(), torch.from_numpy(kc).cuda(), vt,
                    idx.view(si), cnt.view(sc), o, q_scale=torch.from_numpy(qs).cuda(),
                    k_scale=torch.from_numpy(ks).cuda())
    assert bs.attn_check_device_status(plan) == 0
    o_ref, _ = attention.attention_full(qd, kd, vn, lists, wl.T, wl.H, wl.W, wl.tile)
    o_nat = tiling.unreorder(to64(o), wl.T, wl.H, wl.W, wl.tile)
    rel = np.linalg.norm(o_nat - o_ref) / np.linalg.norm(o_ref)
    assert rel <= 1e-2, rel


def test_bad_list_entry_sets_error_word_and_is_skipped(bs):
    wl = SMALL["ragged_topk"]
    plan = _plan(bs, wl)
    q, k, v = make_qkv(wl, "cuda")
    tiled = []
    for x in (q, k, v):
        t = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
        bs.attn_reorder(plan, x, t)
        tiled.append(t)
    si, sc = plan.list_shapes()
    idx = torch.zeros(si, dtype=torch.int32, device="cuda")
    idx[..., 1] = plan.N + 3          # out of range: must be skipped, not read
    idx[0, 0, 0, 2] = -7
    cnt = torch.full(sc, 3, dtype=torch.int32, device="cuda")
    o = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
    bs.attn_forward(plan, *tiled, idx, cnt, o)
    assert bs.attn_check_device_status(plan) == bs.BsattnError(5, "").code
    assert bs.attn_check_device_status(plan) == 0  # cleared
    # result equals attending tile 0 only (listed twice counts as two passes of the same keys)
    idx2 = torch.zeros(si, dtype=torch.int32, device="cuda")
    cnt2 = torch.ones(sc, dtype=torch.int32, device="cuda")
    o2 = torch.empty_like(o)
    bs.attn_forward(plan, *tiled, idx2, cnt2, o2)
    rows = (idx[..., 2] == 0)
    torch.testing.assert_close(o[rows], o2[rows], rtol=2e-2, atol=2e-2)
    cnt_bad = torch.full(sc, plan.kmax + 1, dtype=torch.int32, device="cuda")
    bs.attn_forward(plan, *tiled, idx2, cnt_bad, o2)
    assert bs.attn_check_device_status(plan) == 5


@pytest.mark.parametrize("name", ["tiny_d64", "ragged_topk", "ragged_topp", "ragged_bf16_window",
                                  "ragged_window_fp8", "ragged_d64_fp8", "tile248_window_fp8",
                                  "tile688_topk", "tile488_topp", "tile688_window_fp8",
                                  "tile11x128_d64"])
def test_forward_natural_equals_tiled_path(bs, name):
    """Natural-layout attention (tile reorder folded into its loads) gives
    bit-identical O and lse to reorder -> attn_forward -> unreorder."""
    wl = SMALL[name]
    plan = _plan(bs, wl)
    q, k, v = make_qkv(wl, "cuda")
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    ws = plan.workspace("select")
    bs.attn_select(plan, q, k, idx, cnt, ws)
    ts = plan.tiled_shape()
    vt = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    bs.attn_reorder(plan, v, vt)
    qs = ks = None
    if plan.qk_fp8:
        qa, ka = (torch.empty(ts, dtype=torch.uint8, device="cuda") for _ in range(2))
        qs, ks = (torch.empty((wl.B, wl.heads, plan.N), dtype=torch.float32, device="cuda") for _ in range(2))
        for x, codes, scales in ((q, qa, qs), (k, ka, ks)):
            xt = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
            bs.attn_reorder(plan, x, xt)
            bs.attn_quantize_e4m3(plan, xt, codes, scales)
        qn, kn = qa, ka
    else:
        qa, ka = (torch.empty(ts, dtype=torch.bfloat16, device="cuda") for _ in range(2))
        bs.attn_reorder(plan, q, qa)
        bs.attn_reorder(plan, k, ka)
        qn, kn = q, k
    ot = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    lse_t = torch.empty((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    bs.attn_forward(plan, qa, ka, vt, idx, cnt, ot, lse_t, q_scale=qs, k_scale=ks)
    o_ref = torch.empty_like(q)
    bs.attn_unreorder(plan, ot, o_ref)
    o_nat = torch.full_like(q, float("nan"))
    lse_nat = torch.full((wl.B, wl.heads, plan.L), float("nan"), dtype=torch.float32, device="cuda")
    bs.attn_forward_natural(plan, qn, kn, v, idx, cnt, o_nat, lse_nat, q_scale=qs, k_scale=ks)
    assert bs.attn_check_device_status(plan) == 0
    assert torch.equal(o_nat, o_ref)
    lse_ref = tiling_lse_natural(lse_t, wl, plan)
    assert torch.equal(lse_nat.cpu(), lse_ref)


@pytest.mark.parametrize("name", ["ragged_window_fp8", "ragged_d64_fp8", "tile248_window_fp8",
                                  "tile688_window_fp8"])
def test_layer_e4m3_equals_quantize_chain(bs, name):
    """attn_layer quantises Q and K in one launch straight from the natural
    layout (tiles of one chunk and of several); its output is bit-identical
    to reorder -> attn_quantize_e4m3 -> attn_forward -> unreorder on the same
    kept lists."""
    wl = SMALL[name]
    plan = _plan(bs, wl)
    assert plan.qk_fp8
    q, k, v = make_qkv(wl, "cuda")
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    o_layer = torch.full_like(q, float("nan"))
    bs.attn_layer(plan, q, k, v, o_layer, plan.workspace("layer"), idx=idx, cnt=cnt)
    ts = plan.tiled_shape()
    tiled = []
    for x in (q, k, v):
        t = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
        bs.attn_reorder(plan, x, t)
        tiled.append(t)
    codes = [torch.empty(ts, dtype=torch.uint8, device="cuda") for _ in range(2)]
    scales = [torch.empty((wl.B, wl.heads, plan.N), dtype=torch.float32, device="cuda") for _ in range(2)]
    for t, c, s_ in zip(tiled[:2], codes, scales):
        bs.attn_quantize_e4m3(plan, t, c, s_)
    ot = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    bs.attn_forward(plan, codes[0], codes[1], tiled[2], idx, cnt, ot, q_scale=scales[0], k_scale=scales[1])
    o_chain = torch.empty_like(q)
    bs.attn_unreorder(plan, ot, o_chain)
    assert bs.attn_check_device_status(plan) == 0
    assert torch.equal(o_layer.view(torch.int16), o_chain.view(torch.int16))


def tiling_lse_natural(lse_t, wl, plan):
    """Tiled lse [B, Hh, N, V] -> natural [B, Hh, L] (oracle's tile order)."""
    x = to64(lse_t)
    out = np.stack([tiling.unreorder(x[:, h:h + 1, :, :, None], wl.T, wl.H, wl.W, wl.tile)[..., 0, 0]
                    for h in range(wl.heads)], axis=1)
    return torch.from_numpy(out.astype(np.float32))


def _forward_vs_oracle(bs, wl, lists, tile=(4, 4, 4)):
    """attn_forward on given lists (bf16) against the oracle; returns (O, lse) natural."""
    plan = _plan(bs, wl, qk_fp8=False)
    q, k, v, qn, kn, vn = _oracle_inputs(wl)
    idx, cnt = lists_to_device(lists, plan.kmax)
    tiled = []
    for x in (q, k, v):
        t = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
        bs.attn_reorder(plan, x.cuda(), t)
        tiled.append(t)
    o = torch.empty(plan.tiled_shape(), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    si, sc = plan.list_shapes()
    bs.attn_forward(plan, tiled[0], tiled[1], tiled[2], idx.view(si), cnt.view(sc), o, lse)
    assert bs.attn_check_device_status(plan) == 0
    o_ref, lse_ref = attention.attention_full(qn, kn, vn, lists, wl.T, wl.H, wl.W, wl.tile)
    o_nat = tiling.unreorder(to64(o), wl.T, wl.H, wl.W, wl.tile)
    err = np.abs(o_nat - o_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    lse_nat = tiling_lse_natural(lse, wl, plan).numpy().astype(np.float64)
    finite = np.isfinite(lse_ref)
    np.testing.assert_array_equal(np.isfinite(lse_nat), finite)
    np.testing.assert_allclose(lse_nat[finite], lse_ref[finite], rtol=0, atol=2e-2)
    return o_nat, lse_nat, o_ref


def test_forward_single_tile_grid(bs):
    """A grid smaller than one tile: N = 1, most slots padding."""
    from block_sparse_attention_reorder_b200.datagen import Workload
    wl = Workload("one_tile", 1, 2, 128, 3, 2, 3, "topk", k=1, recipe="iid", seed=21)
    _forward_vs_oracle(bs, wl, [np.array([0])] * 2)


def test_forward_all_tiles_kept_is_dense_attention(bs):
    """k = N: every tile keeps every tile, which is dense attention over the
    real tokens (checked by the oracle against torch SDPA in fp64)."""
    from block_sparse_attention_reorder_b200.datagen import Workload
    wl = Workload("dense", 1, 2, 64, 7, 6, 9, "topk", k=12, recipe="iid", seed=22)
    plan = _plan(bs, wl)
    assert plan.N == 12
    _forward_vs_oracle(bs, wl, [np.arange(12)] * (2 * 12))


def test_forward_empty_lists_give_zero_rows(bs):
    """Query tiles with an empty kept list: O rows are zero and lse is -inf,
    as in the plain definition (a softmax over no keys contributes nothing);
    the other tiles are unaffected."""
    from block_sparse_attention_reorder_b200.datagen import Workload
    wl = Workload("empty_rows", 1, 2, 128, 7, 10, 13, "topk", k=3, recipe="iid", seed=23)
    plan = _plan(bs, wl)
    rng = np.random.default_rng(5)
    lists = []
    for r in range(2 * plan.N):
        lists.append(np.array([], dtype=np.int64) if r % 3 == 0 else
                     np.sort(rng.choice(plan.N, size=3, replace=False)))
    o_nat, lse_nat, o_ref = _forward_vs_oracle(bs, wl, lists)
    tid, _ = tiling.token_tile_and_row(wl.T, wl.H, wl.W)
    for h in range(2):
        empty = [i for i in range(plan.N) if (h * plan.N + i) % 3 == 0]
        tok = np.isin(tid, empty)
        assert np.all(o_nat[0, tok, h] == 0)
        assert np.all(np.isneginf(lse_nat[0, h, tok]))


def test_layer_tile_24x32x32_sampled_tokens(bs):
    """The largest tile of the FPSAttention tile ablation, (24, 32, 32):
    24,576 tokens (384 chunks of 64) per tile. A grid of two such tiles (the
    second mostly padding), top-k 1, through attn_layer; the kept lists equal
    the oracle's, and sampled query tokens of both tiles match the oracle's
    dense masked attention over every key of their kept tile."""
    from block_sparse_attention_reorder_b200.datagen import Workload
    wl = Workload("tile24x32x32", 1, 2, 64, 24, 32, 40, "topk", k=1, seed=24, tile=(24, 32, 32))
    plan = _plan(bs, wl)
    assert plan.N == 2 and plan.V == 24 * 32 * 32
    q, k, v = make_qkv(wl, "cuda")
    o = torch.empty_like(q)
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    bs.attn_layer(plan, q, k, v, o, plan.workspace("layer"), idx=idx, cnt=cnt)
    assert bs.attn_check_device_status(plan) == 0
    qn, kn, vn = to64(q), to64(k), to64(v)
    _, _, S, lists = attention.route(qn, kn, wl.T, wl.H, wl.W, "topk", k=1, tile=wl.tile)
    got = lists_from_device(idx, cnt)
    Sf = S.reshape(-1, plan.N)
    for r, (a, b) in enumerate(zip(got, lists)):
        if not np.array_equal(a, b):  # fp32 against fp64 scores at a near-tie
            assert_valid_selection(a, Sf[r], "topk", k=1)
    tid, _ = tiling.token_tile_and_row(wl.T, wl.H, wl.W, wl.tile)
    rng = np.random.default_rng(4)
    on = to64(o)
    scale = 1.0 / np.sqrt(wl.head_dim)
    for h in range(wl.heads):
        for i in range(plan.N):
            members = np.nonzero(tid == i)[0]
            toks = rng.choice(members, size=48, replace=False)
            keys = np.concatenate([np.nonzero(tid == j)[0] for j in got[h * plan.N + i]])
            allowed = np.ones((toks.size, keys.size), dtype=bool)
            ref, _ = attention.dense_masked(qn[0, toks, h], kn[0, keys, h], vn[0, keys, h], allowed, scale)
            err = np.abs(on[0, toks, h] - ref)
            assert err.max() <= 2e-2 and err.mean() <= 2e-3, (h, i, err.max(), err.mean())
