"""Backward parity: attn_backward (tiled) against the oracle's gradients of
the plain masked-softmax definition, on small ragged grids."""
import numpy as np
import pytest
import torch

from block_sparse_attention_reorder_b200.datagen import make_qkv
from oracle import attention, tiling
from tests.helpers import SMALL, lists_to_device, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bs():
    from block_sparse_attention_reorder_b200 import bsattn
    assert torch.cuda.is_available()
    return bsattn


def _grad_close(got, ref, name):
    err = got - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= 1e-2, (name, rel)
    assert np.abs(err).max() <= 3e-2 * np.abs(ref).max(), (name, np.abs(err).max(), np.abs(ref).max())


@pytest.mark.parametrize("name", ["tiny_d64", "ragged_topk", "ragged_topp", "ragged_bf16_window",
                                  "tile688_topk", "tile488_topp", "tile11x128_d64"])
def test_backward_against_oracle(bs, name):
    wl = SMALL[name]
    plan = bs.Plan.for_workload(wl)
    q, k, v = make_qkv(wl, "cpu")
    g = torch.Generator(device="cpu").manual_seed(100 + wl.seed)
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
    rq, rk, rv = attention.attention_backward_full(qn, kn, vn, don, lists, wl.T, wl.H, wl.W, wl.tile)
    for name_, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        nat = tiling.unreorder(to64(got), wl.T, wl.H, wl.W, wl.tile)
        _grad_close(nat, ref, name_)
    # Padded slots carry zero gradients.
    valid = torch.from_numpy(tiling.tile_valid_rows(wl.T, wl.H, wl.W, wl.tile)).cuda()
    for t in (dq, dk, dv):
        assert torch.all(t[:, :, ~valid] == 0)


def test_backward_rejects_unsupported_plans(bs):
    wl = SMALL["ragged_window_fp8"]
    plan = bs.Plan.for_workload(wl)  # e4m3 Q/K
    ts = plan.tiled_shape()
    x = torch.zeros(ts, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    si, sc = plan.list_shapes()
    idx = torch.zeros(si, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(sc, dtype=torch.int32, device="cuda")
    with pytest.raises(bs.BsattnError) as e:
        bs.attn_backward(plan, x, x, x, x, x, lse, idx, cnt, x, x, x, plan.workspace("backward"))
    assert e.value.code == 2


@pytest.mark.parametrize("name", ["wan1.3b", "wan14b"])
def test_backward_full_size_sampled(bs, name):
    """Full-size layers: dQ of sampled query tiles and dK, dV of sampled key
    tiles (edge tiles included) against the oracle computed tile by tile."""
    from block_sparse_attention_reorder_b200.datagen import WORKLOADS
    wl = WORKLOADS[name]
    plan = bs.Plan.for_workload(wl)
    q, k, v = make_qkv(wl, "cuda")
    g = torch.Generator(device="cuda").manual_seed(200)
    d_o = torch.randn(q.shape, generator=g, device="cuda").to(torch.bfloat16)
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    bs.attn_select(plan, q, k, idx, cnt, plan.workspace("select"))
    ts = plan.tiled_shape()
    t = [torch.empty(ts, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    for x, y in zip((q, k, v, d_o), t):
        bs.attn_reorder(plan, x, y)
    ot = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    bs.attn_forward(plan, t[0], t[1], t[2], idx, cnt, ot, lse)
    grads = [torch.empty(ts, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    bs.attn_backward(plan, t[0], t[1], t[2], ot, t[3], lse, idx, cnt, *grads, plan.workspace("backward"))
    assert bs.attn_check_device_status(plan) == 0
    h = 3
    nat = []
    for gt in grads:
        back = torch.empty_like(q)
        bs.attn_unreorder(plan, gt, back)
        nat.append(to64(back[:, :, h:h + 1]))
    del grads, t
    idx_h = idx[0, h].cpu().numpy()
    cnt_h = cnt[0, h].cpu().numpy()
    qn, kn, vn, don = (to64(x[:, :, h:h + 1]) for x in (q, k, v, d_o))
    lists_h = [idx_h[i, :cnt_h[i]].astype(np.int64) for i in range(plan.N)]
    qt_s, kt_s = [0, plan.N // 3, plan.N - 1], [1, plan.N // 2, plan.N - 1]
    dq_t, dkv_t = attention.attention_backward_tiles(qn, kn, vn, don, lists_h, wl.T, wl.H, wl.W, wl.tile,
                                                     h=0, qtiles=qt_s, ktiles=kt_s)
    got_q = np.concatenate([nat[0][0, tok, 0] for tok, _ in dq_t.values()])
    ref_q = np.concatenate([gq for _, gq in dq_t.values()])
    _grad_close(got_q, ref_q, "dq")
    got_k = np.concatenate([nat[1][0, tok, 0] for tok, _, _ in dkv_t.values()])
    ref_k = np.concatenate([gk for _, gk, _ in dkv_t.values()])
    _grad_close(got_k, ref_k, "dk")
    got_v = np.concatenate([nat[2][0, tok, 0] for tok, _, _ in dkv_t.values()])
    ref_v = np.concatenate([gv for _, _, gv in dkv_t.values()])
    _grad_close(got_v, ref_v, "dv")


def _backward_vs_oracle(bs, wl, lists):
    plan = bs.Plan.for_workload(wl)
    q, k, v = make_qkv(wl, "cpu")
    g = torch.Generator(device="cpu").manual_seed(300 + wl.seed)
    d_o = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qn, kn, vn, don = (to64(x) for x in (q, k, v, d_o))
    idx, cnt = lists_to_device(lists, plan.kmax)
    si, sc = plan.list_shapes()
    idx, cnt = idx.view(si), cnt.view(sc)
    ts = plan.tiled_shape()
    t = []
    for x in (q, k, v, d_o):
        y = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
        bs.attn_reorder(plan, x.cuda(), y)
        t.append(y)
    ot = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    bs.attn_forward(plan, t[0], t[1], t[2], idx, cnt, ot, lse)
    grads = [torch.full(ts, float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    bs.attn_backward(plan, t[0], t[1], t[2], ot, t[3], lse, idx, cnt, *grads, plan.workspace("backward"))
    assert bs.attn_check_device_status(plan) == 0
    ref = attention.attention_backward_full(qn, kn, vn, don, lists, wl.T, wl.H, wl.W, wl.tile)
    out = []
    for name_, got, r in zip(("dq", "dk", "dv"), grads, ref):
        nat = tiling.unreorder(to64(got), wl.T, wl.H, wl.W, wl.tile)
        if np.abs(r).max() > 0:
            _grad_close(nat, r, name_)
        else:
            assert np.all(nat == 0), name_
        out.append(nat)
    return plan, out


def test_backward_single_tile_grid(bs):
    from block_sparse_attention_reorder_b200.datagen import Workload
    wl = Workload("one_tile", 1, 2, 128, 3, 2, 3, "topk", k=1, recipe="iid", seed=21)
    _backward_vs_oracle(bs, wl, [np.array([0])] * 2)


def test_backward_empty_lists_and_all_kept(bs):
    """Query tiles that keep nothing get zero dQ and give nothing to dK, dV;
    a key tile nobody keeps gets zero dK, dV."""
    from block_sparse_attention_reorder_b200.datagen import Workload
    wl = Workload("empty_rows", 1, 2, 128, 7, 10, 13, "topk", k=3, recipe="iid", seed=23)
    plan = bs.Plan.for_workload(wl)
    rng = np.random.default_rng(6)
    lists = []
    for r in range(2 * plan.N):
        if r % 3 == 0:
            lists.append(np.array([], dtype=np.int64))
        else:
            choice = rng.choice(plan.N - 1, size=3, replace=False)  # key tile N-1 is never kept
            lists.append(np.sort(choice))
    _, (dq, dk, dv) = _backward_vs_oracle(bs, wl, lists)
    tid, _ = tiling.token_tile_and_row(wl.T, wl.H, wl.W)
    last = tid == plan.N - 1
    assert np.all(dk[0, last] == 0) and np.all(dv[0, last] == 0)
    for h in range(2):
        empty = [i for i in range(plan.N) if (h * plan.N + i) % 3 == 0]
        assert np.all(dq[0, np.isin(tid, empty), h] == 0)
