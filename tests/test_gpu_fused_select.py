"""Fused block scores + top-k (attn_select_fused) against the unfused path:
the score matrix it does not write is bit-identical when requested as debug
output, and the kept lists equal attn_select's, including rows the fused
kernel hands to the row-wise selection (runs of equal scores, constant rows).
The unfused path is itself pinned against the oracle (block scores within the
fp32 bound, selection bit-exact on the GPU's scores), so equality carries
that parity over."""
import numpy as np
import pytest
import torch

from block_sparse_attention_reorder_b200.datagen import WORKLOADS, Workload, make_qkv
from tests.helpers import SMALL, lists_from_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bs():
    from block_sparse_attention_reorder_b200 import bsattn
    assert torch.cuda.is_available()
    return bsattn


def _workload(name):
    return SMALL[name] if name in SMALL else WORKLOADS[name]


def _lists(plan):
    si, sc = plan.list_shapes()
    return (torch.full(si, -7, dtype=torch.int32, device="cuda"),
            torch.full(sc, -7, dtype=torch.int32, device="cuda"))


def _select_both(bs, plan, q, k, debug=False, repeat=1):
    ws = plan.workspace("select")
    a = _lists(plan)
    bs.attn_select(plan, q, k, *a, ws)
    sdbg = None
    if debug:
        sdbg = torch.full((plan.B, plan.heads, plan.N, plan.N), float("nan"), dtype=torch.float32,
                          device="cuda")
    for _ in range(repeat):
        b = _lists(plan)
        bs.attn_select_fused(plan, q, k, *b, ws, scores_debug=sdbg)
    assert bs.attn_check_device_status(plan) == 0
    return a, b, sdbg


def _assert_same_lists(a, b):
    assert torch.equal(a[1], b[1]), "kept counts differ"
    for x, y in zip(lists_from_device(*a), lists_from_device(*b)):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("name", ["tiny_d64", "ragged_topk", "ragged_d64_fp8", "tile688_topk", "wan1.3b",
                                  "wan14b"])
def test_fused_lists_equal_unfused(bs, name):
    wl = _workload(name)
    plan = bs.Plan.for_workload(wl)
    q, k, _ = make_qkv(wl, "cuda")
    a, b, _ = _select_both(bs, plan, q, k)
    _assert_same_lists(a, b)


@pytest.mark.parametrize("name", ["tiny_d64", "ragged_topk", "wan1.3b"])
def test_fused_debug_scores_equal_block_scores(bs, name):
    wl = _workload(name)
    plan = bs.Plan.for_workload(wl)
    q, k, _ = make_qkv(wl, "cuda")
    _, _, sdbg = _select_both(bs, plan, q, k, debug=True)
    pq = torch.empty((wl.B, wl.heads, plan.N, wl.head_dim), dtype=torch.float32, device="cuda")
    pk = torch.empty_like(pq)
    bs.attn_pool(plan, q, pq)
    bs.attn_pool(plan, k, pk)
    S = torch.empty((wl.B, wl.heads, plan.N, plan.N), dtype=torch.float32, device="cuda")
    bs.attn_block_scores(plan, pq, pk, S)
    assert bs.attn_check_device_status(plan) == 0
    assert torch.equal(sdbg.view(torch.int32), S.view(torch.int32))


def test_fused_rows_settled_by_the_fallback(bs):
    """128 key tiles per row, k = 40. Head 0: every key tile pools to the same
    vector, so every row is constant and goes to the row-wise selection (ties
    broken by index). Head 1: the keys of the later frames repeat the earlier
    ones, so every row has pairs of equal scores that the fused ranking must
    order by index. Head 2: the key tiles of the first four frames are zero,
    so 64 scores of each row are exactly zero and, with about half of the
    others positive, the 40th largest falls among them: a boundary bin of 64
    tiles, which the fused kernel hands to the row-wise selection. Called
    twice: the list of rows to settle starts empty on every call."""
    wl = Workload("fused_ties", 1, 3, 64, 8, 32, 32, "topk", k=40, recipe="iid", seed=5)
    plan = bs.Plan.for_workload(wl)
    assert plan.N == 128
    q, k, _ = make_qkv(wl, "cuda")
    kk = k.view(wl.B, wl.T, wl.H, wl.W, wl.heads, wl.head_dim).clone()
    kk[..., 0, :] = kk[:, :1, :1, :1, 0, :]
    kk[:, wl.T // 2:, :, :, 1, :] = kk[:, :wl.T // 2, :, :, 1, :]
    kk[:, :wl.T // 2, :, :, 2, :] = 0
    k2 = kk.view_as(k).contiguous()
    a, b, _ = _select_both(bs, plan, q, k2, repeat=2)
    _assert_same_lists(a, b)
    # Constant rows keep the k lowest tile indices.
    assert torch.equal(b[0][0, 0, :, :wl.k].cpu(), torch.arange(wl.k, dtype=torch.int32).expand(plan.N, wl.k))


def test_fused_window_equals_select_and_topp_is_unsupported(bs):
    wl = SMALL["ragged_bf16_window"]
    plan = bs.Plan.for_workload(wl)
    q, k, _ = make_qkv(wl, "cuda")
    a, b, _ = _select_both(bs, plan, q, k)
    _assert_same_lists(a, b)
    wl = SMALL["ragged_topp"]
    plan = bs.Plan.for_workload(wl)
    q, k, _ = make_qkv(wl, "cuda")
    with pytest.raises(bs.BsattnError) as e:
        bs.attn_select_fused(plan, q, k, *_lists(plan), plan.workspace("select"))
    assert e.value.code == 2
