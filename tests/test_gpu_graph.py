"""A layer step and the backward inside captured CUDA graphs.

Every per-call entry point only enqueues work on the caller's stream: it
allocates nothing, copies nothing to the host and does not synchronise (those
happen only at plan creation, plan destruction and the device-status check).
So a whole step can be captured once and replayed; replays on new inputs,
copied into the captured buffers, give the same bytes as direct calls.
"""
import dataclasses

import pytest
import torch

from block_sparse_attention_reorder_b200.datagen import make_qkv
from tests.helpers import SMALL, lists_from_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bs():
    from block_sparse_attention_reorder_b200 import bsattn
    assert torch.cuda.is_available()
    return bsattn


def _lists_equal(a_idx, a_cnt, b_idx, b_cnt):
    a, b = lists_from_device(a_idx, a_cnt), lists_from_device(b_idx, b_cnt)
    return len(a) == len(b) and all(bool((x == y).all()) and len(x) == len(y) for x, y in zip(a, b))


@pytest.mark.parametrize("name", ["ragged_topk", "ragged_topp", "ragged_window_fp8", "tile688_topk",
                                  "tiny_d64"])
def test_layer_graph_replay(bs, name):
    wl = SMALL[name]
    plan = bs.Plan.for_workload(wl)
    si, sc = plan.list_shapes()
    inputs = [make_qkv(dataclasses.replace(wl, seed=wl.seed + s), "cuda") for s in range(3)]
    sq, sk, sv = (torch.empty_like(x) for x in inputs[0])
    so = torch.empty_like(sq)
    slse = torch.empty((wl.B, wl.heads, wl.L), dtype=torch.float32, device="cuda")
    sidx = torch.empty(si, dtype=torch.int32, device="cuda")
    scnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    ws = plan.workspace("layer")

    def step():
        bs.attn_layer(plan, sq, sk, sv, so, ws, lse_nat=slse, idx=sidx, cnt=scnt)

    for x, y in zip((sq, sk, sv), inputs[0]):
        x.copy_(y)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture (kernel attributes, lazy loading)
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    ws_ref = plan.workspace("layer")
    for q, k, v in inputs:
        for x, y in zip((sq, sk, sv), (q, k, v)):
            x.copy_(y)
        so.fill_(float("nan"))
        graph.replay()
        o = torch.empty_like(q)
        lse = torch.empty_like(slse)
        idx, cnt = torch.empty_like(sidx), torch.empty_like(scnt)
        bs.attn_layer(plan, q, k, v, o, ws_ref, lse_nat=lse, idx=idx, cnt=cnt)
        torch.cuda.synchronize()
        assert bs.attn_check_device_status(plan) == 0
        assert torch.equal(so, o)
        assert torch.equal(slse, lse)
        assert _lists_equal(sidx, scnt, idx, cnt)
    del graph


@pytest.mark.parametrize("name", ["ragged_topk", "tile688_topk"])
def test_backward_graph_replay(bs, name):
    wl = SMALL[name]
    plan = bs.Plan.for_workload(wl)
    ts = plan.tiled_shape()
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    q, k, _ = make_qkv(wl, "cuda")
    bs.attn_select(plan, q, k, idx, cnt, plan.workspace("select"))
    bufs = {n: torch.empty(ts, dtype=torch.bfloat16, device="cuda") for n in ("q", "k", "v", "o", "do")}
    lse = torch.empty((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    grads = {n: torch.empty(ts, dtype=torch.bfloat16, device="cuda") for n in ("dq", "dk", "dv")}
    ws = plan.workspace("backward")

    def step():
        bs.attn_forward(plan, bufs["q"], bufs["k"], bufs["v"], idx, cnt, bufs["o"], lse)
        bs.attn_backward(plan, bufs["q"], bufs["k"], bufs["v"], bufs["o"], bufs["do"], lse, idx, cnt,
                         grads["dq"], grads["dk"], grads["dv"], ws)

    def load(seed):
        g = torch.Generator(device="cpu").manual_seed(seed)
        for n in ("q", "k", "v", "do"):
            bufs[n].copy_(torch.randn(ts, generator=g).to(torch.bfloat16))

    load(0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    for seed in (1, 2):
        load(seed)
        for t in grads.values():
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        got = {n: t.clone() for n, t in grads.items()}
        step()  # the same calls, not captured
        torch.cuda.synchronize()
        assert bs.attn_check_device_status(plan) == 0
        for n in grads:
            assert torch.equal(got[n], grads[n]), n
    del graph
