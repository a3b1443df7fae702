"""Failure detection without faulting the GPU.

- The device error word -> status mapping of attn_check_device_status, with
  the word written by a plain host-to-device copy (no kernel).
- A bounded wait that runs out: with the testing hook on, every CTA of the
  attention forward first waits on a barrier nothing arrives at, under a
  ~1 ms limit, and must take its timeout path (record TIMEOUT, let its own
  copies and MMAs finish, free tensor memory, return). The context stays
  usable: the next normal call is clean and bit-identical to a run made
  before the timeout.
- Argument errors on a real plan: misaligned pointers and short workspaces
  are rejected before anything is enqueued.
"""
import ctypes

import pytest
import torch

from block_sparse_attention_reorder_b200.datagen import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu

OK, INVALID_ARG, TIMEOUT, INTERNAL, WORKSPACE = 0, 1, 4, 5, 6


@pytest.fixture(scope="module")
def bs():
    from block_sparse_attention_reorder_b200 import bsattn
    return bsattn


@pytest.fixture(scope="module")
def tiny(bs):
    wl = WORKLOADS["tiny"]
    plan = bs.Plan.for_workload(wl)
    q, k, v = make_qkv(wl, "cuda")
    return wl, plan, q, k, v


@pytest.mark.parametrize("bits,status", [(0, OK), (1, INTERNAL), (2, TIMEOUT), (3, TIMEOUT)])
def test_error_word_maps_to_status_and_is_cleared(bs, tiny, bits, status):
    _, plan, *_ = tiny
    bs.attn_testing_set_error_word(plan, bits)
    assert bs.attn_check_device_status(plan) == status
    assert bs.attn_check_device_status(plan) == OK  # read and cleared


def _layer(bs, plan, q, k, v):
    o = torch.empty_like(q)
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    bs.attn_layer(plan, q, k, v, o, plan.workspace("layer"), idx=idx, cnt=cnt)
    return o, idx, cnt


@pytest.mark.parametrize("entry", ["attn_layer", "attn_forward"])
def test_forced_timeout_reports_and_leaves_the_context_usable(bs, tiny, entry):
    wl, plan, q, k, v = tiny
    o_ref, idx, cnt = _layer(bs, plan, q, k, v)
    assert bs.attn_check_device_status(plan) == OK
    ts = plan.tiled_shape()
    tq, tk, tv = (torch.empty(ts, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    for x, y in zip((q, k, v), (tq, tk, tv)):
        bs.attn_reorder(plan, x, y)
    ot_ref = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    bs.attn_forward(plan, tq, tk, tv, idx, cnt, ot_ref)
    assert bs.attn_check_device_status(plan) == OK

    def run():
        if entry == "attn_layer":
            return _layer(bs, plan, q, k, v)[0]
        o = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
        bs.attn_forward(plan, tq, tk, tv, idx, cnt, o)
        return o

    bs.attn_testing_force_timeout(True)
    try:
        run()
        status = bs.attn_check_device_status(plan)
    finally:
        bs.attn_testing_force_timeout(False)
    assert status == TIMEOUT
    # The context is usable and the next call is clean and exact.
    again = run()
    assert bs.attn_check_device_status(plan) == OK
    assert torch.equal(again, o_ref if entry == "attn_layer" else ot_ref)


def test_misaligned_pointers_and_short_workspaces_are_rejected(bs, tiny):
    wl, plan, q, k, v = tiny
    lib = bs._lib
    o = torch.empty_like(q)
    ws = plan.workspace("layer")
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    P = ctypes.c_void_p
    st = P(torch.cuda.current_stream().cuda_stream)
    p = lambda t, off=0: P(t.data_ptr() + off)  # noqa: E731
    nbytes = ws.numel()
    need = plan.info.layer_workspace_bytes
    torch.cuda.synchronize()
    # misaligned inputs / outputs (8 bytes off a 16-byte boundary)
    assert lib.attn_layer(plan.handle, p(q, 8), p(k), p(v), p(o), None, None, None, p(ws), nbytes, st) == INVALID_ARG
    assert lib.attn_layer(plan.handle, p(q), p(k), p(v), p(o, 8), None, None, None, p(ws), nbytes, st) == INVALID_ARG
    assert lib.attn_layer(plan.handle, p(q), p(k), p(v), p(o), None, p(idx, 4), p(cnt), p(ws), nbytes,
                          st) == INVALID_ARG
    # only one of idx_out / cnt_out
    assert lib.attn_layer(plan.handle, p(q), p(k), p(v), p(o), None, p(idx), None, p(ws), nbytes, st) == INVALID_ARG
    # workspace: too small, missing, misaligned
    assert lib.attn_layer(plan.handle, p(q), p(k), p(v), p(o), None, None, None, p(ws), need - 1, st) == WORKSPACE
    assert lib.attn_layer(plan.handle, p(q), p(k), p(v), p(o), None, None, None, None, nbytes, st) == WORKSPACE
    assert lib.attn_layer(plan.handle, p(q), p(k), p(v), p(o), None, None, None, p(ws, 8), nbytes, st) == WORKSPACE
    sel = plan.workspace("select")
    assert lib.attn_select(plan.handle, p(q), p(k), p(idx), p(cnt), p(sel),
                           plan.info.select_workspace_bytes - 1, st) == WORKSPACE
    assert lib.attn_select(plan.handle, p(q, 2), p(k), p(idx), p(cnt), p(sel), sel.numel(), st) == INVALID_ARG
    assert lib.attn_reorder(plan.handle, p(q), p(o, 8), None, st) == INVALID_ARG
    bw = plan.workspace("backward")
    ts = plan.tiled_shape()
    t = [torch.empty(ts, dtype=torch.bfloat16, device="cuda") for _ in range(7)]
    lse = torch.empty((wl.B, wl.heads, plan.N, plan.V), dtype=torch.float32, device="cuda")
    args = [p(x) for x in t[:5]] + [p(lse), p(idx), p(cnt)] + [p(x) for x in t[5:]] + [p(t[0])]
    assert lib.attn_backward(plan.handle, *args, p(bw), plan.info.backward_workspace_bytes - 1, st) == WORKSPACE
    args[0] = p(t[0], 8)
    assert lib.attn_backward(plan.handle, *args, p(bw), bw.numel(), st) == INVALID_ARG
    # Nothing was enqueued and nothing was flagged.
    torch.cuda.synchronize()
    assert bs.attn_check_device_status(plan) == OK
