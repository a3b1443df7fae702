"""attn_select_static: key-tile selection without a caller-provided workspace.

Some callers cannot allocate device memory themselves: code running where
cudaMalloc is not allowed, or embedded in a host application whose device
allocator is owned by someone else. attn_select_static serves them by using
one static device array inside the library as scratch. These checks call it
through the C ABI and compare it with attn_select (same kernels, caller
workspace) on two calls in a row, so that stale scratch contents from the
first call cannot leak into the second. Selection is exact, so the lists
must match exactly. The file sorts last so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_reorder_b200.datagen import WORKLOADS, make_qkv
from tests.helpers import SMALL, lists_from_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bs():
    from block_sparse_attention_reorder_b200 import bsattn
    return bsattn


def _lists(bs, plan, fn, q, k):
    si, sc = plan.list_shapes()
    idx = torch.full(si, -5, dtype=torch.int32, device="cuda")
    cnt = torch.full(sc, -5, dtype=torch.int32, device="cuda")
    fn(idx, cnt)
    assert bs.attn_check_device_status(plan) == 0
    return lists_from_device(idx, cnt)


@pytest.mark.parametrize("name", ["wan1.3b", "tiny", "ragged_topp", "ragged_topk", "ragged_bf16_window"])
def test_static_scratch_matches_workspace_version_twice(bs, name):
    wl = WORKLOADS.get(name) or SMALL[name]
    plan = bs.Plan.for_workload(wl)
    assert plan.info.select_workspace_bytes <= bs.STATIC_SELECT_SCRATCH_BYTES
    ws = plan.workspace("select")
    for call in range(2):  # second call gets different inputs on the same scratch
        q, k, _ = make_qkv(wl, "cuda", batch_offset=call)
        want = _lists(bs, plan, lambda i, c: bs.attn_select(plan, q, k, i, c, ws), q, k)
        got = _lists(bs, plan, lambda i, c: bs.attn_select_static(plan, q, k, i, c), q, k)
        assert len(got) == len(want)
        assert all(np.array_equal(a, b) for a, b in zip(got, want)), f"call {call}"


def test_static_scratch_rejects_problems_beyond_its_capacity(bs):
    plan = bs.Plan.for_workload(WORKLOADS["wan14b"])  # select workspace ~0.4 GB
    assert plan.info.select_workspace_bytes > bs.STATIC_SELECT_SCRATCH_BYTES
    q = torch.zeros(plan.natural_shape(), dtype=torch.bfloat16, device="cuda")
    si, sc = plan.list_shapes()
    idx = torch.empty(si, dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc, dtype=torch.int32, device="cuda")
    with pytest.raises(bs.BsattnError) as e:
        bs.attn_select_static(plan, q, q, idx, cnt)
    assert e.value.code == 2
