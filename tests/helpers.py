"""Shared test utilities: small ragged workloads, tensor conversion, and
oracle-side list checks. Test infrastructure only."""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_attention_reorder_b200.datagen import Workload
from oracle import select

# Small cases the oracle finishes in seconds that still span several tiles
# and a ragged tail along every axis.
SMALL = {
    "tiny_d64": Workload("tiny_d64", 1, 2, 64, 8, 16, 16, "topk", k=8, recipe="iid", seed=0),
    "ragged_topk": Workload("ragged_topk", 2, 3, 128, 7, 10, 13, "topk", k=5, seed=11),
    "ragged_topp": Workload("ragged_topp", 1, 3, 128, 7, 10, 13, "topp", k=3, p=0.9, seed=12,
                            temperature=(0.3, 3.0)),
    "ragged_window_fp8": Workload("ragged_window_fp8", 1, 2, 128, 9, 10, 13, "window",
                                  win=(1, 1, 0), qk_fp8=True, seed=13),
    "ragged_d64_fp8": Workload("ragged_d64_fp8", 1, 2, 64, 5, 9, 6, "topk", k=4, qk_fp8=True,
                               seed=14),
    "ragged_bf16_window": Workload("ragged_bf16_window", 1, 2, 128, 6, 6, 9, "window",
                                   win=(1, 0, 1), seed=15),
    # Other tile shapes: a 64-token tile that is not a cube, and tiles of
    # several 64-row chunks, some of them padding only at the grid's edge.
    "tile248_window_fp8": Workload("tile248_window_fp8", 1, 2, 128, 5, 9, 13, "window",
                                   win=(1, 1, 0), qk_fp8=True, seed=16, tile=(2, 4, 8)),
    "tile688_topk": Workload("tile688_topk", 2, 2, 128, 9, 12, 13, "topk", k=3, seed=17,
                             tile=(6, 8, 8)),
    "tile488_topp": Workload("tile488_topp", 1, 3, 128, 6, 11, 17, "topp", k=2, p=0.9, seed=18,
                             temperature=(0.3, 3.0), tile=(4, 8, 8)),
    "tile688_window_fp8": Workload("tile688_window_fp8", 1, 2, 128, 9, 12, 13, "window",
                                   win=(1, 1, 1), qk_fp8=True, seed=19, tile=(6, 8, 8)),
    "tile11x128_d64": Workload("tile11x128_d64", 1, 2, 64, 3, 5, 70, "topk", k=2, seed=20,
                               tile=(1, 1, 128)),
}


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def lists_from_device(idx: torch.Tensor, cnt: torch.Tensor):
    idx = idx.cpu().numpy().reshape(-1, idx.shape[-1])
    cnt = cnt.cpu().numpy().reshape(-1)
    return [idx[r, :cnt[r]].astype(np.int64) for r in range(cnt.size)]


def lists_to_device(lists, kmax: int, device="cuda"):
    rows = len(lists)
    idx = np.full((rows, kmax), -1, dtype=np.int32)
    cnt = np.zeros((rows,), dtype=np.int32)
    for r, l in enumerate(lists):
        idx[r, :len(l)] = l
        cnt[r] = len(l)
    return torch.from_numpy(idx).to(device), torch.from_numpy(cnt).to(device)


def assert_topp_equal(got, S_row, p, k, tol=1e-12):
    """GPU top-p list vs the oracle's on the same fp32 row.

    The prefix masses c_m are rounded on both sides (the oracle in fp64, the
    kernel in 2^-52 fixed point, < 2.3e-13 for N <= 2048), so any m* whose
    c_m lies within `tol` of p is a rounding tie: the count may be any
    min(N, max(m, k)) for m from the first c_m >= p - tol to the first
    c_m >= p + tol. The kept set must still be that many top-ranked tiles."""
    want_cnt, c = select.topp_count(S_row, p, k)
    order = select.rank_order(S_row)
    N = S_row.shape[0]
    n = len(got)
    if n != want_cnt:
        lo_hit = np.nonzero(c >= p - tol)[0]
        hi_hit = np.nonzero(c >= p + tol)[0]
        lo = int(lo_hit[0]) + 1 if lo_hit.size else N
        hi = int(hi_hit[0]) + 1 if hi_hit.size else N
        allowed = {min(N, max(m, k)) for m in range(lo, hi + 1)}
        assert n in allowed, (n, want_cnt, sorted(allowed)[:4])
    np.testing.assert_array_equal(np.asarray(got), np.sort(order[:n]))


def assert_valid_selection(got, S_row64, rule, k=0, p=0.0, eps=1e-5):
    """Lists computed from fp32 scores are a valid selection under the oracle's
    fp64 scores up to `eps` (only near-ties may be decided differently)."""
    got = np.asarray(got)
    n = S_row64.shape[0]
    dropped = np.setdiff1d(np.arange(n), got)
    if rule == "topk":
        assert got.size == min(k, n)
    if rule in ("topk", "topp") and got.size and dropped.size:
        assert S_row64[got].min() >= S_row64[dropped].max() - eps
