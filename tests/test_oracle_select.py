"""Pins for the oracle's block scores and selection rules (CPU only)."""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import select, tiling
from block_sparse_attention_reorder_b200.datagen import random_scores


def test_scores_hand_example():
    pq = np.array([[1.0, 2.0], [0.0, -1.0]])
    pk = np.array([[3.0, 1.0], [2.0, 2.0]])
    S = select.block_scores(pq, pk, 0.5)
    np.testing.assert_array_equal(S, [[2.5, 3.0], [-0.5, -1.0]])


def brute_topk(row, k):
    n = row.shape[0]
    kept = []
    for j in range(n):
        better = sum(1 for jj in range(n) if row[jj] > row[j] or (row[jj] == row[j] and jj < j))
        if better < k:
            kept.append(j)
    return np.array(kept)


@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (32, 8), (50, 50), (64, 1), (40, 60)])
def test_topk_rank_rule(n, k):
    S = random_scores(12, n, seed=n * 100 + k).numpy()
    for r in range(S.shape[0]):
        got = select.topk_row(S[r], k)
        assert got.size == min(k, n)
        np.testing.assert_array_equal(got, brute_topk(S[r], k))
        assert np.all(np.diff(got) > 0)


def test_topk_scale_invariant_and_signed_zero_ties():
    S = random_scores(8, 40, seed=5).numpy()
    for r in range(8):
        np.testing.assert_array_equal(select.topk_row(S[r], 9), select.topk_row(S[r] * 4.0, 9))
    row = np.array([0.0, -0.0, 0.0, -1.0, -0.0], dtype=np.float32)
    np.testing.assert_array_equal(select.topk_row(row, 2), [0, 1])
    np.testing.assert_array_equal(select.topk_row(row, 4), [0, 1, 2, 4])


def test_nan_rejected():
    with pytest.raises(ValueError):
        select.topk_row(np.array([0.0, np.nan]), 1)


def brute_topp_count(row, p, k):
    """Smallest subset size whose softmax mass reaches p, by enumeration."""
    n = row.shape[0]
    e = [math.exp(v - max(row)) for v in row]
    tot = sum(e)
    pi = [x / tot for x in e]
    for m in range(1, n + 1):
        best = max(sum(pi[j] for j in c) for c in itertools.combinations(range(n), m))
        if best >= p:
            return max(m, k), best
    return n, 1.0


@pytest.mark.parametrize("n", [1, 3, 6, 9])
@pytest.mark.parametrize("p,k", [(0.5, 1), (0.9, 2), (0.99, 0), (1.0, 1), (0.3, 5)])
def test_topp_minimal_subset_by_enumeration(n, p, k):
    rng = np.random.default_rng(n * 31 + int(p * 100) + k)
    for _ in range(5):
        row = (rng.standard_normal(n) * 2.0).astype(np.float32)
        want, _ = brute_topp_count(row.astype(np.float64), p, k)
        cnt, c = select.topp_count(row, p, k)
        want = min(want, n)
        if cnt != want:  # only an fp rounding tie at the boundary may differ
            assert abs(c[min(cnt, want) - 1] - p) < 1e-12
        lst = select.topp_row(row, p, k)
        assert lst.size == cnt
        # kept set is the top-ranked prefix: every kept score >= every dropped one
        dropped = np.setdiff1d(np.arange(n), lst)
        if dropped.size and lst.size:
            assert row[lst].min() >= row[dropped].max()


def test_topp_special_cases():
    row = np.zeros(20)
    row[7] = 100.0
    assert select.topp_count(row, 0.9, 1)[0] == 1
    assert select.topp_count(row, 0.9, 4)[0] == 4
    np.testing.assert_array_equal(select.topp_row(row, 0.9, 3), [0, 1, 7])
    uni = np.zeros(50)
    for p in (0.1, 0.5, 0.9, 0.97):
        cnt = select.topp_count(uni, p, 1)[0]
        assert cnt in (math.ceil(p * 50), math.ceil(p * 50) + 1)
        np.testing.assert_array_equal(select.topp_row(uni, p, 1), np.arange(cnt))


@pytest.mark.parametrize("name", ["window_fp8", "window_fp8_t688"])
def test_window_closed_form(golden_dir, name):
    g = json.load(open(os.path.join(golden_dir, "workload_counts.json")))[name]
    nT, nH, nW = g["tiles"]
    total = sum(select.window_row(i, (nT, nH, nW), (1, 1, 0)).size for i in range(nT * nH * nW))
    assert total == g["kept_pairs_per_head"] == (3 * nT - 2) * (3 * nH - 2) * nW


@pytest.mark.parametrize("grid,half", [((3, 4, 5), (1, 1, 0)), ((2, 2, 2), (0, 0, 0)),
                                       ((4, 3, 5), (2, 1, 1)), ((1, 6, 2), (1, 2, 1))])
def test_window_sets(grid, half):
    nT, nH, nW = grid

    def axis_total(n, a):
        return sum(min(n - 1, i + a) - max(0, i - a) + 1 for i in range(n))

    tot = 0
    for i in range(nT * nH * nW):
        lst = select.window_row(i, grid, half)
        ti, hi, wi = i // (nH * nW), (i // nW) % nH, i % nW
        assert i in lst
        for j in lst:
            tj, hj, wj = j // (nH * nW), (j // nW) % nH, j % nW
            assert abs(tj - ti) <= half[0] and abs(hj - hi) <= half[1] and abs(wj - wi) <= half[2]
        tot += lst.size
    assert tot == axis_total(nT, half[0]) * axis_total(nH, half[1]) * axis_total(nW, half[2])


def test_route_topk_count_on_tiny_workload():
    from block_sparse_attention_reorder_b200.datagen import WORKLOADS, make_qkv
    wl = WORKLOADS["tiny"]
    q, k, _ = (x.float().numpy() for x in make_qkv(wl))
    _, _, S, lists = __import__("oracle").attention.route(q, k, wl.T, wl.H, wl.W, "topk", k=wl.k)
    assert S.shape == (1, 2, 32, 32)
    assert all(len(l) == 8 for l in lists)
    assert tiling.n_blocks(wl.T, wl.H, wl.W) == 32
