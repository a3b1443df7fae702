"""Host-side accounting of bench.py: the attention kernel's issued work and the
committed traffic record, checked on CPU.

`group_accounting` counts what the kernel multiplies when it stacks two
64-token query tiles into one 128-row block: every key tile in the union of
the two kept lists is one step (two 64 x 64 products). Here that count is
recomputed by brute force over explicit tile pairs.
"""
import hashlib
import json
import os
import types

import numpy as np
import pytest
import torch

import bench
from block_sparse_attention_reorder_b200.datagen import Workload


def _fake_plan(nT, nH, nW, kmax):
    N = nT * nH * nW
    info = types.SimpleNamespace(nT=nT, nH=nH, nW=nW)
    return types.SimpleNamespace(N=N, V=64, kmax=kmax, info=info)


def _brute(lists, nT, nH, nW, axis):
    """(issued 64x64 products, K/V loads) for tiles paired along `axis`."""
    nd = (nT, nH, nW)
    issued = loads = 0
    for bh in range(len(lists)):
        for t in range(nT):
            for h in range(nH):
                for w in range(nW):
                    c = [t, h, w]
                    if c[axis] % 2:
                        continue
                    i0 = (t * nH + h) * nW + w
                    c[axis] += 1
                    u = set(lists[bh][i0])
                    if c[axis] < nd[axis]:
                        u |= set(lists[bh][(c[0] * nH + c[1]) * nW + c[2]])
                    loads += len(u)
                    issued += 2 * len(u)
    return issued, loads


@pytest.mark.parametrize("rule,win,axis", [("topk", (0, 0, 0), 0), ("topp", (0, 0, 0), 0),
                                           ("window", (0, 1, 2), 2), ("window", (1, 1, 0), 0),
                                           ("window", (0, 2, 1), 1)])
def test_issued_work_matches_explicit_pairs(rule, win, axis):
    nT, nH, nW, heads, kmax = 5, 2, 3, 3, 7  # odd extents: a last tile without a partner
    N = nT * nH * nW
    rng = np.random.default_rng(7)
    lists = [[np.sort(rng.choice(N, size=rng.integers(0, kmax + 1), replace=False)) for _ in range(N)]
             for _ in range(heads)]
    idx = torch.full((1, heads, N, kmax), -1, dtype=torch.int32)
    cnt = torch.zeros((1, heads, N), dtype=torch.int32)
    for h in range(heads):
        for i in range(N):
            idx[0, h, i, :len(lists[h][i])] = torch.from_numpy(lists[h][i].astype(np.int32))
            cnt[0, h, i] = len(lists[h][i])
    wl = Workload("t", 1, heads, 128, 4 * nT, 4 * nH, 4 * nW, rule, k=3, p=0.9, win=win)
    assert bench.group_axes(wl)[0] == axis
    got = bench.group_accounting(wl, _fake_plan(nT, nH, nW, kmax), idx, cnt)
    assert got == _brute(lists, nT, nH, nW, axis)


def test_traffic_record_matches_the_kernel_source_or_reads_as_missing(tmp_path, monkeypatch):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "attn_tc_traffic.json")) as f:
        rec = json.load(f)
    with open(os.path.join(root, rec["kernel_source"]), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    # The record's figures are reported only while they belong to the kernel
    # source they were captured with.
    if sha == rec["sha256_prefix"]:
        assert bench.measured_traffic("wan1.3b") == rec["per_launch_dram_bytes"]["wan1.3b"]
    else:
        assert bench.measured_traffic("wan1.3b") is None
    # A changed kernel source makes every figure read as missing.
    (tmp_path / "profiles").mkdir()
    changed = dict(rec, kernel_source="attn_tc_changed.cu")
    (tmp_path / "profiles" / "attn_tc_traffic.json").write_text(json.dumps(changed))
    (tmp_path / "attn_tc_changed.cu").write_text("// another kernel\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("wan1.3b") is None


@pytest.mark.parametrize("grid,tile", [((7, 10, 13), (4, 4, 4)), ((9, 12, 13), (6, 8, 8)),
                                       ((8, 8, 8), (4, 4, 4))])
def test_valid_token_flops_counts_real_token_products(grid, tile):
    """The real-token figure, against a per-token count: for every kept tile
    pair, the number of (real query, real key) token pairs times 4 D."""
    from oracle import tiling

    T, H, W = grid
    nT, nH, nW = (-(-n // t) for n, t in zip(grid, tile))
    N, heads, kmax, D = nT * nH * nW, 2, 5, 128
    rng = np.random.default_rng(3)
    lists = [[np.sort(rng.choice(N, size=rng.integers(0, kmax + 1), replace=False)) for _ in range(N)]
             for _ in range(heads)]
    idx = torch.full((1, heads, N, kmax), -1, dtype=torch.int32)
    cnt = torch.zeros((1, heads, N), dtype=torch.int32)
    for h in range(heads):
        for i in range(N):
            idx[0, h, i, :len(lists[h][i])] = torch.from_numpy(lists[h][i].astype(np.int32))
            cnt[0, h, i] = len(lists[h][i])
    # Real tokens per tile from the oracle's token -> tile map.
    tok_tile, _ = tiling.token_tile_and_row(T, H, W, tile)
    real = np.bincount(tok_tile, minlength=N)
    want = sum(4 * D * real[i] * real[j] for h in range(heads) for i in range(N) for j in lists[h][i])
    wl = Workload("t", 1, heads, D, T, H, W, "topk", k=3, tile=tile)
    plan = types.SimpleNamespace(N=N, V=int(np.prod(tile)), kmax=kmax,
                                 info=types.SimpleNamespace(nT=nT, nH=nH, nW=nW))
    assert bench.valid_token_flops(wl, plan, idx, cnt) == float(want)
    if grid == (8, 8, 8):  # no padding: every kept pair counts in full
        kept = sum(len(l) for hl in lists for l in hl)
        assert want == kept * bench.pair_flops(D)
