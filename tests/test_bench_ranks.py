"""The benchmark's multi-rank host logic on CPU: two gloo ranks.

With N GPUs every rank runs its own layer (independent problems, weak
scaling, no data-path collective). What the ranks share is host logic: the
step time is the slowest rank's (an all-reduce MAX), the job's throughput
is N times one rank's work over that time, each rank draws its own inputs,
and only rank 0 runs and prints the reference arm. No GPU is touched.
"""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from block_sparse_attention_reorder_b200.datagen import WORKLOADS, make_qkv

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(1.5 + rank, dist, device="cpu")
        q, _, _ = make_qkv(WORKLOADS["tiny"], "cpu", batch_offset=rank)
        digests = [None] * world
        dist.all_gather_object(digests, float(q.float().abs().sum()))
        out.put((rank, ms, bench.job_tflops(world, 2.0e9, ms), digests))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_time_the_slowest_and_count_both_ranks_work():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(out.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for rank, ms, tflops, digests in res:
        assert ms == 2.5                                       # rank 1's 2.5 ms, seen by both ranks
        assert tflops == pytest.approx(2 * 2.0e9 / 2.5e-3 / 1e12)
        assert digests[0] != digests[1]                        # each rank its own batch


def test_one_rank_keeps_its_own_numbers():
    import bench

    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.job_tflops(1, 1e12, 1.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                                      "--warmup", "0"])
    assert bench.run_reference(bench.parse()) == 0
    assert capsys.readouterr().out == ""
