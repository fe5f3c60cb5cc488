"""Multi-process host logic of bench.py on CPU: two ranks over gloo (127.0.0.1).

The decode path is data parallel over sequences with no collective on the data path; the
only cross-rank steps are the barriers around the timed region and the max over ranks of
the timed interval.  These tests run that logic with world size 2 and check the
reference arm's rank handling (rank 0 alone works, the other ranks exit quietly).
"""
from __future__ import annotations

import os
import socket
import sys
from datetime import timedelta

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local_ms = 100.0 + 25.0 * rank                    # rank 1 is the slower one
        dist.barrier()
        slowest = bench.max_over_ranks(local_ms, world, "cpu")
        rate = bench.whole_job_rate(world, 64, 10, slowest)
        ref = bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"]),
                                  rank, world)
        dist.barrier()
        q.put((rank, slowest, rate, ref, bench.rank_seed_offset(rank)))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_reference_arm():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, slowest, rate, ref, seed = q.get(timeout=120)
        got[rank] = (slowest, rate, ref, seed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's interval; the rate counts all ranks' sequences
    assert got[0][0] == got[1][0] == 125.0
    assert got[0][1] == pytest.approx(2 * 64 * 10 / 0.125)
    # distinct sequences per rank
    assert got[0][3] != got[1][3]
    # reference arm: rank 1 does no work; rank 0 answers (here without a GPU: unavailable)
    assert got[1][2] is None
    assert got[0][2]["impl"] == "reference"
    assert "unavailable" in got[0][2] or got[0][2]["value"] > 0


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_rate(1, 64, 5, 1000.0) == pytest.approx(320.0)
    assert bench.rank_seed_offset(0) == 0
