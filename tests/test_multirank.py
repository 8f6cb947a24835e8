"""CPU (gloo, world size 2): the host logic bench.py runs on N > 1 ranks -- per-rank input
seeds, max-over-ranks device time, whole-job throughput -- with no GPU."""

from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [3.0, 5.0][rank]
        mx = bench.max_over_ranks(elapsed, world)
        from exact_attention_111_b200.inputs import make_inputs
        x = make_inputs(1, 1, 8, 64, bench.rank_seed(1002, rank))["q"]
        gathered = [torch.empty_like(x.float()) for _ in range(world)]
        dist.all_gather(gathered, x.float())
        distinct = not torch.equal(gathered[0], gathered[1])
        q.put((rank, mx, distinct))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_seeds():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [5.0, 5.0]        # every rank sees the slowest rank's time
    assert all(r[2] for r in res)                    # ranks process different heads


def test_aggregate_is_whole_job():
    # 2 ranks, 1 TFLOP per rank-step, 10 steps in 100 ms (slowest rank) -> 200 TFLOP/s
    assert abs(bench.aggregate_tflops(2, 1e12, 10, 100.0) - 200.0) < 1e-9
