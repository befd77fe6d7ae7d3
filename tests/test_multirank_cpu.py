"""Multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

The path partitions into independent problems, so ranks run replicas with no
data-path collective; the only cross-rank steps are the barrier and the
max-over-ranks of the timed duration.  These tests run that logic as two real
processes over gloo on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from seeded_inputs import WORKLOADS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank              # rank 1 is the slowest
        mx = bench.dist_max(local_ms, world)
        w = WORKLOADS["fwdbwd_1x16384_h16_d128_bf16_causal"]
        seed = bench.replica_workload(w, rank).seed
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        bench.dist_barrier(world)
        out[rank] = (mx, tuple(seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0           # every rank sees the slowest time
    assert out[0][1] == out[1][1] and len(set(out[0][1])) == world  # distinct replica seeds


def test_aggregate_counts_every_rank_over_slowest_time():
    f = bench.fwd_flops(WORKLOADS["fwdbwd_1x16384_h16_d128_bf16_causal"]) * 3.5
    one = bench.aggregate_tflops(1, f, 10, 50.0)
    assert bench.aggregate_tflops(4, f, 10, 50.0) == pytest.approx(4 * one)
    assert bench.aggregate_tflops(4, f, 10, 100.0) == pytest.approx(2 * one)


def test_visible_pair_counts():
    # full, causal, window and bottom-right alignment against brute force
    for Nq, Nk, causal, window in [(7, 7, False, (-1, -1)), (7, 7, True, (-1, -1)),
                                   (9, 5, True, (-1, -1)), (6, 11, False, (2, 1)),
                                   (8, 8, True, (3, 3))]:
        off = Nk - Nq
        brute = 0
        for i in range(Nq):
            for j in range(Nk):
                ok = (not causal or j <= i + off)
                ok = ok and (window[0] < 0 or j >= i + off - window[0])
                ok = ok and (window[1] < 0 or j <= i + off + window[1])
                brute += ok
        assert bench.visible_pairs(Nq, Nk, causal, window) == brute
