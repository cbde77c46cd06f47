"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

The path needs no data-path collective (each rank runs an independent problem); the ranks
only agree on timing. These tests run the same helpers bench.py uses, in two processes.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_causal_pooling_b200 import workloads as wl

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r is slower by r seconds: every rank must see the slowest time
        t = bench.max_over_ranks(1.0 + rank, world)
        # the whole-job value counts every rank's work over the slowest time
        v = bench.whole_job_tflops(2e12, world, t)
        # problems differ by seed only
        w = bench.rank_workload(wl.LLAMA_32K, rank)
        shapes = torch.tensor([w.B, w.Hq, w.Hkv, w.S, w.seed], dtype=torch.int64)
        gathered = [torch.zeros_like(shapes) for _ in range(world)]
        dist.all_gather(gathered, shapes)
        out[rank] = (t, v, [g.tolist() for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_slowest_time_and_whole_job_value():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        t, v, shapes = out[r]
        assert t == 2.0
        assert v == pytest.approx(world * 2e12 / 2.0 / 1e12)
        assert shapes[0][:4] == shapes[1][:4]          # same shape on every rank
        assert shapes[0][4] != shapes[1][4]            # independent problems


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_tflops(1e12, 1, 0.5) == pytest.approx(2.0)
