"""Partition of one problem by (batch, kv-head group) across ranks (the multi-GPU split).

Host logic on CPU: the unit ranges cover every (batch, kv head) exactly once, a segment spans
several batch entries only when it holds all their kv heads, and the views are contiguous. Then a world-size-2 run over gloo: each
rank computes its segments with the oracle (no GPU here), writes them into full-size buffers,
the disjoint pieces are summed across ranks, and the result must equal the single-process
oracle on the whole problem: the CSR bit for bit, the output exactly (every step of the path
for a query head reads only its own kv head, so a segment is an independent problem).
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_causal_pooling_b200 import partition as P  # noqa: E402
from block_sparse_causal_pooling_b200 import workloads as wl  # noqa: E402

# B 3, Hkv 2: six units, so the two ranks' ranges cut through batch entry 1
W = wl.LLAMA_32K.replace(name="partition", B=3, Hq=4, Hkv=2, S=5 * 128 + 40, tau=3.0, k_min=2)


@pytest.mark.parametrize("B,Hkv,world", [(1, 8, 1), (1, 8, 2), (1, 8, 8), (3, 2, 2), (3, 2, 4),
                                         (2, 3, 5), (1, 4, 8), (4, 1, 3)])
def test_units_cover_every_kv_head_once(B, Hkv, world):
    seen = []
    for r in range(world):
        u0, u1 = P.rank_units(B, Hkv, r, world)
        segs = P.segments(B, Hkv, r, world)
        units = [b * Hkv + g for s in segs for b in range(s.b0, s.b1) for g in range(s.g0, s.g1)]
        assert units == list(range(u0, u1))
        for s in segs:
            assert 0 <= s.b0 < s.b1 <= B and 0 <= s.g0 < s.g1 <= Hkv
            # several batch entries only when every kv head of them is in the segment
            assert s.b1 == s.b0 + 1 or (s.g0 == 0 and s.g1 == Hkv)
        seen += units
    if world == 1:
        assert P.segments(B, Hkv, 0, 1) == [P.Segment(0, B, 0, Hkv)]  # the whole problem
    assert seen == list(range(B * Hkv))
    # balanced: unit counts differ by at most one
    counts = [P.rank_units(B, Hkv, r, world)[1] - P.rank_units(B, Hkv, r, world)[0]
              for r in range(world)]
    assert max(counts) - min(counts) <= 1


def test_segment_views_are_contiguous_slices():
    q = torch.arange(3 * 4 * 10 * 2).view(3, 4, 10, 2)
    k = torch.arange(3 * 2 * 10 * 2).view(3, 2, 10, 2)
    out = torch.zeros_like(q)
    si = torch.zeros(3, 4, 7, dtype=torch.int32)
    sc = torch.zeros(3, 4, 3, dtype=torch.int32)
    views = list(P.rank_views(q, k, k, out, si, sc, 1, 2))
    assert [tuple(t.shape) for t in views[0]] == [(1, 2, 10, 2), (1, 1, 10, 2), (1, 1, 10, 2),
                                                  (1, 2, 10, 2), (1, 2, 7), (1, 2, 3)]
    # rank 1 of 2 takes units 3..5: (b 1, g 1) then (b 2, g 0..1)
    assert torch.equal(views[0][0], q[1:2, 2:4]) and torch.equal(views[1][1], k[2:3, 0:2])
    assert all(t.is_contiguous() for vs in views for t in vs)
    with pytest.raises(ValueError):
        P.rank_units(1, 8, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, res):
    sys.path.insert(0, ROOT)
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = wl.make_inputs(W, "cpu")
        kk, off = oracle.budget(W.nb, W.rho_min, W.tau, W.k_min)
        cap = int(off[-1])
        out = torch.zeros(W.B, W.Hq, W.nb * W.block, W.D, dtype=torch.float64)
        si = torch.zeros(W.B, W.Hq, cap, dtype=torch.int32)
        sc = torch.zeros(W.B, W.Hq, W.nb, dtype=torch.int32)
        n_seg = 0
        for vq, vk, vv, vo, vsi, vsc in P.rank_views(q, k, v, out, si, sc, rank, world):
            r = oracle.prefill(vq, vk, vv, W.block, W.rho_min, W.tau, W.k_min,
                               with_metric=False)
            vo.copy_(torch.from_numpy(r["out"]).view(vq.shape[0], vq.shape[1], W.nb * W.block,
                                                     W.D))
            vsi.copy_(torch.from_numpy(r["sel_idx"]))
            vsc.copy_(torch.from_numpy(r["sel_cnt"]))
            n_seg += 1
        # disjoint pieces: the sum over ranks is their union
        for t in (out, si, sc):
            dist.all_reduce(t, op=dist.ReduceOp.SUM)
        if rank == 0:
            ref = oracle.prefill(q, k, v, W.block, W.rho_min, W.tau, W.k_min, with_metric=False)
            res["csr"] = (np.array_equal(si.numpy(), ref["sel_idx"]) and
                          np.array_equal(sc.numpy(), ref["sel_cnt"]))
            got = out.view(W.B * W.Hq * W.nb, W.block, W.D).numpy()
            res["out_max_abs"] = float(np.abs(got - ref["out"]).max())
        res[f"segments{rank}"] = n_seg
    finally:
        dist.destroy_process_group()


def test_two_ranks_reassemble_the_single_process_oracle():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    res = mgr.dict()
    mp.spawn(_worker, args=(world, port, res), nprocs=world, join=True)
    assert res["segments0"] == 2 and res["segments1"] == 2  # both ranks cut batch entry 1
    assert res["csr"]
    assert res["out_max_abs"] == 0.0
