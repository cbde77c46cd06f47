"""bench.py's own bookkeeping, on CPU: the kernel launches it claims per call for each method and
split, and the DRAM traffic it reports from the committed ncu captures.

The launch counts follow the library's stage order (block pooling; the pooled scores and the
selection from them per chunk of heads, one fused group-selection kernel, or the anti-diagonal
estimator, its row statistics, the merge into p and the selection from p; the head-pair
schedule; attention). The traffic figures are reported only while the kernel sources hash to
the revision the captures measured, so this test fails when a kernel changes and its capture
is not taken again.
"""

import importlib.util
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_causal_pooling_b200 import workloads as wl  # noqa: E402


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _views(B, Hq, Hkv, S, D):
    q = torch.empty(B, Hq, S, D, device="meta")
    kv = torch.empty(B, Hkv, S, D, device="meta")
    return [(q, kv, kv, q, None, None)]


def test_launches_per_call_by_method():
    b = _bench()
    w = wl.LLAMA_128K
    views = _views(w.B, w.Hq, w.Hkv, w.S, w.D)
    chunks = b.select_chunks(w.B, w.Hq, w.Hkv, w.nb)
    assert chunks == 1  # all 32 heads' score triangles (67 MB) fit the 128 MB region
    assert b.launches_per_call(w, views) == 3 + 2 * chunks
    assert b.launches_per_call(w, views, {"score": "antidiag", "stride": 16}) == 7
    assert b.launches_per_call(w, views, {"share": "group"}) == 4
    # two segments (a rank's share cut through a batch entry): the counts add up
    two = _views(1, 8, 2, w.S, w.D) * 2
    assert b.launches_per_call(w, two) == 2 * (3 + 2 * b.select_chunks(1, 8, 2, w.nb))


def test_score_chunks_at_nb_4096():
    b = _bench()
    # one head's triangle at nb 4096 is 4 * 4096 * 4097 / 2 = 33,562,624 bytes; the region is
    # the head-pair schedule's, 256 + 4 * 8 kv heads * 2 pairs * 8,390,656 = 537,002,240 bytes
    # (above the 128 MB cap), so it holds 16 triangles: 32 heads run in two chunks
    assert b.select_chunks(1, 32, 8, 4096) == 2
    # G = 1 (one head per pair): the schedule region is 256 + 4 * 32 * 8,390,656 bytes, 32
    # triangles, so one chunk
    assert b.select_chunks(1, 32, 32, 4096) == 1


def test_traffic_stamps_match_the_kernel_sources():
    b = _bench()
    assert b.attn_traffic("llama3-8b-128k") == b.ATTN_TRAFFIC["bytes"]
    assert b.antidiag_traffic("llama3-8b-128k", 16) == b.AD_TRAFFIC["bytes"]
    # only the captured workload and stride
    assert b.attn_traffic("llama3-8b-32k") is None
    assert b.antidiag_traffic("llama3-8b-128k", 8) is None
