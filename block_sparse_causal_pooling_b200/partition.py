"""Partition of one prefill problem across ranks by (batch, kv-head group).

Every step of the path for query head h reads only kv head h // G (G = Hq / Hkv): the block
pooling of its Q, K and V, the metric and top-k of its rows, and the attention over its kept
K/V blocks ("Stem: Rethinking Causal Information Flow in Sparse Attention" states the problem
per head: causal prefill over Q, K, V with a per-query-block selection of key blocks, es
technical summary section 1). So the (batch, kv head) units of one problem are independent,
and a rank that takes a contiguous range of them computes exactly its slice of the outputs
with no exchange of data.

The units are ordered batch-major, (b, g) -> b * Hkv + g, and rank r of N takes units
[floor(r U / N), floor((r + 1) U / N)) of the U = B * Hkv. A range is cut into segments that
are contiguous in every tensor of the [B, H, S, D] layout: either whole batch entries
b0 .. b1 (every head), or kv heads g0 .. g1 of one batch entry (query heads g0*G .. g1*G).
The library is called once per segment, on those views, as for a problem of b1 - b0 batch
entries with g1 - g0 kv heads. With one rank the only segment is the whole problem.

Host-side only: this module computes index ranges and views; every step of the path runs in the
library's kernels.
"""

from __future__ import annotations

from typing import Iterator, List, NamedTuple, Tuple


class Segment(NamedTuple):
    b0: int  # first batch entry
    b1: int  # one past the last batch entry
    g0: int  # first kv head (0 when the segment spans several batch entries)
    g1: int  # one past the last kv head (Hkv when it spans several)


def rank_units(B: int, Hkv: int, rank: int, world: int) -> Tuple[int, int]:
    """[u0, u1): the (batch, kv head) units of rank `rank` out of `world`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    U = B * Hkv
    return rank * U // world, (rank + 1) * U // world


def segments(B: int, Hkv: int, rank: int, world: int) -> List[Segment]:
    """The rank's units as contiguous segments, in unit order: a partial batch entry at either
    end of the range, whole batch entries in between merged into one segment."""
    u0, u1 = rank_units(B, Hkv, rank, world)
    out = []
    u = u0
    while u < u1:
        b, g0 = divmod(u, Hkv)
        if g0 == 0 and u1 - u >= Hkv:  # whole batch entries
            nfull = (u1 - u) // Hkv
            out.append(Segment(b, b + nfull, 0, Hkv))
            u += nfull * Hkv
        else:
            g1 = min(Hkv, g0 + (u1 - u))
            out.append(Segment(b, b + 1, g0, g1))
            u += g1 - g0
    return out


def segment_views(seg: Segment, G: int, q, k, v, out, sel_idx, sel_cnt):
    """Contiguous views of one segment: (q, k, v, out, sel_idx, sel_cnt), each
    [b1 - b0, heads, ...]. q/out/sel_idx/sel_cnt are the full [B, Hq, ...] tensors, k/v the full
    [B, Hkv, ...] ones."""
    hq0, hq1 = seg.g0 * G, seg.g1 * G
    bs = slice(seg.b0, seg.b1)
    views = (q[bs, hq0:hq1], k[bs, seg.g0:seg.g1], v[bs, seg.g0:seg.g1], out[bs, hq0:hq1],
             sel_idx[bs, hq0:hq1], sel_cnt[bs, hq0:hq1])
    for t in views:
        if not t.is_contiguous():
            raise ValueError("segment views need contiguous [B, H, ...] tensors")
    return views


def rank_views(q, k, v, out, sel_idx, sel_cnt, rank: int, world: int) -> Iterator[tuple]:
    """The views of every segment of `rank`, in order."""
    B, Hq = q.shape[0], q.shape[1]
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    for seg in segments(B, Hkv, rank, world):
        yield segment_views(seg, G, q, k, v, out, sel_idx, sel_cnt)
