"""CPU oracle for Stem block-sparse causal prefill (ctypes wrapper over stem_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path. It shares no code with
the CUDA library; both take their inputs from the seeded workload generator.

All arithmetic is double precision. The budget parameters cross the library
boundary as single-precision floats, so the oracle rounds rho_min and tau to
float32 first and then widens them to double, exactly as the product does.

Parity status: every function here is pinned by the CPU test suite (budget:
arbitrary-precision recomputation, closed forms; linear budget: cases worked by
hand, closed forms, exact rational recomputation; pooling, metric, selection,
attention: brute force from token-level definitions, the additive-metric
equivalence and closed forms, dense attention via a library routine; a partial
last block: slicing and token-mask brute force, prefix invariance). See the
tests for the pins.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None

_c_i32p = ctypes.POINTER(ctypes.c_int32)
_c_i64p = ctypes.POINTER(ctypes.c_int64)
_c_f64p = ctypes.POINTER(ctypes.c_double)


def _load():
    global _lib
    if _lib is None:
        # STEM_ORACLE_LIB points the pin tests at a deliberately broken copy.
        path = os.environ.get("STEM_ORACLE_LIB") or _build.build()
        lib = ctypes.CDLL(path)
        lib.stem_oracle_threads.restype = ctypes.c_int
        lib.stem_oracle_budget.restype = ctypes.c_int64
        lib.stem_oracle_budget.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                           ctypes.c_int, _c_i32p, _c_i64p]
        lib.stem_oracle_budget_linear.restype = ctypes.c_int64
        lib.stem_oracle_budget_linear.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                                  ctypes.c_int, _c_i32p, _c_i64p]
        lib.stem_oracle_pool.restype = None
        lib.stem_oracle_pool.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 8 + [_c_f64p] * 3
        lib.stem_oracle_metric.restype = None
        lib.stem_oracle_metric.argtypes = [_c_f64p] * 3 + [ctypes.c_int] * 5 + [_c_f64p]
        lib.stem_oracle_metric_additive.restype = None
        lib.stem_oracle_metric_additive.argtypes = ([_c_f64p] * 3 + [ctypes.c_int] * 5 +
                                                    [ctypes.c_double, ctypes.c_int, _c_f64p])
        lib.stem_oracle_select.restype = None
        lib.stem_oracle_select.argtypes = [_c_f64p, _c_i32p, _c_i64p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int64, _c_i32p, _c_i32p]
        lib.stem_oracle_antidiag.restype = None
        lib.stem_oracle_antidiag.argtypes = ([ctypes.c_void_p] * 2 + [ctypes.c_int] * 8 +
                                             [_c_i64p, ctypes.c_int64, _c_f64p])
        lib.stem_oracle_attention.restype = None
        lib.stem_oracle_attention.argtypes = ([ctypes.c_void_p] * 3 + [ctypes.c_int] * 7 +
                                              [_c_i32p, _c_i32p, _c_i64p, ctypes.c_int64,
                                               _c_i64p, ctypes.c_int64, _c_f64p])
        _lib = lib
    return _lib


def threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().stem_oracle_threads())


def f32(x: float) -> float:
    """Round a parameter to single precision, as the C boundary does."""
    return float(np.float32(x))


def _ptr(a: np.ndarray, ct):
    return a.ctypes.data_as(ct)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return 0
    if t.dtype == torch.float32:
        return 1
    raise TypeError(f"oracle takes bf16 or f32 inputs, got {t.dtype}")


def _host(t: torch.Tensor) -> torch.Tensor:
    t = t.detach()
    if t.device.type != "cpu":
        t = t.cpu()
    return t.contiguous()


def budget(nb: int, rho_min: float, tau: float, k_min: int):
    """k[nb] (int32) and off[nb+1] (int64) of the position-decay budget."""
    k = np.zeros(max(nb, 1), dtype=np.int32)
    off = np.zeros(nb + 1, dtype=np.int64)
    _load().stem_oracle_budget(nb, f32(rho_min), f32(tau), int(k_min), _ptr(k, _c_i32p),
                               _ptr(off, _c_i64p))
    return k[:nb].copy(), off


def budget_linear(nb: int, k_start: float, mu: float, k_min: int):
    """k[nb] (int32) and off[nb+1] (int64) of the linear position-decay budget (k_start at
    block 0 down to mu*k_start at block nb-1)."""
    k = np.zeros(max(nb, 1), dtype=np.int32)
    off = np.zeros(nb + 1, dtype=np.int64)
    _load().stem_oracle_budget_linear(nb, f32(k_start), f32(mu), int(k_min), _ptr(k, _c_i32p),
                                      _ptr(off, _c_i64p))
    return k[:nb].copy(), off


def pool(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int, vsum: str = "mean"):
    """Pooled block summaries in double: qbar [B,Hq,nb,D], kbar [B,Hkv,nb,D], vnorm [B,Hkv,nb].
    vsum: "mean" (mean row norm of V per block) or "max" (largest row norm)."""
    if vsum not in ("mean", "max"):
        raise ValueError(vsum)
    q, k, v = _host(q), _host(k), _host(v)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    nb = -(-S // block)  # a partial last block counts
    qbar = np.zeros((B, Hq, nb, D))
    kbar = np.zeros((B, Hkv, nb, D))
    vnorm = np.zeros((B, Hkv, nb))
    _load().stem_oracle_pool(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, Hq,
                             Hkv, S, D, block, int(vsum == "max"), _ptr(qbar, _c_f64p),
                             _ptr(kbar, _c_f64p), _ptr(vnorm, _c_f64p))
    return qbar, kbar, vnorm


def metric(qbar: np.ndarray, kbar: np.ndarray, vnorm: np.ndarray) -> np.ndarray:
    """Output-aware block metric, packed lower triangle: [B, Hq, nb*(nb+1)/2]."""
    qbar = np.ascontiguousarray(qbar, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    vnorm = np.ascontiguousarray(vnorm, dtype=np.float64)
    B, Hq, nb, D = qbar.shape
    Hkv = kbar.shape[1]
    m = np.zeros((B, Hq, nb * (nb + 1) // 2))
    _load().stem_oracle_metric(_ptr(qbar, _c_f64p), _ptr(kbar, _c_f64p), _ptr(vnorm, _c_f64p),
                               B, Hq, Hkv, nb, D, _ptr(m, _c_f64p))
    return m


def metric_additive(qbar: np.ndarray, kbar: np.ndarray, vnorm: np.ndarray, beta: float,
                    clamp: bool = True) -> np.ndarray:
    """The pages' additive output-aware metric s_ij + beta * max(0, log n_j^2), packed like
    metric(); beta is rounded to float32 as the C boundary does."""
    qbar = np.ascontiguousarray(qbar, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    vnorm = np.ascontiguousarray(vnorm, dtype=np.float64)
    B, Hq, nb, D = qbar.shape
    Hkv = kbar.shape[1]
    m = np.zeros((B, Hq, nb * (nb + 1) // 2))
    _load().stem_oracle_metric_additive(_ptr(qbar, _c_f64p), _ptr(kbar, _c_f64p),
                                        _ptr(vnorm, _c_f64p), B, Hq, Hkv, nb, D, f32(beta),
                                        int(bool(clamp)), _ptr(m, _c_f64p))
    return m


def antidiag(q: torch.Tensor, k: torch.Tensor, block: int, stride: int,
             rows: Optional[Sequence] = None) -> np.ndarray:
    """Block probabilities estimated by anti-diagonal sampling (see stem_oracle_antidiag).

    rows=None: every query block, packed by row like metric(): [B, Hq, nb*(nb+1)/2].
    rows = [(b, h, i), ...]: [len(rows), nb], row i's p_ij in columns j <= i."""
    q, k = _host(q), _host(k)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    if stride < 1 or block % stride or S % stride:
        raise ValueError("stride must divide the block and the sequence length")
    nb = -(-S // block)
    if rows is None:
        ids = np.arange(B * Hq * nb, dtype=np.int64)
    else:
        ids = np.array([(b * Hq + h) * nb + i for (b, h, i) in rows], dtype=np.int64)
    out = np.zeros((len(ids), nb))
    if len(ids):
        _load().stem_oracle_antidiag(q.data_ptr(), k.data_ptr(), _dtype_code(q), B, Hq, Hkv, S,
                                     D, block, stride, _ptr(ids, _c_i64p), len(ids),
                                     _ptr(out, _c_f64p))
    if rows is not None:
        return out
    packed = np.zeros((B, Hq, nb * (nb + 1) // 2))
    full = out.reshape(B, Hq, nb, nb)
    for i in range(nb):
        packed[:, :, i * (i + 1) // 2:i * (i + 1) // 2 + i + 1] = full[:, :, i, :i + 1]
    return packed


def metric_from_p(p: np.ndarray, vnorm: np.ndarray, beta: float = 0.0, clamp: bool = True,
                  form: str = "product") -> np.ndarray:
    """Output-aware metric from block probabilities p [B, Hq, T] (packed rows) and the V
    magnitudes vnorm [B, Hkv, nb]: "product" m_ij = p_ij * n_j; "additive"
    M_ij = ln p_ij + beta * max(0, log n_j^2) (clamp=False drops the max; beta == 0 gives
    ln p). ln p_ij plays the part of the pooled score s_ij: within a row they differ by the
    row's log-normaliser only. Query head h reads kv-head h / (Hq/Hkv)."""
    B, Hq, T = p.shape
    Hkv, nb = vnorm.shape[1], vnorm.shape[2]
    G = Hq // Hkv
    jj = np.concatenate([np.arange(i + 1) for i in range(nb)]) if nb else np.zeros(0, int)
    n = np.repeat(vnorm, G, axis=1)[:, :, jj]  # n_j per packed entry
    if form == "product":
        return p * n
    if form != "additive":
        raise ValueError(form)
    with np.errstate(divide="ignore"):
        lp = np.log(p)
        if f32(beta) == 0.0:
            return lp
        e = 2.0 * np.log(n)
    if clamp:
        e = np.maximum(e, 0.0)
    return lp + f32(beta) * e


def metric_group(m: np.ndarray, G: int) -> np.ndarray:
    """GQA-group metric: the per-head metric summed over the G query heads that share a
    kv-head (heads g*G .. g*G+G-1), [B, Hq/G, T]. The pages are silent on GQA; this is the
    group-shared selection's score (one kept list per kv-head group)."""
    B, Hq, T = m.shape
    return m.reshape(B, Hq // G, G, T).sum(axis=2)


def select_group(mg: np.ndarray, k: np.ndarray, off: np.ndarray, G: int):
    """Selection from a group metric [B, Hkv, T], replicated to the G query heads of each
    group: sel_idx [B, Hq, cap], sel_cnt [B, Hq, nb]."""
    gi, gc = select(mg, k, off)
    return np.repeat(gi, G, axis=1), np.repeat(gc, G, axis=1)


def metric_row(m: np.ndarray, b: int, h: int, i: int) -> np.ndarray:
    """Row i (j = 0..i) of a packed metric."""
    s = i * (i + 1) // 2
    return m[b, h, s:s + i + 1]


def select(m: np.ndarray, k: np.ndarray, off: np.ndarray):
    """CSR selection: sel_idx [B, Hq, cap] and sel_cnt [B, Hq, nb] (int32)."""
    m = np.ascontiguousarray(m, dtype=np.float64)
    B, Hq, T = m.shape
    nb = len(k)
    cap = int(off[nb])
    sel_idx = np.full((B, Hq, max(cap, 1)), -1, dtype=np.int32)
    sel_cnt = np.zeros((B, Hq, nb), dtype=np.int32)
    k = np.ascontiguousarray(k, dtype=np.int32)
    off = np.ascontiguousarray(off, dtype=np.int64)
    _load().stem_oracle_select(_ptr(m, _c_f64p), _ptr(k, _c_i32p), _ptr(off, _c_i64p), B, Hq,
                               nb, cap, _ptr(sel_idx, _c_i32p), _ptr(sel_cnt, _c_i32p))
    return sel_idx[:, :, :cap], sel_cnt


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int,
              sel_idx: np.ndarray, sel_cnt: np.ndarray, off: np.ndarray,
              rows: Optional[Sequence] = None) -> np.ndarray:
    """Exact attention over the kept blocks for the listed (b, h, i) query blocks.

    Returns [len(rows), block, D] float64. rows=None means every query block,
    in (b, h, i) order.
    """
    q, k, v = _host(q), _host(k), _host(v)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    nb = -(-S // block)
    if rows is None:
        ids = np.arange(B * Hq * nb, dtype=np.int64)
    else:
        ids = np.array([(b * Hq + h) * nb + i for (b, h, i) in rows], dtype=np.int64)
    cap = int(off[nb])
    sel_idx = np.ascontiguousarray(np.asarray(sel_idx, dtype=np.int32).reshape(B, Hq, cap))
    sel_cnt = np.ascontiguousarray(np.asarray(sel_cnt, dtype=np.int32).reshape(B, Hq, nb))
    off = np.ascontiguousarray(off, dtype=np.int64)
    out = np.zeros((len(ids), block, D))
    if len(ids):
        _load().stem_oracle_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q),
                                      B, Hq, Hkv, S, D, block, _ptr(sel_idx, _c_i32p),
                                      _ptr(sel_cnt, _c_i32p), _ptr(off, _c_i64p), cap,
                                      _ptr(ids, _c_i64p), len(ids), _ptr(out, _c_f64p))
    return out


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int, rho_min: float,
            tau: float, k_min: int, rows: Optional[Sequence] = None, with_metric: bool = True,
            schedule: str = "exp", k_start: float = 0.0, mu: float = 1.0,
            metric_form: str = "product", beta: float = 0.0, clamp: bool = True,
            vsum: str = "mean", share: str = "head", score: str = "pooled", stride: int = 16):
    """All stages. Returns a dict with k, off, qbar, kbar, vnorm, m, sel_idx, sel_cnt and
    out ([len(rows), block, D] for the listed query blocks; all blocks when rows is None).
    schedule "exp" uses rho_min, tau; "linear" uses k_start, mu. metric_form "product" is
    softmax(s) * n, "additive" is s + beta * max(0, log n^2) (clamp=False drops the max).
    share "group" selects once per kv-head group by the metric summed over its query heads
    (metric_group); m is then the group metric replicated to each head. score "antidiag"
    takes the block probabilities from anti-diagonal sampling with the given stride
    (antidiag(), returned as "p") instead of the pooled softmax."""
    B, Hq, S, D = q.shape
    nb = -(-S // block)
    if schedule == "exp":
        kk, off = budget(nb, rho_min, tau, k_min)
    elif schedule == "linear":
        kk, off = budget_linear(nb, k_start, mu, k_min)
    else:
        raise ValueError(schedule)
    qbar, kbar, vnorm = pool(q, k, v, block, vsum)
    p = None
    if score == "antidiag":
        p = antidiag(q, k, block, stride)
        m = metric_from_p(p, vnorm, beta, clamp, metric_form)
    elif score != "pooled":
        raise ValueError(score)
    elif metric_form == "product":
        m = metric(qbar, kbar, vnorm)
    elif metric_form == "additive":
        m = metric_additive(qbar, kbar, vnorm, beta, clamp)
    else:
        raise ValueError(metric_form)
    if share == "group":
        G = q.shape[1] // k.shape[1]
        m = np.repeat(metric_group(m, G), G, axis=1)  # every head of a group: the group metric
        sel_idx, sel_cnt = select_group(m[:, ::G], kk, off, G)
    elif share == "head":
        sel_idx, sel_cnt = select(m, kk, off)
    else:
        raise ValueError(share)
    out = attention(q, k, v, block, sel_idx, sel_cnt, off, rows)
    res = dict(k=kk, off=off, qbar=qbar, kbar=kbar, vnorm=vnorm, sel_idx=sel_idx,
               sel_cnt=sel_cnt, out=out)
    if with_metric:
        res["m"] = m
    if p is not None:
        res["p"] = p
    return res


def row_list(sel_idx: np.ndarray, off: np.ndarray, k: np.ndarray, b: int, h: int, i: int):
    """Kept blocks of query block i of (b, h), ascending."""
    return sel_idx[b, h, off[i]:off[i] + k[i]]
