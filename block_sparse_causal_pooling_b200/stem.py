"""Python binding of libstem.so (the C ABI in include/stem.h), via ctypes.

Argument marshalling only: every step of the path runs in the library's CUDA kernels. The
binding allocates outputs and the workspace with torch when the caller does not pass them,
reads device pointers and the current CUDA stream from torch, and raises StemError on a
non-zero return code. There is no fallback: if libstem.so is missing or cannot be loaded,
importing this module raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libstem.so")

STEM_OK = 0
STEM_ERR_ARG = -1
STEM_ERR_WORKSPACE = -2
STEM_ERR_CUDA = -3
STEM_ERR_TIMEOUT = -4
STEM_ERR_UNSUPPORTED = -5
STEM_BF16 = 0
STEM_F32 = 1
STEM_MAX_NB = 4096
STEM_SCHED_EXP = 0
STEM_SCHED_LINEAR = 1
STEM_METRIC_PRODUCT = 0
STEM_METRIC_ADDITIVE = 1
STEM_VSUM_MEAN = 0
STEM_VSUM_MAX = 1
STEM_SHARE_HEAD = 0
STEM_SHARE_GROUP = 1
STEM_SCORE_POOLED = 0
STEM_SCORE_ANTIDIAG = 1


class StemError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


class stem_method_t(ctypes.Structure):
    _fields_ = [
        ("schedule", ctypes.c_int32), ("rho_min", ctypes.c_float), ("tau", ctypes.c_float),
        ("k_start", ctypes.c_float), ("mu", ctypes.c_float), ("k_min", ctypes.c_int32),
        ("metric", ctypes.c_int32), ("beta", ctypes.c_float), ("clamp", ctypes.c_int32),
        ("vsum", ctypes.c_int32), ("share", ctypes.c_int32),
        ("score", ctypes.c_int32), ("stride", ctypes.c_int32),
    ]


def make_method(schedule: str = "exp", rho_min: float = 1.0, tau: float = 1.0,
                k_start: float = 1.0, mu: float = 1.0, k_min: int = 1, metric: str = "product",
                beta: float = 0.0, clamp: bool = True, vsum: str = "mean",
                share: str = "head", score: str = "pooled", stride: int = 16) -> stem_method_t:
    """Method parameters (stem_method_t): schedule "exp" (rho_min, tau) or "linear" (k_start,
    mu); metric "product" or "additive" (beta, clamp); vsum "mean" or "max"; share "head" or
    "group" (one selection per kv-head group); score "pooled" or "antidiag" (block
    probabilities by anti-diagonal sampling with groups of `stride` tokens)."""
    m = stem_method_t()
    m.schedule = {"exp": STEM_SCHED_EXP, "linear": STEM_SCHED_LINEAR}[schedule]
    m.rho_min, m.tau, m.k_start, m.mu, m.k_min = rho_min, tau, k_start, mu, k_min
    m.metric = {"product": STEM_METRIC_PRODUCT, "additive": STEM_METRIC_ADDITIVE}[metric]
    m.beta, m.clamp = beta, int(bool(clamp))
    m.vsum = {"mean": STEM_VSUM_MEAN, "max": STEM_VSUM_MAX}[vsum]
    m.share = {"head": STEM_SHARE_HEAD, "group": STEM_SHARE_GROUP}[share]
    m.score = {"pooled": STEM_SCORE_POOLED, "antidiag": STEM_SCORE_ANTIDIAG}[score]
    m.stride = stride
    return m


class stem_args_t(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("S", ctypes.c_int32), ("D", ctypes.c_int32), ("block", ctypes.c_int32),
        ("rho_min", ctypes.c_float), ("tau", ctypes.c_float), ("k_min", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("out", ctypes.c_void_p), ("sel_idx", ctypes.c_void_p), ("sel_cnt", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("status", ctypes.c_void_p),
        ("events", ctypes.POINTER(ctypes.c_void_p)),
        ("method", ctypes.POINTER(stem_method_t)),
    ]


class stem_varlen_args_t(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("nseq", ctypes.c_int32), ("cu_seqlens", ctypes.POINTER(ctypes.c_int32)),
        ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
        ("block", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("method", ctypes.POINTER(stem_method_t)),
        ("out", ctypes.c_void_p), ("sel_idx", ctypes.c_void_p), ("sel_cnt", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("status", ctypes.c_void_p),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m block_sparse_causal_pooling_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    M = ctypes.POINTER(stem_method_t)
    sig = {
        "stem_prefill": (I, [P, P, P, I, I, I, I, I, I, F, F, I, P, P, P]),
        "stem_prefill_ex": (I, [ctypes.POINTER(stem_args_t), P]),
        "stem_prefill_host": (I, [ctypes.POINTER(stem_args_t)]),
        "stem_budget": (I, [I, F, F, I, P, P]),
        "stem_sel_capacity": (ctypes.c_int64, [I, F, F, I]),
        "stem_workspace_size": (Z, [I, I, I, I, I, I]),
        "stem_strerror": (ctypes.c_char_p, [I]),
        "stem_pool": (I, [P, P, P, I, I, I, I, I, I, I, P, P, P, P]),
        "stem_select": (I, [P, P, P, I, I, I, I, I, F, F, I, P, P, P, P, Z, P]),
        "stem_sparse_attn": (I, [P, P, P, I, I, I, I, I, I, I, F, F, I, P, P, P, P, Z, P, P]),
        "stem_select_static": (I, [P, P, P, I, I, I, I, I, F, F, I, P, P, P]),
        "stem_budget_m": (I, [I, M, P, P]),
        "stem_sel_capacity_m": (ctypes.c_int64, [I, M]),
        "stem_pool_m": (I, [P, P, P, I, I, I, I, I, I, I, M, P, P, P, P]),
        "stem_select_m": (I, [P, P, P, I, I, I, I, I, M, P, P, P, P, Z, P]),
        "stem_sparse_attn_m": (I, [P, P, P, I, I, I, I, I, I, I, M, P, P, P, P, Z, P, P]),
        "stem_test_withhold_q": (I, [I]),
        "stem_prefill_varlen": (I, [ctypes.POINTER(stem_varlen_args_t), P]),
        "stem_varlen_workspace_size": (Z, [I, ctypes.POINTER(ctypes.c_int32), I, I, I, I]),
        "stem_varlen_sel_capacity": (ctypes.c_int64, [I, ctypes.POINTER(ctypes.c_int32), I, M]),
        "stem_workspace_size_m": (Z, [I, I, I, I, I, I, M]),
        "stem_antidiag_m": (I, [P, P, I, I, I, I, I, I, I, M, P, P, Z, P, P]),
        "stem_select_p_m": (I, [P, P, I, I, I, I, M, P, P, P, P, Z, P]),
        "stem_varlen_workspace_size_m": (Z, [I, ctypes.POINTER(ctypes.c_int32), I, I, I, I, M]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()

# Every symbol include/stem.h declares.
EXPORTED = ("stem_prefill", "stem_prefill_ex", "stem_prefill_host", "stem_budget",
            "stem_sel_capacity", "stem_workspace_size", "stem_strerror", "stem_pool",
            "stem_select", "stem_sparse_attn", "stem_budget_m", "stem_sel_capacity_m",
            "stem_pool_m", "stem_select_m", "stem_sparse_attn_m", "stem_prefill_varlen",
            "stem_varlen_workspace_size", "stem_varlen_sel_capacity", "stem_select_static",
            "stem_test_withhold_q", "stem_workspace_size_m", "stem_antidiag_m", "stem_select_p_m",
            "stem_varlen_workspace_size_m")


def lib() -> ctypes.CDLL:
    return _lib


def strerror(code: int) -> str:
    return _lib.stem_strerror(int(code)).decode()


def _check(rc: int, where: str) -> None:
    if rc != STEM_OK:
        raise StemError(rc, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return STEM_BF16
    if t.dtype == torch.float32:
        return STEM_F32
    raise TypeError(f"inputs must be bfloat16 or float32, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------ host-only helpers


def stem_budget(nb: int, rho_min: float, tau: float, k_min: int):
    """(k [nb] int32, off [nb+1] int32) of the position-decay budget (host)."""
    k = torch.zeros(max(nb, 1), dtype=torch.int32)
    off = torch.zeros(nb + 1, dtype=torch.int32)
    _check(_lib.stem_budget(nb, rho_min, tau, k_min, _ptr(k), _ptr(off)), "stem_budget")
    return k[:nb].clone(), off


def stem_sel_capacity(nb: int, rho_min: float, tau: float, k_min: int, method=None) -> int:
    if method is not None:
        cap = int(_lib.stem_sel_capacity_m(nb, ctypes.byref(method)))
    else:
        cap = int(_lib.stem_sel_capacity(nb, rho_min, tau, k_min))
    if cap < 0:
        raise StemError(cap, "stem_sel_capacity")
    return cap


def stem_budget_m(nb: int, method: stem_method_t):
    """(k [nb] int32, off [nb+1] int32) of the budget of `method` (host)."""
    k = torch.zeros(max(nb, 1), dtype=torch.int32)
    off = torch.zeros(nb + 1, dtype=torch.int32)
    _check(_lib.stem_budget_m(nb, ctypes.byref(method), _ptr(k), _ptr(off)), "stem_budget_m")
    return k[:nb].clone(), off


def stem_workspace_size(B: int, Hq: int, Hkv: int, S: int, D: int, block: int,
                        method=None) -> int:
    if method is not None:
        return int(_lib.stem_workspace_size_m(B, Hq, Hkv, S, D, block, ctypes.byref(method)))
    return int(_lib.stem_workspace_size(B, Hq, Hkv, S, D, block))


# ------------------------------------------------------------------ device calls


def _shape(q: torch.Tensor, k: torch.Tensor):
    B, Hq, S, D = q.shape
    return B, Hq, k.shape[1], S, D


def alloc_outputs(q: torch.Tensor, k: torch.Tensor, block: int, rho_min: float, tau: float,
                  k_min: int, method=None):
    """(out, sel_idx, sel_cnt) allocated on q's device."""
    B, Hq, Hkv, S, D = _shape(q, k)
    nb = -(-S // block)  # a partial last block counts
    cap = stem_sel_capacity(nb, rho_min, tau, k_min, method)
    out = torch.empty_like(q)
    sel_idx = torch.empty((B, Hq, max(cap, 1)), dtype=torch.int32, device=q.device)
    sel_cnt = torch.empty((B, Hq, max(nb, 1)), dtype=torch.int32, device=q.device)
    return out, sel_idx, sel_cnt


def alloc_workspace(q: torch.Tensor, k: torch.Tensor, block: int, method=None) -> torch.Tensor:
    B, Hq, Hkv, S, D = _shape(q, k)
    n = stem_workspace_size(B, Hq, Hkv, S, D, block, method)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)


def make_args(q, k, v, block, rho_min, tau, k_min, out, sel_idx, sel_cnt, workspace=None,
              status=None, events=None, method=None) -> stem_args_t:
    B, Hq, Hkv, S, D = _shape(q, k)
    a = stem_args_t()
    a.q, a.k, a.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    a.B, a.Hq, a.Hkv, a.S, a.D, a.block = B, Hq, Hkv, S, D, block
    a.rho_min, a.tau, a.k_min = rho_min, tau, k_min
    a.dtype = _dtype_code(q)
    a.out, a.sel_idx, a.sel_cnt = out.data_ptr(), sel_idx.data_ptr(), sel_cnt.data_ptr()
    if workspace is not None:
        a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel()
    if status is not None:
        a.status = status.data_ptr()
    if events is not None:  # 4 cudaEvent_t handles (ints) or torch.cuda.Event objects
        arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(getattr(e, "cuda_event", e))
                                      for e in events])
        a._events_keepalive = arr
        a.events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    if method is not None:
        a._method_keepalive = method
        a.method = ctypes.pointer(method)
    return a


def stem_prefill_ex(q, k, v, block, rho_min, tau, k_min, out=None, sel_idx=None, sel_cnt=None,
                    workspace=None, status=None, stream=None, events=None, method=None):
    """Whole path on device tensors [B,H,S,D] (bf16 or f32). Returns (out, sel_idx, sel_cnt).
    Asynchronous on `stream` (default: torch's current stream). `events`: optional four
    torch.cuda.Event recorded before pooling, selection, attention and after attention.
    `method`: optional stem_method_t (make_method); it replaces rho_min, tau and k_min."""
    if out is None or sel_idx is None or sel_cnt is None:
        out, sel_idx, sel_cnt = alloc_outputs(q, k, block, rho_min, tau, k_min, method)
    if workspace is None:
        workspace = alloc_workspace(q, k, block, method)
    a = make_args(q, k, v, block, rho_min, tau, k_min, out, sel_idx, sel_cnt, workspace, status,
                  events, method)
    _check(_lib.stem_prefill_ex(ctypes.byref(a), _stream(stream)), "stem_prefill_ex")
    return out, sel_idx, sel_cnt


def stem_prefill(q, k, v, block, rho_min, tau, k_min, out=None, sel_idx=None, sel_cnt=None):
    """Whole path, bf16 device tensors, the legacy default stream, the library's own workspace."""
    if out is None or sel_idx is None or sel_cnt is None:
        out, sel_idx, sel_cnt = alloc_outputs(q, k, block, rho_min, tau, k_min)
    B, Hq, Hkv, S, D = _shape(q, k)
    _check(_lib.stem_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Hq, Hkv, S, D, block,
                             rho_min, tau, k_min, out.data_ptr(), sel_idx.data_ptr(),
                             sel_cnt.data_ptr()), "stem_prefill")
    return out, sel_idx, sel_cnt


def stem_prefill_host(q, k, v, block, rho_min, tau, k_min, out, sel_idx, sel_cnt,
                      method=None) -> None:
    """Whole path on HOST tensors (pinned for speed); synchronous."""
    a = make_args(q, k, v, block, rho_min, tau, k_min, out, sel_idx, sel_cnt, method=method)
    _check(_lib.stem_prefill_host(ctypes.byref(a)), "stem_prefill_host")


def stem_pool(q, k, v, block, qbar=None, kbar=None, vnorm=None, stream=None, method=None):
    B, Hq, Hkv, S, D = _shape(q, k)
    nb = -(-S // block)  # a partial last block counts
    dev = q.device
    if qbar is None:
        qbar = torch.empty((B, Hq, nb, D), dtype=torch.float32, device=dev)
        kbar = torch.empty((B, Hkv, nb, D), dtype=torch.float32, device=dev)
        vnorm = torch.empty((B, Hkv, nb), dtype=torch.float32, device=dev)
    if method is not None:
        _check(_lib.stem_pool_m(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, Hq,
                                Hkv, S, D, block, ctypes.byref(method), qbar.data_ptr(),
                                kbar.data_ptr(), vnorm.data_ptr(), _stream(stream)), "stem_pool_m")
        return qbar, kbar, vnorm
    _check(_lib.stem_pool(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, Hq, Hkv,
                          S, D, block, qbar.data_ptr(), kbar.data_ptr(), vnorm.data_ptr(),
                          _stream(stream)), "stem_pool")
    return qbar, kbar, vnorm


def stem_select(qbar, kbar, vnorm, rho_min, tau, k_min, with_metric=False, workspace=None,
                sel_idx=None, sel_cnt=None, stream=None, method=None):
    """CSR selection from pooled summaries (float32 device tensors). Returns (sel_idx, sel_cnt,
    m or None)."""
    B, Hq, nb, D = qbar.shape
    Hkv = kbar.shape[1]
    dev = qbar.device
    cap = stem_sel_capacity(nb, rho_min, tau, k_min, method)
    if sel_idx is None:
        sel_idx = torch.empty((B, Hq, max(cap, 1)), dtype=torch.int32, device=dev)
        sel_cnt = torch.empty((B, Hq, max(nb, 1)), dtype=torch.int32, device=dev)
    m = (torch.empty((B, Hq, nb * (nb + 1) // 2), dtype=torch.float32, device=dev)
         if with_metric else None)
    if workspace is None:
        workspace = torch.empty(max(stem_workspace_size(B, Hq, Hkv, nb * 64, D, 64), 256),
                                dtype=torch.uint8, device=dev)
    if method is not None:
        _check(_lib.stem_select_m(qbar.data_ptr(), kbar.data_ptr(), vnorm.data_ptr(), B, Hq, Hkv,
                                  nb, D, ctypes.byref(method), sel_idx.data_ptr(),
                                  sel_cnt.data_ptr(), _ptr(m), workspace.data_ptr(),
                                  workspace.numel(), _stream(stream)), "stem_select_m")
        return sel_idx, sel_cnt, m
    _check(_lib.stem_select(qbar.data_ptr(), kbar.data_ptr(), vnorm.data_ptr(), B, Hq, Hkv, nb,
                            D, rho_min, tau, k_min, sel_idx.data_ptr(), sel_cnt.data_ptr(),
                            _ptr(m), workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "stem_select")
    return sel_idx, sel_cnt, m


def stem_sparse_attn(q, k, v, block, rho_min, tau, k_min, sel_idx, sel_cnt, out=None,
                     workspace=None, status=None, stream=None, method=None):
    B, Hq, Hkv, S, D = _shape(q, k)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(q, k, block)
    if method is not None:
        _check(_lib.stem_sparse_attn_m(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q),
                                       B, Hq, Hkv, S, D, block, ctypes.byref(method),
                                       sel_idx.data_ptr(), sel_cnt.data_ptr(), out.data_ptr(),
                                       workspace.data_ptr(), workspace.numel(), _ptr(status),
                                       _stream(stream)), "stem_sparse_attn_m")
        return out
    _check(_lib.stem_sparse_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, Hq,
                                 Hkv, S, D, block, rho_min, tau, k_min, sel_idx.data_ptr(),
                                 sel_cnt.data_ptr(), out.data_ptr(), workspace.data_ptr(),
                                 workspace.numel(), _ptr(status), _stream(stream)),
           "stem_sparse_attn")
    return out


def stem_antidiag(q, k, block, method, p=None, workspace=None, status=None, stream=None):
    """Block probabilities by anti-diagonal sampling (bf16 device tensors; groups of
    method.stride tokens). Returns p [B, Hq, nb*(nb+1)/2] float32, row i at i*(i+1)/2."""
    B, Hq, Hkv, S, D = _shape(q, k)
    nb = -(-S // block)
    if p is None:
        p = torch.empty((B, Hq, max(nb * (nb + 1) // 2, 1)), dtype=torch.float32, device=q.device)
    if workspace is None:
        m = stem_method_t.from_buffer_copy(method)
        m.score = STEM_SCORE_ANTIDIAG
        workspace = alloc_workspace(q, k, block, m)
    _check(_lib.stem_antidiag_m(q.data_ptr(), k.data_ptr(), _dtype_code(q), B, Hq, Hkv, S, D,
                                block, ctypes.byref(method), p.data_ptr(), workspace.data_ptr(),
                                workspace.numel(), _ptr(status), _stream(stream)),
           "stem_antidiag_m")
    return p


def stem_select_p(p, vnorm, Hq, method, with_metric=False, workspace=None, sel_idx=None,
                  sel_cnt=None, stream=None):
    """CSR selection from block probabilities p [B, Hq, T] and V magnitudes vnorm [B, Hkv, nb]
    (float32 device tensors). Returns (sel_idx, sel_cnt, m or None)."""
    B, Hkv, nb = vnorm.shape
    dev = p.device
    cap = stem_sel_capacity(nb, 1.0, 1.0, 1, method)
    if sel_idx is None:
        sel_idx = torch.empty((B, Hq, max(cap, 1)), dtype=torch.int32, device=dev)
        sel_cnt = torch.empty((B, Hq, max(nb, 1)), dtype=torch.int32, device=dev)
    m = (torch.empty((B, Hq, nb * (nb + 1) // 2), dtype=torch.float32, device=dev)
         if with_metric else None)
    if workspace is None:
        workspace = torch.empty(max(stem_workspace_size(B, Hq, Hkv, nb * 64, 64, 64), 256),
                                dtype=torch.uint8, device=dev)
    _check(_lib.stem_select_p_m(p.data_ptr(), vnorm.data_ptr(), B, Hq, Hkv, nb,
                                ctypes.byref(method), sel_idx.data_ptr(), sel_cnt.data_ptr(),
                                _ptr(m), workspace.data_ptr(), workspace.numel(),
                                _stream(stream)), "stem_select_p_m")
    return sel_idx, sel_cnt, m


def stem_select_static(qbar, kbar, vnorm, rho_min, tau, k_min, sel_idx=None, sel_cnt=None,
                       stream=None):
    """stem_select without a workspace or any device allocation by the library: its scratch
    (the budget plan) sits in a fixed device array inside libstem.so. For callers that cannot
    allocate device memory. Calls that overlap on the GPU race on that array."""
    B, Hq, nb, D = qbar.shape
    Hkv = kbar.shape[1]
    if sel_idx is None:
        cap = stem_sel_capacity(nb, rho_min, tau, k_min)
        sel_idx = torch.empty((B, Hq, max(cap, 1)), dtype=torch.int32, device=qbar.device)
        sel_cnt = torch.empty((B, Hq, max(nb, 1)), dtype=torch.int32, device=qbar.device)
    _check(_lib.stem_select_static(qbar.data_ptr(), kbar.data_ptr(), vnorm.data_ptr(), B, Hq,
                                   Hkv, nb, D, rho_min, tau, k_min, sel_idx.data_ptr(),
                                   sel_cnt.data_ptr(), _stream(stream)), "stem_select_static")
    return sel_idx, sel_cnt


# ------------------------------------------------------------------ variable-length batches


def _cu_array(cu_seqlens):
    cu = [int(x) for x in cu_seqlens]
    return (ctypes.c_int32 * len(cu))(*cu), len(cu) - 1


def pack_varlen(seqs):
    """Pack per-sequence [H, S_s, D] tensors back to back (the varlen layout)."""
    return torch.cat([t.reshape(-1) for t in seqs]), [0] + list(
        __import__("itertools").accumulate(t.shape[-2] for t in seqs))


def stem_varlen_sel_capacity(cu_seqlens, block, method) -> int:
    arr, n = _cu_array(cu_seqlens)
    cap = int(_lib.stem_varlen_sel_capacity(n, arr, block, ctypes.byref(method)))
    if cap < 0:
        raise StemError(cap, "stem_varlen_sel_capacity")
    return cap


def stem_prefill_varlen(q, k, v, cu_seqlens, Hq, Hkv, D, block, method, out=None, sel_idx=None,
                        sel_cnt=None, workspace=None, status=None, stream=None):
    """Variable-length batch on device tensors in the packed layout (pack_varlen): returns
    (out, sel_idx [Hq * total cap], sel_cnt [Hq * total nb]) as flat tensors."""
    arr, n = _cu_array(cu_seqlens)
    dev = q.device
    cap = stem_varlen_sel_capacity(cu_seqlens, block, method)
    nbt = sum(-(-(int(cu_seqlens[s + 1]) - int(cu_seqlens[s])) // block) for s in range(n))
    if out is None:
        out = torch.empty_like(q)
        sel_idx = torch.empty(max(Hq * cap, 1), dtype=torch.int32, device=dev)
        sel_cnt = torch.empty(max(Hq * nbt, 1), dtype=torch.int32, device=dev)
    if workspace is None:
        nbytes = int(_lib.stem_varlen_workspace_size_m(n, arr, Hq, Hkv, D, block,
                                                       ctypes.byref(method)))
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    a = stem_varlen_args_t()
    a.q, a.k, a.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    a.nseq, a.cu_seqlens = n, arr
    a.Hq, a.Hkv, a.D, a.block, a.dtype = Hq, Hkv, D, block, _dtype_code(q)
    a.method = ctypes.pointer(method)
    a.out, a.sel_idx, a.sel_cnt = out.data_ptr(), sel_idx.data_ptr(), sel_cnt.data_ptr()
    a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel()
    if status is not None:
        a.status = status.data_ptr()
    _check(_lib.stem_prefill_varlen(ctypes.byref(a), _stream(stream)), "stem_prefill_varlen")
    return out, sel_idx, sel_cnt
