"""Comparison helpers for the CUDA path against the oracle.

Selection: counts must equal k(i) exactly and every row must be ascending, distinct, inside
[0, i] and contain 0 and i. Kept sets must equal the oracle's, except where the two differ only
by swapping blocks whose oracle metrics are within REL_TIE of each other (several selections
are then equally correct). For the product metric m = exp(key - logsumexp) that is a relative
gap; the additive metric M is itself a key, so the same gap is taken absolutely, scaled by
max(1, |M|): |M_a - M_b| <= REL_TIE * max(1, |M_a|, |M_b|).

Attention output: max-abs error <= 2e-2 and mean-abs error <= 1e-3 against the oracle's
double-precision result for bfloat16 inputs (float32 accumulation); tighter for float32 inputs.
The 2e-2 bound holds for every element whose reference is below 8 in magnitude. From 8 up a
bfloat16 output cannot be within 2e-2 of the reference at all (half a bfloat16 ulp there is
2^-5 or more, so even the exactly rounded value can miss by 0.031), and the named workloads
have such outputs (rows whose attention peaks on a x5 V row of the 128K workload reach 13): for
those elements alone the bound adds half a bfloat16 ulp of the reference, and the mean bound
the mean of those half-ulps.

Rows whose kept set differs from the oracle's by a tie swap are compared with the oracle's
attention over the GPU's own kept set (several selections are correct there, and each has its
own exact output), under the same bounds.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle

REL_TIE = 1e-6
TOL_BF16 = dict(max_abs=2e-2, mean_abs=1e-3)
TOL_F32 = dict(max_abs=2e-4, mean_abs=2e-5)


def tol_for(dtype: torch.dtype):
    return TOL_BF16 if dtype == torch.bfloat16 else TOL_F32


def compare_selection(gpu_idx, gpu_cnt, ref_idx, ref_cnt, m_ref, k, off, rel=REL_TIE,
                      additive=False):
    """Returns dict(rows, identical, tie_swaps, violations=[...])."""
    gi = np.asarray(gpu_idx.cpu() if torch.is_tensor(gpu_idx) else gpu_idx)
    gc = np.asarray(gpu_cnt.cpu() if torch.is_tensor(gpu_cnt) else gpu_cnt)
    B, Hq, nb = ref_cnt.shape
    cap = int(off[nb])
    gi = gi.reshape(B, Hq, -1)[:, :, :cap]
    gc = gc.reshape(B, Hq, -1)[:, :, :nb]
    violations = []
    if not np.array_equal(gc, ref_cnt):
        bad = np.argwhere(gc != ref_cnt)[:5]
        violations.append(f"counts differ at {bad.tolist()}")
    row_of = np.repeat(np.arange(nb), k)  # row index of every CSR slot
    diff = gi != ref_idx
    tie_swaps = 0
    rows_bad = set()
    for b, h, slot in np.argwhere(diff):
        rows_bad.add((int(b), int(h), int(row_of[slot])))
    # structure of every GPU row
    ii = row_of[None, None, :]
    if np.any(gi < 0) or np.any(gi > ii):
        violations.append("index outside [0, i]")
    starts = off[:-1]
    if np.any(gi[:, :, starts] != 0):
        violations.append("row does not start with the sink block 0")
    ends = off[1:] - 1
    if np.any(gi[:, :, ends] != np.arange(nb)[None, None, :]):
        violations.append("row does not end with the diagonal block i")
    for (b, h, i) in sorted(rows_bad):
        g = gi[b, h, off[i]:off[i + 1]]
        r = ref_idx[b, h, off[i]:off[i + 1]]
        if np.any(np.diff(g) <= 0):
            violations.append(f"row {(b, h, i)} not strictly ascending")
            continue
        extra = np.setdiff1d(g, r)
        missing = np.setdiff1d(r, g)
        mrow = oracle.metric_row(m_ref, b, h, i)
        hi = mrow[missing].max()
        lo = mrow[extra].min()
        scale = max(1.0, abs(hi), abs(lo)) if additive else hi
        if hi - lo <= rel * scale:
            tie_swaps += 1
        else:
            violations.append(f"row {(b, h, i)}: kept {extra.tolist()} over {missing.tolist()} "
                              f"(rel gap {(hi - lo) / scale:.3e})")
    return dict(rows=B * Hq * nb, identical=B * Hq * nb - len(rows_bad), tie_swaps=tie_swaps,
                violations=violations, rows_bad=sorted(rows_bad))


def out_rows(out: torch.Tensor, rows, block: int) -> np.ndarray:
    """GPU output gathered to [len(rows), block, D] float64 for the listed (b, h, i). Rows of
    a partial last block past the sequence end are 0, as in the oracle's output."""
    o = out.detach()
    pad = lambda x: torch.nn.functional.pad(x, (0, 0, 0, block - x.shape[0]))  # noqa: E731
    parts = [pad(o[b, h, i * block:(i + 1) * block]) for (b, h, i) in rows]
    if not parts:
        return np.zeros((0, block, out.shape[-1]))
    return torch.stack(parts).double().cpu().numpy()


def out_error(gpu: np.ndarray, ref: np.ndarray):
    d = np.abs(gpu - ref)
    return dict(max_abs=float(d.max()) if d.size else 0.0,
                mean_abs=float(d.mean()) if d.size else 0.0,
                max_ref=float(np.abs(ref).max()) if ref.size else 0.0)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bfloat16 ulp at |x| (8 significant bits): 2^(floor(log2|x|) - 8), for x != 0."""
    ax = np.maximum(np.abs(x), np.finfo(np.float64).tiny)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def assert_out_close(gpu: np.ndarray, ref: np.ndarray, dtype: torch.dtype, what: str = ""):
    """Max-abs and mean-abs error against the oracle, element by element.

    bfloat16: every element with |reference| < 8 within 2e-2; elements with |reference| >= 8
    within 2e-2 plus half a bfloat16 ulp of the reference (the output format's own rounding);
    mean within 1e-3 plus the mean of those half-ulps."""
    e = out_error(gpu, ref)
    t = tol_for(dtype)
    bound = np.full(ref.shape, t["max_abs"])
    mean_bound = t["mean_abs"]
    if dtype == torch.bfloat16 and ref.size:
        big = np.abs(ref) >= 8.0
        extra = np.where(big, bf16_half_ulp(ref), 0.0)
        bound = bound + extra
        mean_bound += float(extra.mean())
        err = np.abs(gpu - ref)
        e["n_ref_at_least_8"] = int(big.sum())
        e["max_abs_below_8"] = float(err[~big].max()) if (~big).any() else 0.0
        # elements that needed the format allowance (all of them at |reference| >= 8)
        e["n_above_plain_bound"] = int((err > t["max_abs"]).sum())
        e["mean_bound"] = mean_bound
        ref_b = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
        e["max_abs_vs_bf16_ref"] = float(np.abs(gpu - ref_b).max())
    worst = float(np.max(np.abs(gpu - ref) - bound)) if ref.size else 0.0
    assert worst <= 0 and e["mean_abs"] <= mean_bound, (what, e, t)
    return e


def gpu_csr(sel_idx, sel_cnt, B: int, Hq: int, nb: int, cap: int):
    """The GPU's CSR as int32 numpy arrays [B, Hq, cap] and [B, Hq, nb]."""
    gi = np.asarray(sel_idx.cpu() if torch.is_tensor(sel_idx) else sel_idx, dtype=np.int32)
    gc = np.asarray(sel_cnt.cpu() if torch.is_tensor(sel_cnt) else sel_cnt, dtype=np.int32)
    return (np.ascontiguousarray(gi.reshape(B, Hq, -1)[:, :, :cap]),
            np.ascontiguousarray(gc.reshape(B, Hq, -1)[:, :, :nb]))


def assert_prefill_out(out: torch.Tensor, cpu_inputs, block: int, ref_out: np.ndarray,
                       ref_rows, res: dict, sel_idx, sel_cnt, off, dtype: torch.dtype,
                       what: str = ""):
    """Output check of an end-to-end call. ref_out[t] is the oracle's output for ref_rows[t]
    on the oracle's selection. Rows whose GPU selection is a tie swap of the oracle's (listed
    in res["rows_bad"] by compare_selection) are instead compared with the oracle's attention
    over the GPU's own kept blocks. Returns (error on agreeing rows, error on swapped rows)."""
    swapped = set(res["rows_bad"])
    keep = [t for t, r in enumerate(ref_rows) if r not in swapped]
    e1 = assert_out_close(out_rows(out, [ref_rows[t] for t in keep], block), ref_out[keep],
                          dtype, what)
    sw = [r for r in ref_rows if r in swapped]
    e2 = None
    if sw:
        q, k, v = cpu_inputs
        B, Hq, S_, _ = q.shape
        nb = -(-S_ // block)
        gi, gc = gpu_csr(sel_idx, sel_cnt, B, Hq, nb, int(off[nb]))
        ref_sw = oracle.attention(q, k, v, block, gi, gc, off, sw)
        e2 = assert_out_close(out_rows(out, sw, block), ref_sw, dtype, what + " (tie rows)")
    return e1, e2
