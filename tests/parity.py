"""Comparison helpers for the CUDA path against the oracle.

Selection: counts must equal k(i) exactly and every row must be ascending, distinct, inside
[0, i] and contain 0 and i. Kept sets must equal the oracle's, except where the two differ only
by swapping blocks whose oracle metrics are within REL_TIE of each other (several selections
are then equally correct). For the product metric m = exp(key - logsumexp) that is a relative
gap; the additive metric M is itself a key, so the same gap is taken absolutely, scaled by
max(1, |M|): |M_a - M_b| <= REL_TIE * max(1, |M_a|, |M_b|).

Attention output: max-abs error <= 2e-2 and mean-abs error <= 1e-3 against the oracle's
double-precision result for bfloat16 inputs (float32 accumulation); tighter for float32 inputs.
For bfloat16 the per-element max-abs bound grows as 2^-7 |reference| above |reference| = 2.56
(the bfloat16 rounding of P and of the output; see assert_out_close), and the mean-abs bound by
the mean of 2^-8 |reference| over those elements.
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


def assert_out_close(gpu: np.ndarray, ref: np.ndarray, dtype: torch.dtype, what: str = ""):
    """Max-abs and mean-abs error against the oracle. For bfloat16 the per-element bound is
    max(max_abs, 2^-7 |reference|): P enters P V rounded to bfloat16 (relative error <= 2^-9)
    and the output is rounded to bfloat16 (<= 2^-8 relative), so where one key dominates a
    large output the error of any such kernel approaches 2^-7 |out|. Up to |out| = 2.56 the
    bound is max_abs itself."""
    e = out_error(gpu, ref)
    t = tol_for(dtype)
    bound = t["max_abs"]
    if dtype == torch.bfloat16 and ref.size:
        bound = np.maximum(t["max_abs"], np.abs(ref) * 2.0 ** -7)
        e["n_bound_above_max_abs"] = int((np.abs(ref) * 2.0 ** -7 > t["max_abs"]).sum())
        # reported, not asserted: the error against the oracle rounded to bf16 (what an exact
        # bf16 kernel would return) and how many outputs exceed 8 in magnitude (where a bf16
        # half-ulp alone is 0.031)
        ref_b = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
        e["max_abs_vs_bf16_ref"] = float(np.abs(gpu - ref_b).max())
        e["n_ref_above_8"] = int((np.abs(ref) > 8).sum())
    worst = float(np.max(np.abs(gpu - ref) - bound)) if ref.size else 0.0
    # the mean bound grows the same way: elements above |reference| = 2.56 add their own share
    # of the bf16 rounding, 2^-8 |reference| each (0 for the named workloads, whose outputs stay
    # below 2.56)
    mean_bound = t["mean_abs"]
    if dtype == torch.bfloat16 and ref.size:
        big = np.abs(ref) > 2.56
        mean_bound += float((np.abs(ref) * 2.0 ** -8 * big).mean())
        e["mean_bound"] = mean_bound
    assert worst <= 0 and e["mean_abs"] <= mean_bound, (what, e, t)
    return e
