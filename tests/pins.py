"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each `pin_*` function raises AssertionError on failure. They run as ordinary
CPU tests (tests/test_oracle_pins.py) and again against deliberately broken
copies of the oracle (tests/test_oracle_mutants.py), which must each fail at
least one pin.

What pins what:
  budget     arbitrary-precision (decimal, 60 digits) recomputation of the
             exponential-ratio schedule; closed forms at rho_min = 1 and tau -> 0;
             the invariants k <= i+1, k >= min(i+1, k_min), k(0) = 1, k(i >= 1) >= 2.
  pooling    closed forms: constant blocks, +x/-x alternating rows (mean of norms
             is not the norm of the mean), arithmetic-progression rows; numpy
             brute force on random tensors.
  metric     Q = 0 gives m_ij = n_j/(i+1); two-block logistic closed form; each
             row of m/n sums to 1; the ranking equals that of the pages' printed
             additive score s_ij + beta*log(n_j^2) at beta = 1/2, no clamp; numpy
             brute force.
  selection  all-equal metric keeps {0, 1, ..., k-2, i} (ties to the lower
             index); Q = 0 keeps the top norms; full-sort brute force; structural
             invariants.
  attention  rho_min = 1 equals dense causal attention from torch's
             scaled_dot_product_attention in float64; token 0 returns V[0];
             a constant-key block gives the mean of the visible V rows; dense
             token-mask brute force.
"""

from __future__ import annotations

import math
from decimal import ROUND_CEILING, Decimal, getcontext

import numpy as np
import torch

import oracle
from tests import brute

# --------------------------------------------------------------------------- helpers


def _rand(shape, gen, dtype=torch.float32):
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(dtype)


def _tiny_inputs(seed, B=1, Hq=4, Hkv=2, S=256, D=16, block=16, dtype=torch.float32,
                 sink=True, v_out=True):
    g = torch.Generator().manual_seed(seed)
    q = _rand((B, Hq, S, D), g)
    k = _rand((B, Hkv, S, D), g)
    v = _rand((B, Hkv, S, D), g)
    if sink:
        k[:, :, 0, :] *= 8.0
    if v_out:
        for b in range(B):
            for h in range(Hkv):
                rows = torch.randperm(S, generator=g)[: max(1, S // 32)]
                v[b, h, rows, :] *= 5.0
    return q.to(dtype), k.to(dtype), v.to(dtype)


def _kept_from_csr(sel_idx, sel_cnt, off, B, Hq, nb):
    out = {}
    for b in range(B):
        for h in range(Hq):
            for i in range(nb):
                out[(b, h, i)] = sel_idx[b, h, off[i]:off[i] + sel_cnt[b, h, i]].tolist()
    return out


# --------------------------------------------------------------------------- budget


def budget_decimal(nb, rho_min, tau, k_min):
    """The schedule evaluated in 60-digit decimal arithmetic from the float32
    parameter values. Returns (k list, ambiguous index set): an index is
    ambiguous when rho(i)*(i+1) is within 1e-12 of an integer, where double
    rounding could legitimately decide the ceiling either way."""
    getcontext().prec = 60
    r = Decimal(float(np.float32(rho_min)))
    t = Decimal(float(np.float32(tau)))
    ks, amb = [], set()
    for i in range(nb):
        rho = r + (1 - r) * (Decimal(-i) / t).exp()
        x = rho * (i + 1)
        c = int(x.to_integral_value(rounding=ROUND_CEILING))
        if abs(x - x.to_integral_value()) < Decimal("1e-12"):
            amb.add(i)
        k = min(i + 1, max(k_min, c))
        if i == 0:
            k = 1
        elif k < 2:
            k = 2
        ks.append(k)
    return ks, amb


BUDGET_CASES = [
    # (nb, rho_min, tau, k_min): the five workloads' parameters and extra spread
    (16, 0.25, 4.0, 2),
    (256, 0.1, 32.0, 4),
    (1024, 0.05, 64.0, 8),
    (512, 0.1, 48.0, 4),
    (1024, 0.1, 64.0, 8),
    (1024, 0.2, 64.0, 8),
    (1024, 0.5, 64.0, 8),
    (128, 0.05, 64.0, 8),
    (300, 0.7, 5.5, 1),
    (2048, 0.01, 300.0, 3),
    (64, 0.33, 0.7, 1),
    (777, 0.9, 1000.0, 17),
]


def pin_budget_decimal():
    for nb, r, t, km in BUDGET_CASES:
        k, off = oracle.budget(nb, r, t, km)
        ref, amb = budget_decimal(nb, r, t, km)
        for i in range(nb):
            if i in amb:
                continue
            assert k[i] == ref[i], (nb, r, t, km, i, k[i], ref[i])
        assert off[0] == 0 and np.all(np.diff(off) == k), "offsets are the prefix sums"


def pin_budget_closed_forms():
    # rho_min = 1: every causal block is kept.
    for nb in (1, 2, 17, 1024):
        k, off = oracle.budget(nb, 1.0, 64.0, 8)
        assert np.array_equal(k, np.arange(1, nb + 1)), "rho_min = 1 must be dense"
        assert off[nb] == nb * (nb + 1) // 2
    # tau -> 0+: rho(i) = rho_min for i >= 1.
    for rmin, km in ((0.05, 8), (0.3, 1), (0.5, 3)):
        k, _ = oracle.budget(500, rmin, 1e-30, km)
        rf = float(np.float32(rmin))
        for i in range(1, 500):
            want = min(i + 1, max(km, math.ceil(rf * (i + 1))))
            assert k[i] == max(2, want), (rmin, km, i, k[i], want)
    # invariants
    for nb, r, t, km in BUDGET_CASES:
        k, _ = oracle.budget(nb, r, t, km)
        i = np.arange(nb)
        assert k[0] == 1
        assert np.all(k <= i + 1)
        assert np.all(k >= np.minimum(i + 1, km))
        assert np.all(k[1:] >= 2)


# --------------------------------------------------------------------------- pooling


def pin_pool_closed_forms():
    B, Hq, Hkv, S, D, block = 1, 2, 1, 64, 8, 16
    nb = S // block
    g = torch.Generator().manual_seed(3)
    # constant blocks: every row of block i equals x_i
    xq = torch.randn(B, Hq, nb, D, generator=g, dtype=torch.float64)
    xk = torch.randn(B, Hkv, nb, D, generator=g, dtype=torch.float64)
    q = xq.repeat_interleave(block, dim=2).float()
    k = xk.repeat_interleave(block, dim=2).float()
    # V: rows alternate +x / -x, so the mean of the norms is |x| while the norm of the
    # mean is 0
    xv = torch.randn(B, Hkv, nb, D, generator=g, dtype=torch.float64).float()
    sign = torch.tensor([1.0, -1.0]).repeat(S // 2).view(1, 1, S, 1)
    v = xv.repeat_interleave(block, dim=2) * sign
    qbar, kbar, vnorm = oracle.pool(q, k, v, block)
    np.testing.assert_allclose(qbar, xq.float().double().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(kbar, xk.float().double().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(vnorm, torch.linalg.vector_norm(xv.double(), dim=-1).numpy(),
                               rtol=1e-12)
    # arithmetic progression along the rows: row r of each block is r * e_0 (+ block
    # offset), mean (block-1)/2
    ap = torch.zeros(B, Hq, S, D)
    ap[..., 0] = torch.arange(S, dtype=torch.float32) % block
    ap[..., 1] = torch.arange(S, dtype=torch.float32) // block
    qbar, _, _ = oracle.pool(ap, k, v, block)
    np.testing.assert_allclose(qbar[..., 0], (block - 1) / 2.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(qbar[0, 0, :, 1], np.arange(nb), rtol=0, atol=1e-12)
    # row norms r (rows r*e_3): mean norm is (block-1)/2
    vap = torch.zeros(B, Hkv, S, D)
    vap[..., 3] = torch.arange(S, dtype=torch.float32) % block
    _, _, vn = oracle.pool(q, k, vap, block)
    np.testing.assert_allclose(vn, (block - 1) / 2.0, rtol=0, atol=1e-12)


def pin_pool_brute():
    for dtype in (torch.float32, torch.bfloat16):
        q, k, v = _tiny_inputs(11, dtype=dtype)
        got = oracle.pool(q, k, v, 16)
        ref = brute.pool(q, k, v, 16)
        for a, b in zip(got, ref):
            np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------- metric


def pin_metric_closed_forms():
    B, Hq, Hkv, S, D, block = 1, 2, 1, 128, 16, 16
    nb = S // block
    q, k, v = _tiny_inputs(5, B=B, Hq=Hq, Hkv=Hkv, S=S, D=D, block=block)
    # Q = 0: uniform routing, m_ij = n_j / (i + 1)
    z = torch.zeros_like(q)
    qbar, kbar, vnorm = oracle.pool(z, k, v, block)
    m = oracle.metric(qbar, kbar, vnorm)
    for h in range(Hq):
        for i in range(nb):
            np.testing.assert_allclose(oracle.metric_row(m, 0, h, i), vnorm[0, 0, : i + 1] / (i + 1),
                                       rtol=1e-13)
    # two blocks, known logits: p_10 = logistic(s_10 - s_11)
    a, b0, b1 = 0.9, 1.7, -0.4
    q2 = torch.zeros(1, 1, 2 * block, D)
    k2 = torch.zeros(1, 1, 2 * block, D)
    v2 = torch.ones(1, 1, 2 * block, D)
    q2[..., block:, 0] = a
    k2[..., :block, 0] = b0
    k2[..., block:, 0] = b1
    qbar, kbar, vnorm = oracle.pool(q2, k2, v2, block)
    m = oracle.metric(qbar, kbar, vnorm)
    s10 = float(np.float32(a)) * float(np.float32(b0)) / math.sqrt(D)
    s11 = float(np.float32(a)) * float(np.float32(b1)) / math.sqrt(D)
    p10 = 1.0 / (1.0 + math.exp(s11 - s10))
    row = oracle.metric_row(m, 0, 0, 1)
    np.testing.assert_allclose(row, [p10 * math.sqrt(D), (1 - p10) * math.sqrt(D)], rtol=1e-13)
    # m / n sums to one per row
    qbar, kbar, vnorm = oracle.pool(q, k, v, block)
    m = oracle.metric(qbar, kbar, vnorm)
    for h in range(Hq):
        for i in range(nb):
            np.testing.assert_allclose((oracle.metric_row(m, 0, h, i) / vnorm[0, 0, : i + 1]).sum(),
                                       1.0, rtol=1e-13)


def pin_metric_additive_equivalence():
    """Within a row, ranking by p_ij * n_j equals ranking by the additive form the
    pages print, s_ij + beta*max(0, log ||V_j||^2), with beta = 1/2, the clamp
    removed and block-level quantities (||V_j|| read as the pooled norm n_j),
    because log(p_ij n_j) = s_ij - logsumexp_i + log n_j."""
    for seed in (1, 2, 3):
        q, k, v = _tiny_inputs(seed, Hq=2, Hkv=1, S=512, D=32, block=16)
        qbar, kbar, vnorm = oracle.pool(q, k, v, 16)
        m = oracle.metric(qbar, kbar, vnorm)
        nb, D = qbar.shape[2], qbar.shape[3]
        for h in range(2):
            for i in range(2, nb):
                s = qbar[0, h, i] @ kbar[0, 0, : i + 1].T / math.sqrt(D)
                add = s + 0.5 * np.log(vnorm[0, 0, : i + 1] ** 2)
                mr = oracle.metric_row(m, 0, h, i)
                o1 = np.lexsort((np.arange(i + 1), -mr))
                o2 = np.lexsort((np.arange(i + 1), -add))
                assert np.array_equal(o1, o2), (seed, h, i)


def pin_metric_brute():
    for dtype in (torch.float32, torch.bfloat16):
        q, k, v = _tiny_inputs(21, dtype=dtype, Hq=4, Hkv=2)
        qbar, kbar, vnorm = oracle.pool(q, k, v, 16)
        m = oracle.metric(qbar, kbar, vnorm)
        md = brute.metric_dense(*brute.pool(q, k, v, 16))
        B, Hq, nb, _ = md.shape
        for h in range(Hq):
            for i in range(nb):
                np.testing.assert_allclose(oracle.metric_row(m, 0, h, i), md[0, h, i, : i + 1],
                                           rtol=1e-11, atol=1e-15)


# --------------------------------------------------------------------------- selection


def pin_select_ties_and_special_cases():
    # all-equal metric (Q = 0 and every V row of norm 1): ties break to the lower index
    B, Hq, Hkv, S, D, block = 1, 2, 2, 512, 8, 16
    nb = S // block
    q = torch.zeros(B, Hq, S, D)
    g = torch.Generator().manual_seed(9)
    k = torch.randn(B, Hkv, S, D, generator=g)
    v = torch.zeros(B, Hkv, S, D)
    v[..., 2] = 1.0
    res = oracle.prefill(q, k, v, block, 0.3, 3.0, 2, rows=[])
    kk, off = res["k"], res["off"]
    for h in range(Hq):
        for i in range(nb):
            got = oracle.row_list(res["sel_idx"], off, kk, 0, h, i).tolist()
            want = [0] if i == 0 else sorted(set([0, i] + list(range(1, kk[i] - 1))))
            assert got == want, (h, i, got, want)
    # Q = 0 with distinct norms: keep the largest pooled norms
    v = torch.randn(B, Hkv, S, D, generator=g)
    res = oracle.prefill(q, k, v, block, 0.3, 3.0, 2, rows=[])
    _, _, vn = brute.pool(q, k, v, block)
    kk, off = res["k"], res["off"]
    for h in range(Hq):
        for i in range(2, nb):
            cand = np.arange(1, i)
            best = cand[np.argsort(-vn[0, h, 1:i], kind="stable")][: kk[i] - 2]
            want = sorted(set([0, i] + best.tolist()))
            assert oracle.row_list(res["sel_idx"], off, kk, 0, h, i).tolist() == want


def pin_select_brute_and_invariants():
    for seed, (Hq, Hkv) in ((4, (4, 2)), (5, (2, 2)), (6, (6, 3))):
        q, k, v = _tiny_inputs(seed, Hq=Hq, Hkv=Hkv, S=512, block=16)
        res = oracle.prefill(q, k, v, 16, 0.2, 5.0, 3, rows=[])
        kk, off = res["k"], res["off"]
        nb = 32
        md = brute.metric_dense(*brute.pool(q, k, v, 16))
        want = brute.select_rows(md, kk)
        for h in range(Hq):
            for i in range(nb):
                got = oracle.row_list(res["sel_idx"], off, kk, 0, h, i)
                assert got.tolist() == want[(0, h, i)], (seed, h, i)
                assert res["sel_cnt"][0, h, i] == kk[i]
                assert got[0] == 0 and got[-1] == i
                assert np.all(np.diff(got) > 0)


# --------------------------------------------------------------------------- attention


def _sdpa_dense(q, k, v):
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    kk = k.double().repeat_interleave(G, dim=1)
    vv = v.double().repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q.double(), kk, vv,
                                                            is_causal=True).numpy()


def pin_attention_dense_sdpa():
    for dtype, (Hq, Hkv) in ((torch.float32, (4, 2)), (torch.bfloat16, (3, 1))):
        q, k, v = _tiny_inputs(31, Hq=Hq, Hkv=Hkv, S=256, D=16, block=16, dtype=dtype)
        res = oracle.prefill(q, k, v, 16, 1.0, 8.0, 1)
        B, _, S, D = q.shape
        out = res["out"].reshape(B, Hq, S, D)
        np.testing.assert_allclose(out, _sdpa_dense(q, k, v), rtol=1e-10, atol=1e-12)


def pin_attention_closed_forms():
    q, k, v = _tiny_inputs(41, Hq=2, Hkv=1, S=128, D=8, block=16)
    res = oracle.prefill(q, k, v, 16, 0.25, 2.0, 2)
    out = res["out"].reshape(1, 2, 128, 8)
    # token 0 sees only itself
    np.testing.assert_array_equal(out[0, :, 0, :], v[0, 0, 0].double().numpy()[None, :].repeat(2, 0))
    # every key of the sequence equal: uniform weights over the visible tokens
    kc = torch.ones_like(k)
    res = oracle.prefill(q, kc, v, 16, 0.25, 2.0, 2)
    out = res["out"].reshape(1, 2, 128, 8)
    kept = _kept_from_csr(res["sel_idx"], res["sel_cnt"], res["off"], 1, 2, 8)
    V = v[0, 0].double().numpy()
    for h in range(2):
        for i in range(8):
            for r in (0, 7, 15):
                tok = i * 16 + r
                vis = [j * 16 + c for j in kept[(0, h, i)] for c in range(16) if j * 16 + c <= tok]
                np.testing.assert_allclose(out[0, h, tok], V[vis].mean(axis=0), rtol=1e-12, atol=1e-14)


def pin_attention_brute():
    for dtype in (torch.float32, torch.bfloat16):
        q, k, v = _tiny_inputs(51, Hq=4, Hkv=2, S=256, D=16, block=16, dtype=dtype)
        res = oracle.prefill(q, k, v, 16, 0.2, 3.0, 2)
        kept = _kept_from_csr(res["sel_idx"], res["sel_cnt"], res["off"], 1, 4, 16)
        ref = brute.attention_masked(q, k, v, 16, kept)
        np.testing.assert_allclose(res["out"].reshape(ref.shape), ref, rtol=1e-10, atol=1e-12)


PINS = [
    pin_budget_decimal,
    pin_budget_closed_forms,
    pin_pool_closed_forms,
    pin_pool_brute,
    pin_metric_closed_forms,
    pin_metric_additive_equivalence,
    pin_metric_brute,
    pin_select_ties_and_special_cases,
    pin_select_brute_and_invariants,
    pin_attention_dense_sdpa,
    pin_attention_closed_forms,
    pin_attention_brute,
]


def run_all() -> None:
    """Run every pin; raise on the first failure."""
    for fn in PINS:
        fn()


if __name__ == "__main__":
    run_all()
    print("all pins hold")
