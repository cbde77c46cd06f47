"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each `pin_*` function raises AssertionError on failure. They run as ordinary
CPU tests (tests/test_oracle_pins.py) and again against deliberately broken
copies of the oracle (tests/test_oracle_mutants.py), which must each fail at
least one pin.

What pins what:
  budget     arbitrary-precision (decimal, 60 digits) recomputation of the
             exponential-ratio schedule; closed forms at rho_min = 1 and tau -> 0;
             the invariants k <= i+1, k >= min(i+1, k_min), k(0) = 1, k(i >= 1) >= 2.
             Linear schedule: two cases worked by hand (tests/golden/
             budget_linear_hand.txt); mu = 1 is a constant budget; the last block
             gets ceil(mu * k_start); the unclamped budget never grows with i;
             exact rational recomputation.
  pooling    closed forms: constant blocks, +x/-x alternating rows (mean of norms
             is not the norm of the mean), arithmetic-progression rows; numpy
             brute force on random tensors. Max-pooled V: rows of norm r give
             block-1; numpy brute force.
  metric     Q = 0 gives m_ij = n_j/(i+1); two-block logistic closed form; each
             row of m/n sums to 1; the ranking equals that of the pages' printed
             additive score s_ij + beta*log(n_j^2) at beta = 1/2, no clamp; numpy
             brute force. Additive metric: beta = 0 gives the numpy scores; at
             beta = 1/2 without the clamp, M_ij - log m_ij equals the row's
             logsumexp (scipy); constant-norm blocks give the clamp's known values.
  selection  all-equal metric keeps {0, 1, ..., k-2, i} (ties to the lower
             index); Q = 0 keeps the top norms; full-sort brute force; structural
             invariants.
  attention  rho_min = 1 equals dense causal attention from torch's
             scaled_dot_product_attention in float64; token 0 returns V[0];
             a constant-key block gives the mean of the visible V rows; dense
             token-mask brute force.
  group      GQA-group-shared selection: G = 1 is the per-head selection; query heads
             that are all equal give the per-head selection of any of them; the full
             sort of the numpy brute-force metric summed over the group's heads; the
             additive form sums to sum_h s + G*beta*e.
  antidiag   block probabilities by anti-diagonal sampling: two cases worked by hand
             (tests/golden/antidiag_hand.txt); the samples picked by index out of the full
             numpy logit matrix (brute force); stride 1 is the block mass of exact causal
             attention (torch softmax in float64); stride = block with keys constant per
             block is the pooled softmax; rows sum to 1; a prefix gives the same rows. The
             metric from p: the product form in the pooled limit equals the pooled metric,
             the additive form at beta = 1/2 without the clamp is the log of the product.
  ragged S   S % block != 0: pooling and attention against the slicing / token-mask
             brute force; a partial block of constant rows pools to that row; the
             full blocks do not depend on the tokens past them (a prefix of the
             sequence gives the same pooled values, selection and outputs).
"""

from __future__ import annotations

import math
import os
from decimal import ROUND_CEILING, Decimal, getcontext
from fractions import Fraction

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


def _hand_linear_cases():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                        "budget_linear_hand.txt")
    cases = []
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        head, ks = line.split(":")
        nb, ks0, mu, km = head.split()
        cases.append((int(nb), float(ks0), float(mu), int(km), [int(x) for x in ks.split()]))
    return cases


def budget_linear_exact(nb, k_start, mu, k_min):
    """Exact rational k(i) of the linear schedule from the float32-rounded parameters, and the
    blocks whose unrounded budget lies within 1e-9 of an integer (where double rounding
    could fall either way)."""
    ksf = Fraction(float(np.float32(k_start)))
    muf = Fraction(float(np.float32(mu)))
    ks, amb = [], set()
    for i in range(nb):
        t = Fraction(i, nb - 1) if nb > 1 else Fraction(0)
        lin = ksf * (1 - (1 - muf) * t)
        c = math.ceil(lin)
        if abs(lin - round(lin)) < Fraction(1, 10 ** 9):
            amb.add(i)
        kk = min(i + 1, max(k_min, c))
        ks.append(1 if i == 0 else max(2, kk))
    return ks, amb


def pin_budget_linear():
    for nb, ks0, mu, km, want in _hand_linear_cases():
        k, off = oracle.budget_linear(nb, ks0, mu, km)
        assert list(k) == want, (nb, ks0, mu, km, list(k), want)
        assert off[nb] == sum(want)
    # mu = 1: a constant budget ceil(k_start), floored and capped as usual
    for nb, ks0, km in ((64, 9.5, 1), (300, 40.0, 8), (17, 3.2, 5)):
        k, _ = oracle.budget_linear(nb, ks0, 1.0, km)
        for i in range(1, nb):
            assert k[i] == max(2, min(i + 1, max(km, math.ceil(ks0)))), (nb, ks0, km, i)
    # the last block gets ceil(mu * k_start) (values chosen away from integers)
    for nb, ks0, mu in ((1024, 36.0, 0.7), (512, 50.0, 0.35), (100, 90.0, 0.123)):
        k, _ = oracle.budget_linear(nb, ks0, mu, 1)
        assert k[nb - 1] == max(2, math.ceil(ks0 * mu)), (nb, ks0, mu, k[nb - 1])
    # exact recomputation and the invariants
    for nb, ks0, mu, km in ((1024, 36.0, 0.7, 8), (256, 20.0, 0.5, 4), (1000, 700.0, 0.05, 1),
                            (2, 5.0, 0.2, 1), (1, 4.0, 0.7, 1)):
        k, off = oracle.budget_linear(nb, ks0, mu, km)
        ref, amb = budget_linear_exact(nb, ks0, mu, km)
        for i in range(nb):
            if i not in amb:
                assert k[i] == ref[i], (nb, ks0, mu, km, i, k[i], ref[i])
        i = np.arange(nb)
        assert k[0] == 1 and np.all(k <= i + 1) and np.all(k >= np.minimum(i + 1, km))
        assert np.all(k[1:] >= 2) and off[0] == 0 and np.all(np.diff(off) == k)
        # where neither the floor nor the cap binds, the budget never grows with i
        free = [j for j in range(1, nb) if k[j] < j + 1 and k[j] > max(km, 2)]
        for a_, b_ in zip(free, free[1:]):
            assert k[b_] <= k[a_], (nb, ks0, mu, km, a_, b_)


# --------------------------------------------------------------------------- pooling


def pin_pool_max():
    B, Hkv, S, D, block = 1, 2, 64, 8, 16
    # row r of each block is r * e_3: largest norm block - 1
    z = torch.zeros(B, Hkv, S, D)
    vap = torch.zeros(B, Hkv, S, D)
    vap[..., 3] = torch.arange(S, dtype=torch.float32) % block
    _, _, vn = oracle.pool(z, z, vap, block, "max")
    np.testing.assert_allclose(vn, block - 1.0, rtol=0, atol=1e-12)
    # random rows against numpy; pooled Q and K do not depend on the V summary
    for dtype in (torch.float32, torch.bfloat16):
        q, k, v = _tiny_inputs(13, dtype=dtype)
        qb1, kb1, _ = oracle.pool(q, k, v, 16)
        qb2, kb2, vn2 = oracle.pool(q, k, v, 16, "max")
        V = brute.f64(v)
        B_, Hkv_, S_, D_ = V.shape
        want = np.linalg.norm(V, axis=-1).reshape(B_, Hkv_, S_ // 16, 16).max(axis=3)
        np.testing.assert_allclose(vn2, want, rtol=1e-13)
        assert np.array_equal(qb1, qb2) and np.array_equal(kb1, kb2)


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


def pin_metric_additive_closed_forms():
    from scipy.special import logsumexp
    q, k, v = _tiny_inputs(31, Hq=4, Hkv=2, S=512, D=32, block=16)
    qbar, kbar, vnorm = oracle.pool(q, k, v, 16)
    B, Hq, nb, D = qbar.shape
    G = Hq // kbar.shape[1]
    # beta = 0: the routing score alone, from numpy
    m0 = oracle.metric_additive(qbar, kbar, vnorm, 0.0, True)
    for h in range(Hq):
        for i in range(nb):
            s = qbar[0, h, i] @ kbar[0, h // G, : i + 1].T / math.sqrt(D)
            np.testing.assert_allclose(oracle.metric_row(m0, 0, h, i), s, rtol=1e-12, atol=1e-14)
    # beta = 1/2, no clamp: M_ij - log(m_ij) is the row's logsumexp of s (product metric pinned
    # above; logsumexp from scipy)
    mh = oracle.metric_additive(qbar, kbar, vnorm, 0.5, False)
    mp = oracle.metric(qbar, kbar, vnorm)
    for h in range(Hq):
        for i in range(nb):
            s = qbar[0, h, i] @ kbar[0, h // G, : i + 1].T / math.sqrt(D)
            diff = oracle.metric_row(mh, 0, h, i) - np.log(oracle.metric_row(mp, 0, h, i))
            np.testing.assert_allclose(diff, logsumexp(s), rtol=1e-11, atol=1e-11)
    # clamp: V blocks of constant rows with norm 3 (odd blocks) and 0.5 (even blocks); Q = 0
    # so M = beta * max(0, log n^2): 0.2 * 2 ln 3 and 0 (clamped) or 0.2 * 2 ln 0.5 (not)
    S, block, Dv = 128, 16, 8
    nbv = S // block
    vv = torch.zeros(1, 1, S, Dv)
    for j in range(nbv):
        vv[0, 0, j * block:(j + 1) * block, 0] = 3.0 if j % 2 else 0.5
    z = torch.zeros(1, 1, S, Dv)
    qb, kb, vn = oracle.pool(z, z, vv, block)
    beta = float(np.float32(0.2))
    mc = oracle.metric_additive(qb, kb, vn, 0.2, True)
    mu_ = oracle.metric_additive(qb, kb, vn, 0.2, False)
    row_c = oracle.metric_row(mc, 0, 0, nbv - 1)
    row_u = oracle.metric_row(mu_, 0, 0, nbv - 1)
    for j in range(nbv):
        want_c = beta * 2 * math.log(3.0) if j % 2 else 0.0
        want_u = beta * 2 * math.log(3.0 if j % 2 else 0.5)
        assert abs(row_c[j] - want_c) < 1e-13 and abs(row_u[j] - want_u) < 1e-13, (j, row_c[j], row_u[j])


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


def pin_group():
    q, k, v = _tiny_inputs(71, Hq=4, Hkv=2, S=256, D=16, block=16)
    G = 2
    # G = 1: one head per group, the group metric is the head's metric
    res1 = oracle.prefill(q[:, :2], k, v, 16, 0.2, 3.0, 2)
    resg = oracle.prefill(q[:, :2], k, v, 16, 0.2, 3.0, 2, share="group")
    np.testing.assert_array_equal(res1["sel_idx"], resg["sel_idx"])
    # identical query heads in each group: the group keeps what each head keeps
    qq = q[:, ::G].repeat_interleave(G, dim=1)
    ref = oracle.prefill(qq, k, v, 16, 0.2, 3.0, 2)
    got = oracle.prefill(qq, k, v, 16, 0.2, 3.0, 2, share="group")
    np.testing.assert_array_equal(got["sel_idx"], ref["sel_idx"])
    # brute force: numpy metric summed over the group's heads, full sort, replicated
    res = oracle.prefill(q, k, v, 16, 0.2, 3.0, 2, share="group")
    md = brute.metric_dense(*brute.pool(q, k, v, 16))  # [B, Hq, nb, nb]
    mg = md.reshape(1, 2, G, 16, 16).sum(axis=2)
    rows = brute.select_rows(mg, res["k"])
    kept = _kept_from_csr(res["sel_idx"], res["sel_cnt"], res["off"], 1, 4, 16)
    for (b, g, i), lst in rows.items():
        for h in range(G):
            assert kept[(b, g * G + h, i)] == lst, (g, h, i)
    # additive: the group score is sum_h s + G * beta * max(0, log n^2)
    qb, kb, vn = oracle.pool(q, k, v, 16)
    ma = oracle.metric_additive(qb, kb, vn, 0.2, True)
    mga = oracle.metric_group(ma, G)
    beta = float(np.float32(0.2))
    for g in range(2):
        for i in (3, 9, 15):
            s_sum = sum(qb[0, g * G + h, i] @ kb[0, g, : i + 1].T for h in range(G)) / 4.0
            e = np.maximum(0.0, np.log(vn[0, g, : i + 1] ** 2))
            np.testing.assert_allclose(oracle.metric_row(mga, 0, g, i), s_sum + G * beta * e,
                                       rtol=1e-12, atol=1e-12)


def pin_ragged():
    for dtype in (torch.float32, torch.bfloat16):
        S, block = 16 * 7 + 5, 16
        q, k, v = _tiny_inputs(61, Hq=4, Hkv=2, S=S, D=16, block=block, dtype=dtype)
        got = oracle.pool(q, k, v, block)
        ref = brute.pool(q, k, v, block)
        for a, b in zip(got, ref):
            assert a.shape == b.shape and a.shape[2] == 8
            np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
        res = oracle.prefill(q, k, v, block, 0.3, 3.0, 2)
        nb = 8
        kept = _kept_from_csr(res["sel_idx"], res["sel_cnt"], res["off"], 1, 4, nb)
        out = brute.attention_masked(q, k, v, block, kept)  # [1, 4, S, D]
        got = res["out"].reshape(1, 4, nb, block, 16)
        for h in range(4):
            for i in range(nb):
                n = min(block, S - i * block)
                np.testing.assert_allclose(got[0, h, i, :n], out[0, h, i * block:i * block + n],
                                           rtol=1e-10, atol=1e-12)
                assert not got[0, h, i, n:].any(), "rows past S stay 0"
        # prefix: the first 7 full blocks alone give the same everything for those blocks
        pre = oracle.prefill(q[:, :, :112], k[:, :, :112], v[:, :, :112], block, 0.3, 3.0, 2)
        for a, b in (("qbar", 2), ("kbar", 2), ("vnorm", 2)):
            np.testing.assert_array_equal(res[a][:, :, :7], pre[a])
        off7 = pre["off"]
        np.testing.assert_array_equal(res["sel_idx"][:, :, :off7[7]], pre["sel_idx"])
        np.testing.assert_array_equal(res["out"].reshape(1, 4, nb, block, 16)[:, :, :7],
                                      pre["out"].reshape(1, 4, 7, block, 16))
    # a partial block of 5 identical rows x pools to x, its V norm to |x|
    x = torch.randn(1, 1, 1, 8, generator=torch.Generator().manual_seed(9))
    z = torch.zeros(1, 1, 16, 8)
    qq = torch.cat([z, x.repeat(1, 1, 5, 1)], dim=2)
    qb, kb, vn = oracle.pool(qq, qq, qq, 16)
    np.testing.assert_allclose(qb[0, 0, 1], x[0, 0, 0].double().numpy(), rtol=1e-12)
    np.testing.assert_allclose(vn[0, 0, 1], float(torch.linalg.vector_norm(x.double())),
                               rtol=1e-12)


# --------------------------------------------------------------------------- anti-diagonal


def _hand_antidiag_cases():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                        "antidiag_hand.txt")
    cases = []
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        head, qs, ks, ps = line.split("|")
        S, D, block, stride = (int(x) for x in head.split())
        rows = [[float(x) for x in r.split()] for r in ps.split(";")]
        cases.append((S, D, block, stride, [float(x) for x in qs.split()],
                      [float(x) for x in ks.split()], rows))
    return cases


def pin_antidiag_hand():
    cases = _hand_antidiag_cases()
    assert len(cases) == 2
    for S, D, block, stride, qv, kv, rows in cases:
        for dtype in (torch.float32, torch.bfloat16):  # every value is exact in bf16
            q = torch.tensor(qv).reshape(1, 1, S, D).to(dtype)
            k = torch.tensor(kv).reshape(1, 1, S, D).to(dtype)
            got = oracle.antidiag(q, k, block, stride, rows=[(0, 0, i) for i in range(len(rows))])
            for i, want in enumerate(rows):
                np.testing.assert_allclose(got[i, :i + 1], want, rtol=1e-14, atol=1e-15)


def pin_antidiag_brute():
    for dtype, (S, block, stride) in ((torch.float32, (128, 16, 4)),
                                      (torch.bfloat16, (16 * 5 + 8, 16, 8)),
                                      (torch.float32, (96, 32, 2))):
        q, k, _ = _tiny_inputs(81, Hq=4, Hkv=2, S=S, D=8, block=block, dtype=dtype)
        got = oracle.antidiag(q, k, block, stride)
        ref = brute.antidiag(q, k, block, stride)
        nb = ref.shape[2]
        for i in range(nb):
            np.testing.assert_allclose(oracle.metric_row(got, 0, 1, i), ref[0, 1, i, :i + 1],
                                       rtol=1e-11, atol=1e-14)
            np.testing.assert_allclose(got[0, :, i * (i + 1) // 2:i * (i + 1) // 2 + i + 1],
                                       ref[0, :, i, :i + 1], rtol=1e-11, atol=1e-14)


def pin_antidiag_stride1():
    # one token per group: a_uw is the token logit and p_ij the block mass of exact causal
    # attention, averaged over the block's query tokens
    for dtype, S in ((torch.float32, 128), (torch.bfloat16, 16 * 6 + 5)):
        q, k, _ = _tiny_inputs(83, Hq=4, Hkv=2, S=S, D=16, block=16, dtype=dtype)
        got = oracle.antidiag(q, k, 16, 1)
        kk = k.double().repeat_interleave(2, dim=1)
        X = q.double() @ kk.transpose(-1, -2) / 4.0
        X = X.masked_fill(~torch.ones(S, S, dtype=torch.bool).tril(), float("-inf"))
        P = torch.softmax(X, dim=-1).numpy()  # [1, 4, S, S]
        nb = -(-S // 16)
        for h in range(4):
            for i in range(nb):
                r0, r1 = i * 16, min(S, i * 16 + 16)
                want = [P[0, h, r0:r1, j * 16:min(S, j * 16 + 16)].sum(axis=1).mean()
                        for j in range(i + 1)]
                np.testing.assert_allclose(oracle.metric_row(got, 0, h, i), want, rtol=1e-11,
                                           atol=1e-14)


def pin_antidiag_pooled_limit_and_metric():
    # stride = block and keys constant inside each block: a_ij = qbar_i . k_j / sqrt(D), the
    # pooled score, so p is the pooled softmax and the product metric the pooled metric
    q, k, v = _tiny_inputs(85, Hq=4, Hkv=2, S=128, D=16, block=16)
    kc = k.reshape(1, 2, 8, 16, 16)[:, :, :, :1, :].expand(1, 2, 8, 16, 16).reshape(1, 2, 128, 16)
    kc = kc.contiguous()
    p = oracle.antidiag(q, kc, 16, 16)
    qb, kb, vn = oracle.pool(q, kc, v, 16)
    np.testing.assert_allclose(p, oracle.metric(qb, kb, np.ones_like(vn)), rtol=1e-11,
                               atol=1e-14)
    np.testing.assert_allclose(oracle.metric_from_p(p, vn), oracle.metric(qb, kb, vn),
                               rtol=1e-11, atol=1e-14)
    # additive at beta = 1/2 without the clamp: ln p + ln n = ln(p n)
    p = oracle.antidiag(q, k, 16, 4)
    _, _, vn = oracle.pool(q, k, v, 16)
    np.testing.assert_allclose(oracle.metric_from_p(p, vn, 0.5, False, "additive"),
                               np.log(oracle.metric_from_p(p, vn)), rtol=1e-12, atol=1e-12)
    # beta = 0: ln p
    np.testing.assert_allclose(oracle.metric_from_p(p, vn, 0.0, True, "additive"), np.log(p),
                               rtol=0, atol=0)


def pin_antidiag_invariants():
    S, block, stride = 16 * 7 + 8, 16, 8
    q, k, _ = _tiny_inputs(87, Hq=4, Hkv=2, S=S, D=16, block=block, dtype=torch.bfloat16)
    p = oracle.antidiag(q, k, block, stride)
    nb = 8
    for h in range(4):
        for i in range(nb):
            row = oracle.metric_row(p, 0, h, i)
            assert np.all(row > 0)
            assert abs(row.sum() - 1.0) < 1e-12
    # causality: the first 7 blocks of a prefix give the same rows
    pre = oracle.antidiag(q[:, :, :112], k[:, :, :112], block, stride)
    np.testing.assert_array_equal(p[:, :, :pre.shape[2]], pre)


PINS = [
    pin_budget_decimal,
    pin_budget_closed_forms,
    pin_pool_closed_forms,
    pin_pool_brute,
    pin_pool_max,
    pin_budget_linear,
    pin_metric_closed_forms,
    pin_metric_additive_equivalence,
    pin_metric_additive_closed_forms,
    pin_metric_brute,
    pin_select_ties_and_special_cases,
    pin_select_brute_and_invariants,
    pin_attention_dense_sdpa,
    pin_attention_closed_forms,
    pin_attention_brute,
    pin_ragged,
    pin_group,
    pin_antidiag_hand,
    pin_antidiag_brute,
    pin_antidiag_stride1,
    pin_antidiag_pooled_limit_and_metric,
    pin_antidiag_invariants,
]


def run_all() -> None:
    """Run every pin; raise on the first failure."""
    for fn in PINS:
        fn()


if __name__ == "__main__":
    run_all()
    print("all pins hold")
