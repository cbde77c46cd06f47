"""Property tests of the CPU oracle over randomised inputs (hypothesis, derandomised so every
run draws the same examples). They complement the fixed pins in tests/pins.py with invariants
and brute-force agreement on shapes the pins do not cover: ragged lengths, GQA ratios, strides.
"""

import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle
from tests import brute

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)


@SETTINGS
@given(nb=st.integers(1, 300), rho=st.floats(0.01, 1.0), tau=st.floats(0.1, 200.0),
       k_min=st.integers(1, 16))
def test_exponential_budget_bounds(nb, rho, tau, k_min):
    k, off = oracle.budget(nb, rho, tau, k_min)
    i = np.arange(nb)
    assert k[0] == 1
    assert np.all(k <= i + 1) and np.all(k[1:] >= 2)
    assert np.all(k >= np.minimum(i + 1, k_min))
    # unless clamped, k(i) is the ceiling of rho(i) * (i + 1)
    r = np.float64(np.float32(rho)) + (1 - np.float64(np.float32(rho))) * np.exp(
        -i / np.float64(np.float32(tau)))
    free = (k > np.maximum(2, k_min)) & (k < i + 1)
    assert np.all(k[free] >= r[free] * (i[free] + 1) - 1e-9)
    assert np.all(k[free] < r[free] * (i[free] + 1) + 1)
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(k)]))


@SETTINGS
@given(nb=st.integers(1, 300), k_start=st.floats(0.5, 300.0), mu=st.floats(0.05, 1.0),
       k_min=st.integers(1, 16))
def test_linear_budget_bounds(nb, k_start, mu, k_min):
    k, off = oracle.budget_linear(nb, k_start, mu, k_min)
    i = np.arange(nb)
    assert k[0] == 1
    assert np.all(k <= i + 1) and np.all(k[1:] >= 2)
    assert np.all(k >= np.minimum(i + 1, k_min))
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(k)]))


def _inputs(seed, B, Hq, Hkv, S, D, dtype):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, S, D), generator=g).to(dtype)
    k = torch.randn((B, Hkv, S, D), generator=g).to(dtype)
    v = torch.randn((B, Hkv, S, D), generator=g).to(dtype)
    return q, k, v


@SETTINGS
@given(seed=st.integers(0, 10 ** 6), G=st.integers(1, 3), Hkv=st.integers(1, 2),
       nb=st.integers(1, 6), tail=st.integers(0, 15), bf16=st.booleans())
def test_pooling_matches_brute_force(seed, G, Hkv, nb, tail, bf16):
    block = 16
    S = max(1, nb * block - tail)
    q, k, v = _inputs(seed, 1, G * Hkv, Hkv, S, 8, torch.bfloat16 if bf16 else torch.float32)
    for got, ref in zip(oracle.pool(q, k, v, block), brute.pool(q, k, v, block)):
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


@SETTINGS
@given(seed=st.integers(0, 10 ** 6), G=st.integers(1, 3), nb=st.integers(1, 5),
       stride=st.sampled_from([1, 2, 4, 8, 16]), groups_less=st.integers(0, 3))
def test_antidiag_rows_and_brute_force(seed, G, nb, stride, groups_less):
    block = 16
    S = max(stride, nb * block - stride * min(groups_less, block // stride - 1))
    q, k, _ = _inputs(seed, 1, G, 1, S, 8, torch.float32)
    p = oracle.antidiag(q, k, block, stride)
    ref = brute.antidiag(q, k, block, stride)
    nbl = -(-S // block)
    for h in range(G):
        for i in range(nbl):
            row = oracle.metric_row(p, 0, h, i)
            assert abs(row.sum() - 1.0) < 1e-12 and np.all(row > 0)
            np.testing.assert_allclose(row, ref[0, h, i, :i + 1], rtol=1e-10, atol=1e-14)


@SETTINGS
@given(seed=st.integers(0, 10 ** 6), nb=st.integers(1, 40), rho=st.floats(0.05, 1.0),
       k_min=st.integers(1, 6))
def test_selection_structure(seed, nb, rho, k_min):
    rng = np.random.default_rng(seed)
    m = rng.random((1, 2, nb * (nb + 1) // 2))
    kk, off = oracle.budget(nb, rho, 4.0, k_min)
    si, sc = oracle.select(m, kk, off)
    assert np.array_equal(sc[0, 0], kk)
    for h in range(2):
        for i in range(nb):
            row = si[0, h, off[i]:off[i + 1]]
            assert len(row) == kk[i] and row[0] == 0 and row[-1] == i
            assert np.all(np.diff(row) > 0)
            # the kept middle blocks are the largest of 1..i-1
            mid = row[1:-1]
            if len(mid):
                mrow = oracle.metric_row(m, 0, h, i)
                rest = np.setdiff1d(np.arange(1, i), mid)
                if len(rest):
                    assert mrow[mid].min() >= mrow[rest].max()
