"""Workload generator properties and the stored budget fixture (CPU only)."""

import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_causal_pooling_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "budget_sums.txt")


def golden_rows():
    rows = []
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        name, nb, r, t, km, tot, kmax, klast = line.split()
        rows.append((name, int(nb), float(r), float(t), int(km), int(tot), int(kmax), int(klast)))
    return rows


def test_golden_covers_every_workload():
    assert {r[0] for r in golden_rows()} == set(wl.WORKLOADS)


@pytest.mark.parametrize("row", golden_rows(), ids=lambda r: r[0])
def test_oracle_reproduces_golden_budget(row):
    name, nb, r, t, km, tot, kmax, klast = row
    w = wl.WORKLOADS[name]
    assert (w.nb, w.rho_min, w.tau, w.k_min) == (nb, r, t, km)
    k, off = oracle.budget(nb, r, t, km)
    assert (int(off[-1]), int(k.max()), int(k[-1])) == (tot, kmax, klast)


def test_generator_is_deterministic_and_shaped():
    w = wl.LLAMA_32K.replace(S=1024, Hq=4, Hkv=2)
    a = wl.make_inputs(w)
    b = wl.make_inputs(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    q, k, v = a
    assert q.shape == (1, 4, 1024, 128) and k.shape == v.shape == (1, 2, 1024, 128)
    assert q.dtype == torch.bfloat16
    # planted sink: token 0's K row is 8x larger than typical rows
    kn = k.float().norm(dim=-1)
    assert torch.all(kn[:, :, 0] > 4 * kn[:, :, 1:].median())
    # V outliers: round(0.005 * S) rows per kv-head scaled by 5
    vn = v.float().norm(dim=-1)
    n_out = w.n_v_outliers()
    assert n_out == 5
    assert int((vn > 3 * vn.median()).sum()) == n_out * 2


def test_rope_preserves_pair_norms():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(1, 2, 64, 16, generator=g)
    y = wl.apply_rope(x.clone(), 5e5)
    n0 = x[..., :8] ** 2 + x[..., 8:] ** 2
    n1 = y[..., :8] ** 2 + y[..., 8:] ** 2
    torch.testing.assert_close(n0, n1, rtol=1e-5, atol=1e-5)
    torch.testing.assert_close(x[:, :, 0], y[:, :, 0])  # position 0 is the identity


def test_heavy_tails_present():
    w = wl.QWEN_64K.replace(S=2048)
    q, k, v = wl.make_inputs(w)
    frac_big = float((q.float().abs() > 6).float().mean())
    assert 1e-4 < frac_big < 0.02  # N(0,1) alone gives ~2e-9


def test_sample_rows_deterministic():
    a = wl.sample_rows(wl.LLAMA_128K, heads=[0, 5])
    b = wl.sample_rows(wl.LLAMA_128K, heads=[0, 5])
    assert a == b and len(a) == 2 * 64
    assert (0, 0, 0) in a and (0, 5, 1023) in a
