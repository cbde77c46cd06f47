"""The C ABI on the CPU: exports, host-only functions, argument validation (no GPU needed)."""

import ctypes
import json
import os
import re
import subprocess
import sys

import numpy as np
import pytest

import oracle
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "stem.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(stem_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(S.EXPORTED)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", S.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(S.lib(), f)


@pytest.mark.parametrize("case", pins.BUDGET_CASES + [
    (w.nb, w.rho_min, w.tau, w.k_min) for w in wl.WORKLOADS.values()])
def test_budget_matches_oracle(case):
    nb, r, t, km = case
    k, off = S.stem_budget(nb, r, t, km)
    ko, offo = oracle.budget(nb, r, t, km)
    assert np.array_equal(k.numpy(), ko)
    assert np.array_equal(off.numpy().astype(np.int64), offo)
    assert S.stem_sel_capacity(nb, r, t, km) == int(offo[-1])


LINEAR_CASES = [(8, 8.0, 0.5, 1), (6, 10.0, 0.35, 3), (1024, 36.0, 0.7, 8), (512, 40.0, 0.7, 4),
                (128, 12.0, 0.7, 8), (1000, 700.0, 0.05, 1), (1, 4.0, 0.7, 1), (0, 4.0, 0.7, 1),
                (4096, 64.0, 0.3, 2)]


@pytest.mark.parametrize("case", LINEAR_CASES, ids=lambda c: "-".join(map(str, c)))
def test_linear_budget_matches_oracle(case):
    nb, ks, mu, km = case
    m = S.make_method("linear", k_start=ks, mu=mu, k_min=km)
    k, off = S.stem_budget_m(nb, m)
    ko, offo = oracle.budget_linear(nb, ks, mu, km)
    assert np.array_equal(k.numpy(), ko)
    assert np.array_equal(off.numpy().astype(np.int64), offo)
    assert S.stem_sel_capacity(nb, 0.0, 0.0, 0, method=m) == int(offo[-1])


def test_method_budget_defaults_equal_plain_calls():
    for nb, r, t, km in [(1024, 0.05, 64.0, 8), (256, 0.1, 32.0, 4), (16, 0.25, 4.0, 2)]:
        m = S.make_method("exp", rho_min=r, tau=t, k_min=km, metric="additive", beta=0.2,
                          vsum="max")
        k1, off1 = S.stem_budget_m(nb, m)
        k2, off2 = S.stem_budget(nb, r, t, km)
        assert np.array_equal(k1.numpy(), k2.numpy()) and np.array_equal(off1.numpy(), off2.numpy())


@pytest.mark.parametrize("bad", [
    dict(schedule="linear", k_start=0.0, mu=0.7), dict(schedule="linear", k_start=-3.0, mu=0.7),
    dict(schedule="linear", k_start=float("inf"), mu=0.7),
    dict(schedule="linear", k_start=8.0, mu=0.0), dict(schedule="linear", k_start=8.0, mu=1.5),
    dict(schedule="linear", k_start=8.0, mu=float("nan")),
    dict(schedule="exp", rho_min=0.0, tau=4.0), dict(schedule="exp", rho_min=0.5, tau=0.0),
    dict(schedule="exp", rho_min=0.5, tau=4.0, k_min=0),
    dict(schedule="exp", rho_min=0.5, tau=4.0, metric="additive", beta=-0.1),
    dict(schedule="exp", rho_min=0.5, tau=4.0, metric="additive", beta=float("nan")),
], ids=lambda d: ",".join(f"{k}={v}" for k, v in d.items()))
def test_method_validation(bad):
    m = S.make_method(**{"k_min": 1, **bad})
    assert S.lib().stem_budget_m(64, ctypes.byref(m), None, None) == S.STEM_ERR_ARG
    assert S.lib().stem_sel_capacity_m(64, ctypes.byref(m)) == S.STEM_ERR_ARG
    # enum fields outside their sets
    for field, val in (("schedule", 2), ("metric", 5), ("vsum", -1)):
        m2 = S.make_method("exp", rho_min=0.5, tau=4.0, k_min=1)
        setattr(m2, field, val)
        assert S.lib().stem_budget_m(64, ctypes.byref(m2), None, None) == S.STEM_ERR_ARG
    m3 = S.make_method("exp", rho_min=0.5, tau=4.0, k_min=1, metric="additive", beta=0.2)
    m3.clamp = 2
    assert S.lib().stem_budget_m(64, ctypes.byref(m3), None, None) == S.STEM_ERR_ARG
    assert S.lib().stem_budget_m(64, None, None, None) == S.STEM_ERR_ARG


def test_varlen_capacity_and_workspace():
    m = S.make_method("exp", rho_min=0.2, tau=8.0, k_min=3)
    cu = [0, 4096, 4173, 4173, 6746]
    total = sum(S.stem_sel_capacity(-(-(cu[s + 1] - cu[s]) // 128), 0, 0, 0, method=m)
                for s in range(4))
    assert S.stem_varlen_sel_capacity(cu, 128, m) == total
    arr = (ctypes.c_int32 * 5)(*cu)
    ws = S.lib().stem_varlen_workspace_size(4, arr, 8, 2, 128, 128)
    assert ws == max(S.stem_workspace_size(1, 8, 2, cu[s + 1] - cu[s], 128, 128)
                     for s in range(4))
    for bad in ([1, 5], [0, 5, 3]):
        arr = (ctypes.c_int32 * len(bad))(*bad)
        assert S.lib().stem_varlen_sel_capacity(len(bad) - 1, arr, 128, ctypes.byref(m)) == \
            S.STEM_ERR_ARG
        assert S.lib().stem_varlen_workspace_size(len(bad) - 1, arr, 8, 2, 128, 128) == 0


def test_withhold_switch_is_host_state_only():
    """The test switch for the timeout path is a host-side flag: it toggles, reports the previous
    value and is left off."""
    L = S.lib()
    assert L.stem_test_withhold_q(0) in (0, 1)
    assert L.stem_test_withhold_q(1) == 0
    assert L.stem_test_withhold_q(7) == 1
    assert L.stem_test_withhold_q(0) == 1
    assert L.stem_test_withhold_q(0) == 0


def test_workspace_size_layout():
    B, Hq, Hkv, Sq, D, block = 1, 32, 8, 131072, 128, 128
    nb = Sq // block
    n = S.stem_workspace_size(B, Hq, Hkv, Sq, D, block)
    pooled = 4 * (B * Hq * nb * D + B * Hkv * nb * D + B * Hkv * nb)
    # one region shared by the selection's score triangles (every head's, up to 128 MB) and,
    # later in the call, the head-pair step schedule (one uint32 per causal block pair per head
    # pair, after a 256-byte work counter): the larger of the two
    sched = 256 + 4 * B * Hkv * ((Hq // Hkv + 1) // 2) * nb * (nb + 1) // 2
    scores = min(4 * B * Hq * nb * (nb + 1) // 2, 128 << 20)
    assert pooled + max(sched, scores) < n < pooled + max(sched, scores) + 64 * 1024
    # a partial last block is a block of its own: 1000 tokens need the layout of 8 blocks
    assert S.stem_workspace_size(B, Hq, Hkv, 1000, D, block) == \
        S.stem_workspace_size(B, Hq, Hkv, 1024, D, block) > 0
    assert S.stem_workspace_size(B, Hq, Hkv, 1000, 96, block) == 0  # unsupported D
    assert S.stem_workspace_size(0, Hq, Hkv, Sq, D, block) == 0  # empty
    # anti-diagonal scoring adds p (packed rows) and the estimator's partials, per head:
    # R*nb*(nb+1)/2 block sums, c*n - 32*c*(c-1)/2 chunk maxima (c = ceil(n/32) chunks of the
    # n = S/stride groups) and each part's max and sum (t = ceil(n/128) query tiles, parts =
    # ceil(ceil(n/256)/4) per tile), after a 256-byte work counter
    ad = S.make_method("exp", rho_min=0.05, tau=64.0, k_min=8, score="antidiag", stride=16)
    assert S.stem_workspace_size(B, Hq, Hkv, Sq, D, block, ad.__class__.from_buffer_copy(
        S.make_method("exp", rho_min=0.05, tau=64.0, k_min=8))) == n
    na = S.stem_workspace_size(B, Hq, Hkv, Sq, D, block, ad)
    p_bytes = 4 * B * Hq * nb * (nb + 1) // 2
    nred, R = Sq // 16, block // 16
    c, t = -(-nred // 32), -(-nred // 128)
    parts = -(-(-(-nred // 256)) // 4)
    scratch = 4 * B * Hq * (R * nb * (nb + 1) // 2 + c * nred - 32 * c * (c - 1) // 2 +
                            2 * 128 * t * parts)
    assert scratch == 688914432  # about 690 MB
    assert n + p_bytes + scratch + 256 <= na < n + p_bytes + scratch + 1024  # + work counter
    ad.stride = 24
    assert S.stem_workspace_size(B, Hq, Hkv, Sq, D, block, ad) == 0


def test_strerror_covers_every_code():
    for c in range(-5, 1):
        msg = S.strerror(c)
        assert msg and msg != "unknown error code"
    assert S.strerror(-99) == "unknown error code"


def test_argument_validation_rejects_before_any_device_work():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "abi_probe.py")], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    res = json.loads(r.stdout.strip().splitlines()[-1])
    want = {k: S.STEM_ERR_ARG for k in res}
    want.update({
        "workspace_null": S.STEM_ERR_WORKSPACE,
        "workspace_small": S.STEM_ERR_WORKSPACE,
        "workspace_misaligned": S.STEM_ERR_WORKSPACE,
        "select_no_workspace": S.STEM_ERR_WORKSPACE,
        "select_m_no_workspace": S.STEM_ERR_WORKSPACE,
        "varlen_small_workspace": S.STEM_ERR_WORKSPACE,
        "varlen_all_empty": S.STEM_OK,
        "attn_small_workspace": S.STEM_ERR_WORKSPACE,
        "nb_too_large": S.STEM_ERR_UNSUPPORTED,
        "select_nb_too_large": S.STEM_ERR_UNSUPPORTED,
        "static_nb_too_large": S.STEM_ERR_UNSUPPORTED,
        "group_nb_too_large": S.STEM_ERR_UNSUPPORTED,
        "empty_B": S.STEM_OK,
        "empty_S": S.STEM_OK,
        "ad_f32": S.STEM_ERR_UNSUPPORTED,
        "ad_small_workspace": S.STEM_ERR_WORKSPACE,
        "antidiag_m_f32": S.STEM_ERR_UNSUPPORTED,
        "antidiag_m_small_workspace": S.STEM_ERR_WORKSPACE,
        "antidiag_m_empty": S.STEM_OK,
        "select_p_no_workspace": S.STEM_ERR_WORKSPACE,
        "select_p_nb_too_large": S.STEM_ERR_UNSUPPORTED,
    })
    assert res == want
