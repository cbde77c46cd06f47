"""The C ABI on the CPU: exports, host-only functions, argument validation (no GPU needed)."""

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


def test_workspace_size_layout():
    B, Hq, Hkv, Sq, D, block = 1, 32, 8, 131072, 128, 128
    nb = Sq // block
    n = S.stem_workspace_size(B, Hq, Hkv, Sq, D, block)
    pooled = 4 * (B * Hq * nb * D + B * Hkv * nb * D + B * Hkv * nb)
    # head-pair step schedule, bounded for any budget: one uint32 per causal block pair
    sched = 4 * B * Hkv * ((Hq // Hkv + 1) // 2) * nb * (nb + 1) // 2
    assert pooled + sched < n < pooled + sched + 64 * 1024
    assert S.stem_workspace_size(B, Hq, Hkv, 1000, D, block) == 0  # ragged: invalid
    assert S.stem_workspace_size(0, Hq, Hkv, Sq, D, block) == 0  # empty


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
        "attn_small_workspace": S.STEM_ERR_WORKSPACE,
        "nb_too_large": S.STEM_ERR_UNSUPPORTED,
        "select_nb_too_large": S.STEM_ERR_UNSUPPORTED,
        "static_nb_too_large": S.STEM_ERR_UNSUPPORTED,
        "empty_B": S.STEM_OK,
        "empty_S": S.STEM_OK,
    })
    assert res == want
