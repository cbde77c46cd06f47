"""The tensor-core kernels' bounded waits, on a B200 (attention at block 128 and 64, and the
anti-diagonal estimator below): a wait that runs out (a Q tile the producer
never sends, via the library's test switch) ends the kernel with STEM_ERR_TIMEOUT in the status
word instead of hanging it, and the CUDA context stays usable: the next call is exact again.
"""

import time

import pytest
import torch

import oracle
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("block", [128, 64])
def test_expired_wait_reports_timeout_and_the_context_survives(block):
    w = wl.LLAMA_32K.replace(name=f"timeout-4k-blk{block}", Hq=8, Hkv=2, S=4096, block=block)
    q, k, v = wl.make_inputs(w, "cpu")
    dq, dk, dv = (t.to(DEV) for t in (q, k, v))
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    lib = S.lib()
    assert lib.stem_test_withhold_q(1) == 0
    try:
        t0 = time.perf_counter()
        S.stem_prefill_ex(dq, dk, dv, w.block, w.rho_min, w.tau, w.k_min, status=status)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        lib.stem_test_withhold_q(0)
    assert int(status.item()) == S.STEM_ERR_TIMEOUT
    assert elapsed < 30.0, elapsed  # one bounded wait (2 s) plus the bounded drains
    # the context is usable and the next call is exact
    status.fill_(7)
    out, sel_idx, sel_cnt = S.stem_prefill_ex(dq, dk, dv, w.block, w.rho_min, w.tau, w.k_min,
                                              status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.prefill(q, k, v, w.block, w.rho_min, w.tau, w.k_min)
    res = parity.compare_selection(sel_idx, sel_cnt, ref["sel_idx"], ref["sel_cnt"], ref["m"],
                                   ref["k"], ref["off"])
    assert not res["violations"], res["violations"][:5]
    rows = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)]
    parity.assert_prefill_out(out, (q, k, v), w.block, ref["out"], rows, res, sel_idx, sel_cnt,
                              ref["off"], w.torch_dtype, "after timeout")


def test_estimator_expired_wait_reports_timeout_and_the_context_survives():
    w = wl.LLAMA_32K.replace(name="timeout-ad-4k", Hq=8, Hkv=2, S=4096)
    q, k, _ = wl.make_inputs(w, "cpu")
    dq, dk = q.to(DEV), k.to(DEV)
    m = S.make_method("exp", rho_min=w.rho_min, tau=w.tau, k_min=w.k_min, score="antidiag",
                      stride=16)
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    lib = S.lib()
    assert lib.stem_test_withhold_q(1) == 0
    try:
        t0 = time.perf_counter()
        S.stem_antidiag(dq, dk, w.block, m, status=status)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        lib.stem_test_withhold_q(0)
    assert int(status.item()) == S.STEM_ERR_TIMEOUT
    assert elapsed < 30.0, elapsed  # one bounded wait (2 s) plus the bounded drains
    # the context is usable and the next call is exact
    status.fill_(7)
    p = S.stem_antidiag(dq, dk, w.block, m, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.antidiag(q, k, w.block, 16)
    import numpy as np
    got = p.double().cpu().numpy()
    assert float(np.max(np.abs(got - ref) / ref)) < 1e-3
