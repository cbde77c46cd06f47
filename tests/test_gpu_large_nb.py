"""More than 1024 query blocks per head: the selection kernel's smaller row tiles (16 rows per
CTA for nb <= 2048, 8 rows up to STEM_MAX_NB = 4096, whose score rows fill its shared memory)
and the attention kernels at that length, on a B200.

Each case uses the Llama-shaped value recipe (RoPE, planted sink, V outliers) with few heads,
so the oracle finishes in seconds. Stage parity: the selection kernel on the oracle's pooled
values (rounded to float32) against the oracle's selection and float64 metric from the same
values, every row. End to end: stem_prefill_ex's selection against the oracle on every row,
its output on sampled query blocks (and on every tie-swapped row, over the GPU's own kept set).
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import parity
from tests.test_gpu_fullsize import sample

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DEV = "cuda:0"


def _w(name, S_, block, **kw):
    return wl.LLAMA_128K.replace(**dict(dict(name=name, Hq=2, Hkv=1, S=S_, block=block), **kw))


CASES = {
    "nb1025-blk128": _w("nb1025-blk128", 1025 * 128, 128),                 # 16-row tiles
    "nb2048-blk64": _w("nb2048-blk64", 2048 * 64, 64),                     # 16-row tiles
    "nb2048-blk128-gqa": _w("nb2048-blk128-gqa", 2048 * 128, 128, Hq=4),  # 16, four q heads
    "nb2049-blk64": _w("nb2049-blk64", 2049 * 64, 64),                     # 8-row tiles
    "nb3001-ragged": _w("nb3001-ragged", 3000 * 64 + 17, 64, rho_min=0.1, tau=32.0),
    "nb4096-blk64": _w("nb4096-blk64", 4096 * 64, 64),                     # 8-row tiles, max nb
}


def _pooled(w):
    q, k, v = wl.make_inputs(w, DEV)
    cpu = tuple(t.cpu() for t in (q, k, v))
    return (q, k, v), cpu, oracle.pool(*cpu, w.block)


@pytest.mark.parametrize("name", list(CASES))
def test_select_stage_on_oracle_pooling(name):
    w = CASES[name]
    assert w.nb > 1024
    _, _, (rq, rk, rn) = _pooled(w)
    q32, k32, n32 = (torch.from_numpy(x).float() for x in (rq, rk, rn))
    m = oracle.metric(q32.double().numpy(), k32.double().numpy(), n32.double().numpy())
    kk, off = oracle.budget(w.nb, w.rho_min, w.tau, w.k_min)
    ref_idx, ref_cnt = oracle.select(m, kk, off)
    sel_idx, sel_cnt, m_gpu = S.stem_select(q32.to(DEV), k32.to(DEV), n32.to(DEV), w.rho_min,
                                            w.tau, w.k_min, with_metric=True)
    torch.cuda.synchronize()
    res = parity.compare_selection(sel_idx, sel_cnt, ref_idx, ref_cnt, m, kk, off)
    assert not res["violations"], res["violations"][:5]
    assert res["tie_swaps"] <= max(1, res["rows"] // 100), res
    np.testing.assert_allclose(m_gpu.double().cpu().numpy(), m, rtol=2e-5, atol=1e-30)


@pytest.mark.parametrize("name", list(CASES))
def test_end_to_end(name):
    w = CASES[name]
    (q, k, v), cpu, (rq, rk, rn) = _pooled(w)
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    out, sel_idx, sel_cnt = S.stem_prefill_ex(q, k, v, w.block, w.rho_min, w.tau, w.k_min,
                                              status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kk, off = oracle.budget(w.nb, w.rho_min, w.tau, w.k_min)
    m = oracle.metric(rq, rk, rn)
    ref_idx, ref_cnt = oracle.select(m, kk, off)
    res = parity.compare_selection(sel_idx, sel_cnt, ref_idx, ref_cnt, m, kk, off)
    assert not res["violations"], res["violations"][:5]
    assert res["tie_swaps"] <= max(1, res["rows"] // 100), res
    rows = sorted(set(sample(w, kk)) | set(res["rows_bad"]))
    ref = oracle.attention(*cpu, w.block, ref_idx, ref_cnt, off, rows)
    parity.assert_prefill_out(out, cpu, w.block, ref, rows, res, sel_idx, sel_cnt, off,
                              w.torch_dtype, name)
