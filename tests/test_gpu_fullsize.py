"""Full-size parity: every named workload at its real shape, through the same C-ABI call and
launch configuration the benchmark times (stem_prefill_ex, caller workspace, torch's stream).

Selection is compared with the oracle on every (b, head, query block) row (ties within 1e-6
relative allowed). Attention is compared on a deterministic sample of query blocks that the
fp64 oracle computes one by one (bounded to a few tens of GFLOP per workload), and, for the
dense budget rho_min = 1, on the whole output against torch's scaled_dot_product_attention in
float32.
"""

import random

import numpy as np
import pytest
import torch
from torch.nn.attention import SDPBackend, sdpa_kernel

import oracle
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import parity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DEV = "cuda:0"
FULL = ([wl.LLAMA_32K, wl.LLAMA_128K, wl.QWEN_64K] + list(wl.SWEEP_128K[1:]) +
        list(wl.SWEEP_B4_16K) +
        [wl.LLAMA_128K.replace(name="llama3-8b-128k-ragged", S=131072 - 37)])
ORACLE_GFLOP_BUDGET = 40.0


def sample(w, kk, seed=7):
    """Blocks 0, 1, nb-1 of heads 0 and Hq-1, then random (b, h, i) rows while the oracle's
    effective work stays within the budget."""
    rng = random.Random(seed)
    rows, total = [], 0.0
    for (b, h, i) in [(0, 0, 0), (0, 0, 1), (0, w.Hq - 1, 0), (0, w.Hq - 1, w.nb - 1),
                      (w.B - 1, 0, w.nb - 1)]:
        rows.append((b, h, i))
        total += wl.effective_flops(int(kk[i]), w.block, w.D)
    tries = 0
    while tries < 500:
        tries += 1
        r = (rng.randrange(w.B), rng.randrange(w.Hq), rng.randrange(w.nb))
        f = wl.effective_flops(int(kk[r[2]]), w.block, w.D)
        if r in rows or total + f > ORACLE_GFLOP_BUDGET * 1e9:
            continue
        rows.append(r)
        total += f
    return sorted(set(rows))


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_selection_and_sampled_attention(w):
    q, k, v = wl.make_inputs(w, DEV)
    out, sel_idx, sel_cnt = S.alloc_outputs(q, k, w.block, w.rho_min, w.tau, w.k_min)
    ws = S.alloc_workspace(q, k, w.block)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    S.stem_prefill_ex(q, k, v, w.block, w.rho_min, w.tau, w.k_min, out, sel_idx, sel_cnt, ws,
                      status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    kk, off = oracle.budget(w.nb, w.rho_min, w.tau, w.k_min)
    qb, kb, vn = oracle.pool(qc, kc, vc, w.block)
    m = oracle.metric(qb, kb, vn)
    ref_idx, ref_cnt = oracle.select(m, kk, off)
    res = parity.compare_selection(sel_idx, sel_cnt, ref_idx, ref_cnt, m, kk, off)
    assert not res["violations"], res["violations"][:5]
    assert res["tie_swaps"] <= max(1, res["rows"] // 100), res
    # sampled rows, plus every tie-swapped row (checked on the GPU's own kept set)
    rows = sorted(set(sample(w, kk)) | set(res["rows_bad"]))
    ref = oracle.attention(qc, kc, vc, w.block, ref_idx, ref_cnt, off, rows)
    parity.assert_prefill_out(out, (qc, kc, vc), w.block, ref, rows, res, sel_idx, sel_cnt, off,
                              w.torch_dtype, w.name)
    if w.rho_min == 1.0:  # dense: the whole output against the library routine in float32
        G = w.Hq // w.Hkv
        for b in range(w.B):
            for h0 in range(0, w.Hq, 4):
                h1 = min(w.Hq, h0 + 4)
                sl = (slice(b, b + 1), slice(h0, h1))
                kv = (slice(b, b + 1), slice(h0 // G, (h1 - 1) // G + 1))
                k_rep = k[kv].float().repeat_interleave(G, 1)[:, h0 % G:h0 % G + h1 - h0]
                v_rep = v[kv].float().repeat_interleave(G, 1)[:, h0 % G:h0 % G + h1 - h0]
                # the memory-efficient kernel takes float32 at any length (no S x S scores)
                with sdpa_kernel([SDPBackend.EFFICIENT_ATTENTION]):
                    ref_d = torch.nn.functional.scaled_dot_product_attention(
                        q[sl].float(), k_rep, v_rep, is_causal=True)
                parity.assert_out_close(out[sl].double().cpu().numpy(),
                                        ref_d.double().cpu().numpy(), w.torch_dtype,
                                        f"{w.name} dense b{b} h{h0}")
