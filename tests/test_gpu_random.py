"""Seeded random shapes and methods against the oracle, on a B200.

Each case draws its shape (batch, GQA ratio, a sequence length that is usually not a multiple
of the block, block 64 or 128, D 64 or 128, bf16 or f32) and its method (budget schedule, metric
form, V summary, group sharing, pooled or anti-diagonal scores) from a fixed seed, runs the whole
path through stem_prefill_ex and compares selection and output with the oracle, as the fixed
cases do.
"""

import math
import random

import pytest
import torch

import oracle
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import parity, test_gpu_antidiag

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
N_CASES = 40


def draw(seed):
    rng = random.Random(1000 + seed)
    block = rng.choice([64, 128])
    D = rng.choice([64, 128])
    dtype = "bf16" if rng.random() < 0.75 else "f32"
    Hkv = rng.choice([1, 2])
    G = rng.choice([1, 2, 3, 4])
    nb = rng.randint(1, 14)
    S_ = nb * block - rng.choice([0, 0, 1, 37, block - 1]) if nb > 1 else rng.randint(1, block)
    S_ = max(S_, 1)
    md = dict(k_min=rng.randint(1, 4))
    if rng.random() < 0.5:
        md.update(schedule="exp", rho_min=rng.choice([0.05, 0.2, 0.5, 1.0]),
                  tau=rng.choice([1.0, 3.0, 8.0]))
    else:
        md.update(schedule="linear", k_start=rng.choice([2.5, 6.0, 11.3]),
                  mu=rng.choice([0.35, 0.7, 1.0]))
    if rng.random() < 0.4:
        md.update(metric="additive", beta=rng.choice([0.0, 0.2, 0.5]),
                  clamp=rng.random() < 0.5)
    md["vsum"] = rng.choice(["mean", "max"])
    md["share"] = "group" if (G > 1 and rng.random() < 0.3) else "head"
    # anti-diagonal scores need bf16 and a stride dividing both block and S
    strides = [s for s in (4, 8, 16, 32) if block % s == 0 and block // s <= 32 and S_ % s == 0]
    if dtype == "bf16" and strides and rng.random() < 0.5:
        md.update(score="antidiag", stride=rng.choice(strides))
    # V outliers: the float32 tiny workload's 16 rows per kv head; bfloat16 cases take the
    # bfloat16 workloads' density, 0.5% of the rows (16 x5 rows among a few hundred tokens put
    # a bfloat16 kernel's P rounding, 2^-9 per weight, past 2e-2 on outputs below 8)
    vo = dict(v_outlier_rows=None, v_outlier_frac=0.005) if dtype == "bf16" else {}
    w = wl.TINY.replace(name=f"random-{seed}", B=rng.choice([1, 2]), Hq=Hkv * G, Hkv=Hkv, S=S_,
                        D=D, block=block, dtype=dtype, seed=wl.BASE_SEED + 500 + seed, **vo)
    return w, md


def oracle_kwargs(md):
    return dict(rho_min=md.get("rho_min", 1.0), tau=md.get("tau", 1.0), k_min=md["k_min"],
                schedule=md["schedule"], k_start=md.get("k_start", 0.0), mu=md.get("mu", 1.0),
                metric_form=md.get("metric", "product"), beta=md.get("beta", 0.0),
                clamp=md.get("clamp", True), vsum=md["vsum"], share=md["share"],
                score=md.get("score", "pooled"), stride=md.get("stride", 16))


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_case(seed):
    w, md = draw(seed)
    q, k, v = wl.make_inputs(w, "cpu")
    ref = oracle.prefill(q, k, v, w.block, **oracle_kwargs(md))
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    out, sel_idx, sel_cnt = S.stem_prefill_ex(q.to(DEV), k.to(DEV), v.to(DEV), w.block, 0.0, 0.0,
                                              0, status=status, method=S.make_method(**md))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    additive = md.get("metric") == "additive"
    rel = parity.REL_TIE
    if md.get("score") == "antidiag":
        t = test_gpu_antidiag.p_rel_tol(q, k, md["stride"])
        rel = 2.0 * (math.log1p(t) + 1e-6 if additive else t)
    res = parity.compare_selection(sel_idx, sel_cnt, ref["sel_idx"], ref["sel_cnt"], ref["m"],
                                   ref["k"], ref["off"], rel=rel, additive=additive)
    assert not res["violations"], (w, md, res["violations"][:5])
    assert res["tie_swaps"] <= max(1, res["rows"] // 20), res
    rows = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)]
    parity.assert_prefill_out(out, (q, k, v), w.block, ref["out"], rows, res, sel_idx, sel_cnt,
                              ref["off"], w.torch_dtype, f"{w} {md}")
