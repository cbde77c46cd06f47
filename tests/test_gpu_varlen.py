"""Variable-length batches (stem_prefill_varlen) on a B200: sequences of different lengths
(an empty one, one shorter than a block, ragged ones) packed back to back; each must match the
oracle run on that sequence alone, and bit for bit the library's own single-sequence call."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import parity, test_gpu_antidiag

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = {
    "bf16-blk128": (wl.LLAMA_32K.replace(name="varlen", Hq=8, Hkv=2), [4096, 77, 0, 2573],
                    dict(schedule="exp", rho_min=0.2, tau=6.0, k_min=3)),
    "bf16-pages": (wl.LLAMA_32K.replace(name="varlen", Hq=8, Hkv=2), [1500, 3200],
                   dict(schedule="linear", k_start=10.0, mu=0.7, k_min=3, metric="additive",
                        beta=0.2, vsum="max")),
    "bf16-blk64": (wl.LLAMA_32K.replace(name="varlen", Hq=4, Hkv=2, block=64), [700, 1300, 64],
                   dict(schedule="exp", rho_min=0.3, tau=4.0, k_min=2)),
    "f32": (wl.TINY.replace(name="varlen", Hq=4, Hkv=2, D=128, block=128), [900, 130],
            dict(schedule="exp", rho_min=0.3, tau=4.0, k_min=2)),
    # block scores by anti-diagonal sampling (every length a multiple of the 16-token group)
    "bf16-antidiag": (wl.LLAMA_32K.replace(name="varlen", Hq=8, Hkv=2), [2048, 80, 0, 1600],
                      dict(schedule="exp", rho_min=0.2, tau=6.0, k_min=3, score="antidiag",
                           stride=16)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_varlen_matches_each_sequence(name):
    w, lengths, md = CASES[name]
    m = S.make_method(**md)
    seqs = [wl.make_inputs(w.replace(S=max(L, 1), seed=w.seed + 11 * n), "cpu")
            for n, L in enumerate(lengths)]
    seqs = [tuple(t[:, :, :L].contiguous() for t in qkv) for qkv, L in zip(seqs, lengths)]
    q, cu = S.pack_varlen([s_[0][0] for s_ in seqs])
    k, _ = S.pack_varlen([s_[1][0] for s_ in seqs])
    v, _ = S.pack_varlen([s_[2][0] for s_ in seqs])
    assert cu == [0] + list(np.cumsum(lengths))
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    out, si, sc = S.stem_prefill_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu, w.Hq, w.Hkv, w.D,
                                        w.block, m, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    out, si, sc = out.cpu(), si.cpu(), sc.cpu()
    capo = nbo = 0
    okw = dict(rho_min=md.get("rho_min", 1.0), tau=md.get("tau", 1.0), k_min=md["k_min"],
               schedule=md["schedule"], k_start=md.get("k_start", 0.0), mu=md.get("mu", 1.0),
               metric_form=md.get("metric", "product"), beta=md.get("beta", 0.0),
               vsum=md.get("vsum", "mean"), score=md.get("score", "pooled"),
               stride=md.get("stride", 16))
    for (qs, ks, vs), L, t0 in zip(seqs, lengths, cu[:-1]):
        if L == 0:
            continue
        nb = -(-L // w.block)
        ref = oracle.prefill(qs, ks, vs, w.block, **okw)
        cap = int(ref["off"][-1])
        g_out = out[w.Hq * w.D * t0: w.Hq * w.D * (t0 + L)].view(1, w.Hq, L, w.D)
        g_si = si[w.Hq * capo: w.Hq * (capo + cap)].view(1, w.Hq, cap)
        g_sc = sc[w.Hq * nbo: w.Hq * (nbo + nb)].view(1, w.Hq, nb)
        # anti-diagonal scores: near-ties within the bound derived from their arithmetic
        rel = (2.0 * test_gpu_antidiag.p_rel_tol(qs, ks, md["stride"])
               if md.get("score") == "antidiag" else parity.REL_TIE)
        res = parity.compare_selection(g_si, g_sc, ref["sel_idx"], ref["sel_cnt"], ref["m"],
                                       ref["k"], ref["off"], rel=rel,
                                       additive=md.get("metric") == "additive")
        assert not res["violations"], (L, res["violations"][:5])
        rows = [(0, h, i) for h in range(w.Hq) for i in range(nb)]
        parity.assert_prefill_out(g_out, (qs, ks, vs), w.block, ref["out"], rows, res, g_si,
                                  g_sc, ref["off"], w.torch_dtype, f"{name} L={L}")
        # bit for bit the single-sequence call
        o1, s1, c1 = S.stem_prefill_ex(qs.to(DEV), ks.to(DEV), vs.to(DEV), w.block, 0.0, 0.0, 0,
                                       method=m)
        torch.cuda.synchronize()
        assert torch.equal(o1.cpu(), g_out) and torch.equal(s1.cpu(), g_si)
        assert torch.equal(c1.cpu(), g_sc)
        capo += cap
        nbo += nb
