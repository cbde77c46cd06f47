"""Parity of block scoring by anti-diagonal sampling (stem_method_t score = antidiag) with the
CPU oracle, on a B200.

The estimator ("Stem: Rethinking Causal Information Flow in Sparse Attention", gist.science/fr
"Resume technique" 2.C step 1) runs on the tensor cores: each a_uw is a sum of stride*D exact
bfloat16 products accumulated in float32. Its tolerance is derived from that arithmetic and the
inputs, never from the GPU's output:
  |da_uw| <= stride*D * 2^-24 * |Q'_u| |K'_w| / (stride sqrt(D))   (float32 summation bound,
                                                                      Cauchy-Schwarz)
  |dp_ij| / p_ij <= exp(2 max|da|) - 1 + 2e-5                       (softmax of perturbed a;
                                                                      float32 exp2 and sums)
Selections may differ from the oracle's only where the two swapped blocks' oracle metrics are
within twice that relative error (then both selections are correct up to the arithmetic).
"""

import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

WORKLOADS = {
    "llama-4k": wl.LLAMA_32K.replace(name="llama-4k", Hq=8, Hkv=2, S=4096),
    "llama-ragged": wl.LLAMA_32K.replace(name="llama-ragged", Hq=4, Hkv=2, S=4096 - 48),
    "qwen-3k": wl.QWEN_64K.replace(name="qwen-3k", Hq=7, Hkv=1, S=3072, tau=6.0),
    "d64-blk64": wl.LLAMA_32K.replace(name="d64-blk64", Hq=4, Hkv=2, S=2560, D=64, block=64,
                                      tau=8.0),
    "short": wl.LLAMA_32K.replace(name="short", Hq=2, Hkv=1, S=200, tau=2.0),
}

P_CASES = [("llama-4k", 16), ("llama-4k", 4), ("llama-4k", 32), ("llama-4k", 64),
           ("llama-4k", 128), ("llama-ragged", 16), ("qwen-3k", 16), ("d64-blk64", 8),
           ("d64-blk64", 2), ("short", 8)]


def inputs(w):
    q, k, v = wl.make_inputs(w, "cpu")
    return (q, k, v), (q.to(DEV), k.to(DEV), v.to(DEV))


def a_error_bound(q, k, stride):
    """Largest |a_uw| error of a float32 sum of stride*D exact products (see module doc)."""
    B, Hq, Sq, D = q.shape
    qn = q.double().reshape(B, Hq, Sq // stride, stride * D).norm(dim=-1).max().item()
    kn = k.double().reshape(B, k.shape[1], Sq // stride, stride * D).norm(dim=-1).max().item()
    n = stride * D
    return n * 2.0 ** -24 * qn * kn / (stride * math.sqrt(D))


def p_rel_tol(q, k, stride):
    return math.expm1(2.0 * a_error_bound(q, k, stride)) + 2e-5


def method(w, stride, **kw):
    d = dict(schedule="exp", rho_min=w.rho_min, tau=w.tau, k_min=w.k_min, score="antidiag",
             stride=stride)
    d.update(kw)
    return S.make_method(**d)


@pytest.mark.parametrize("wname,stride", P_CASES)
def test_block_probabilities(wname, stride):
    w = WORKLOADS[wname]
    cpu, dev = inputs(w)
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    p = S.stem_antidiag(dev[0], dev[1], w.block, method(w, stride), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.antidiag(cpu[0], cpu[1], w.block, stride)
    got = p.double().cpu().numpy()
    tol = p_rel_tol(cpu[0], cpu[1], stride)
    err = np.abs(got - ref)
    assert np.all(err <= tol * ref + 1e-12), (float((err / np.maximum(ref, 1e-300)).max()), tol)
    # typical error far below the worst-case bound
    assert float(np.median(err / np.maximum(ref, 1e-300))) < 1e-5
    # every row of p sums to 1 over j <= i
    for i in range(w.nb):
        s = got[:, :, i * (i + 1) // 2:i * (i + 1) // 2 + i + 1].sum(axis=-1)
        np.testing.assert_allclose(s, 1.0, rtol=0, atol=1e-4)


SEL_CASES = [("llama-4k", 16, {}), ("llama-4k", 16, dict(metric="additive", beta=0.2)),
             ("llama-4k", 16, dict(share="group")),
             ("llama-4k", 16, dict(share="group", metric="additive", beta=0.2, vsum="max")),
             ("llama-ragged", 16, {}), ("qwen-3k", 32, dict(metric="additive", beta=0.0)),
             ("d64-blk64", 8, dict(schedule="linear", k_start=10.0, mu=0.7, k_min=4)),
             ("short", 8, {})]


def _oracle_kwargs(w, stride, kw):
    return dict(rho_min=w.rho_min, tau=w.tau, k_min=kw.get("k_min", w.k_min),
                schedule=kw.get("schedule", "exp"), k_start=kw.get("k_start", 0.0),
                mu=kw.get("mu", 1.0), metric_form=kw.get("metric", "product"),
                beta=kw.get("beta", 0.0), clamp=kw.get("clamp", True), vsum=kw.get("vsum", "mean"),
                share=kw.get("share", "head"), score="antidiag", stride=stride)


def _sel_rel(cpu, stride, additive):
    t = p_rel_tol(cpu[0], cpu[1], stride)
    # product metrics: relative gap of p n; additive: absolute gap of ln p (+ float32 beta e)
    return 2.0 * (t if not additive else math.log1p(t) + 1e-6)


@pytest.mark.parametrize("wname,stride,kw", SEL_CASES,
                         ids=[f"{a}-{b}-{'-'.join(f'{k}={v}' for k, v in c.items()) or 'default'}"
                              for a, b, c in SEL_CASES])
def test_end_to_end(wname, stride, kw):
    w = WORKLOADS[wname]
    cpu, dev = inputs(w)
    ok = _oracle_kwargs(w, stride, kw)
    ref = oracle.prefill(*cpu, w.block, **ok)
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    out, sel_idx, sel_cnt = S.stem_prefill_ex(*dev, w.block, 0.0, 0.0, 0, status=status,
                                              method=method(w, stride, **kw))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    additive = ok["metric_form"] == "additive"
    res = parity.compare_selection(sel_idx, sel_cnt, ref["sel_idx"], ref["sel_cnt"], ref["m"],
                                   ref["k"], ref["off"], rel=_sel_rel(cpu, stride, additive),
                                   additive=additive)
    assert not res["violations"], res["violations"][:5]
    assert res["tie_swaps"] <= max(1, res["rows"] // 20), res
    if ok["share"] == "group":
        G = w.Hq // w.Hkv
        si = sel_idx.cpu().numpy()[:, :, :int(ref["off"][-1])]
        for h in range(w.Hq):
            assert np.array_equal(si[:, h], si[:, (h // G) * G])
    rows = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)]
    parity.assert_prefill_out(out, cpu, w.block, ref["out"], rows, res, sel_idx, sel_cnt,
                              ref["off"], w.torch_dtype, f"antidiag/{wname}")


def test_stage_calls_match_the_full_path():
    """pool_m -> antidiag_m -> select_p_m -> sparse_attn_m reproduce stem_prefill_ex bit for
    bit, and the host-buffer API matches the device one."""
    w = WORKLOADS["llama-4k"]
    cpu, dev = inputs(w)
    m = method(w, 16, metric="additive", beta=0.2)
    out, sel_idx, sel_cnt = S.stem_prefill_ex(*dev, w.block, 0.0, 0.0, 0, method=m)
    _, _, vnorm = S.stem_pool(*dev, w.block, method=m)
    p = S.stem_antidiag(dev[0], dev[1], w.block, m)
    si, sc, _ = S.stem_select_p(p, vnorm, w.Hq, m)
    o2 = S.stem_sparse_attn(*dev, w.block, 0.0, 0.0, 0, si, sc, method=m)
    torch.cuda.synchronize()
    assert torch.equal(si, sel_idx) and torch.equal(sc, sel_cnt)
    assert torch.equal(o2, out)
    out_h, si_h, sc_h = (torch.empty_like(x, device="cpu").pin_memory()
                         for x in (out, sel_idx, sel_cnt))
    S.stem_prefill_host(*(t.pin_memory() for t in cpu), w.block, 0.0, 0.0, 0, out_h, si_h, sc_h,
                        method=m)
    assert torch.equal(out_h, out.cpu()) and torch.equal(si_h, sel_idx.cpu())
    assert torch.equal(sc_h, sel_cnt.cpu())


def test_select_p_metric_output():
    """stem_select_p_m from the oracle's own p (rounded to float32): the diagnostic metric and
    the selection against the oracle's metric of those same values."""
    w = WORKLOADS["qwen-3k"]
    cpu, _ = inputs(w)
    p_ref = oracle.antidiag(cpu[0], cpu[1], w.block, 16)
    _, _, vn = oracle.pool(*cpu, w.block)
    p32 = torch.from_numpy(p_ref).float()
    n32 = torch.from_numpy(vn).float()
    for kw in ({}, dict(metric="additive", beta=0.2, clamp=False)):
        m = method(w, 16, **kw)
        form = kw.get("metric", "product")
        mref = oracle.metric_from_p(p32.double().numpy(), n32.double().numpy(), kw.get("beta", 0.0),
                                    kw.get("clamp", True), form)
        kk, off = oracle.budget(w.nb, w.rho_min, w.tau, w.k_min)
        ref_idx, ref_cnt = oracle.select(mref, kk, off)
        si, sc, mg = S.stem_select_p(p32.to(DEV), n32.to(DEV), w.Hq, m, with_metric=True)
        torch.cuda.synchronize()
        res = parity.compare_selection(si, sc, ref_idx, ref_cnt, mref, kk, off,
                                       additive=form == "additive")
        assert not res["violations"], res["violations"][:5]
        assert res["tie_swaps"] <= max(1, res["rows"] // 100), res
        mgd = mg.double().cpu().numpy()
        if form == "additive":
            np.testing.assert_allclose(mgd, mref, rtol=0, atol=2e-5 * max(1.0, np.abs(mref).max()))
        else:
            np.testing.assert_allclose(mgd, mref, rtol=2e-6, atol=1e-35)


def _full_rows(w, seed=11, n_random=9):
    import random

    rng = random.Random(seed)
    rows = {(0, 0, 0), (0, 0, 1), (0, w.Hq - 1, w.nb - 1), (w.B - 1, 0, w.nb - 1)}
    while len(rows) < 4 + n_random:
        rows.add((rng.randrange(w.B), rng.randrange(w.Hq), rng.randrange(w.nb)))
    return sorted(rows)


@pytest.mark.slow
@pytest.mark.parametrize("w", [wl.LLAMA_128K, wl.QWEN_64K], ids=lambda w: w.name)
def test_full_size_sampled(w):
    """The bench's workloads at full size, in its launch configuration (stem_prefill_ex with a
    caller workspace on torch's stream): every row of p sums to 1; sampled rows of p, their
    selections and their outputs against the oracle computed row by row."""
    stride = 16
    m = method(w, stride)
    q, k, v = wl.make_inputs(w, DEV)
    out, sel_idx, sel_cnt = S.alloc_outputs(q, k, w.block, w.rho_min, w.tau, w.k_min, m)
    ws = S.alloc_workspace(q, k, w.block, m)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    S.stem_prefill_ex(q, k, v, w.block, 0.0, 0.0, 0, out, sel_idx, sel_cnt, ws, status,
                      method=m)
    p = S.stem_antidiag(q, k, w.block, m)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # row sums, every row (a float32 sum of up to nb values each)
    tri_i = torch.repeat_interleave(torch.arange(w.nb, device=DEV),
                                    torch.arange(1, w.nb + 1, device=DEV))
    sums = torch.zeros((w.B, w.Hq, w.nb), dtype=torch.float64, device=DEV)
    sums.index_add_(2, tri_i, p.double())
    assert float((sums - 1.0).abs().max()) < 1e-4
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    rows = _full_rows(w)
    pref = oracle.antidiag(qc, kc, w.block, stride, rows=rows)
    tol = p_rel_tol(qc, kc, stride)
    pc = p.cpu().double().numpy()
    # selection of the sampled rows from the oracle's p rows (other rows: placeholders)
    _, _, vn = oracle.pool(qc, kc, vc, w.block)
    kk, off = oracle.budget(w.nb, w.rho_min, w.tau, w.k_min)
    pp = np.ones((w.B, w.Hq, w.nb * (w.nb + 1) // 2))
    for (b, h, i), r in zip(rows, pref):
        lo = i * (i + 1) // 2
        got = pc[b, h, lo:lo + i + 1]
        assert np.all(np.abs(got - r[:i + 1]) <= tol * r[:i + 1] + 1e-12), (b, h, i)
        pp[b, h, lo:lo + i + 1] = r[:i + 1]
    mref = oracle.metric_from_p(pp, vn)
    ref_idx, ref_cnt = oracle.select(mref, kk, off)
    si = sel_idx.cpu().numpy()
    rel = _sel_rel((qc, kc), stride, False)
    keep = []
    for (b, h, i) in rows:
        assert int(sel_cnt[b, h, i]) == int(kk[i])
        g = si[b, h, off[i]:off[i + 1]]
        r = ref_idx[b, h, off[i]:off[i + 1]]
        if np.array_equal(g, r):
            keep.append((b, h, i))
            continue
        extra, missing = np.setdiff1d(g, r), np.setdiff1d(r, g)
        mrow = oracle.metric_row(mref, b, h, i)
        hi, lo_ = mrow[missing].max(), mrow[extra].min()
        assert hi - lo_ <= rel * hi, ((b, h, i), extra, missing)
    assert len(keep) >= len(rows) - 2
    ref_out = oracle.attention(qc, kc, vc, w.block, ref_idx, ref_cnt, off, keep)
    parity.assert_out_close(parity.out_rows(out, keep, w.block), ref_out, w.torch_dtype,
                            f"antidiag/{w.name}")
    # rows whose selection is a near-tie swap: the oracle's attention over the GPU's own list
    swapped = [r for r in rows if r not in set(keep)]
    if swapped:
        gi, gc = parity.gpu_csr(sel_idx, sel_cnt, w.B, w.Hq, w.nb, int(off[w.nb]))
        ref_sw = oracle.attention(qc, kc, vc, w.block, gi, gc, off, swapped)
        parity.assert_out_close(parity.out_rows(out, swapped, w.block), ref_sw, w.torch_dtype,
                                f"antidiag/{w.name} (tie rows)")
