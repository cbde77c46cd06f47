"""Parity of the method parameterisations (stem_method_t) with the CPU oracle, on a B200.

The pages' own forms: the linear position-decay budget (gist.science/es "Resumen tecnico" 2.A
and its translations), the additive output-aware metric s + beta * max(0, log n^2) (es 2.B,
it 2.B, nl OAM, fr 2.B) and the max-pooled V magnitude (nl Implementatie step 1), alone and
combined, through the same C-ABI calls as the default path. Stage by stage (each stage fed the
oracle's upstream values) and end to end.
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

METHODS = {
    # the pages' parameterisation with their ablation optimum mu = 0.7, beta = 0.2
    "pages": dict(schedule="linear", k_start=12.0, mu=0.7, k_min=4, metric="additive", beta=0.2,
                  clamp=True, vsum="max"),
    "linear-product": dict(schedule="linear", k_start=9.5, mu=0.35, k_min=3),
    "additive-noclamp": dict(schedule="exp", rho_min=0.2, tau=4.0, k_min=3, metric="additive",
                             beta=0.2, clamp=False),
    "routing-only": dict(schedule="exp", rho_min=0.2, tau=4.0, k_min=3, metric="additive",
                         beta=0.0),
    "product-vmax": dict(schedule="exp", rho_min=0.2, tau=4.0, k_min=3, vsum="max"),
    # GQA-group-shared selection (one list per kv-head group)
    "group-product": dict(schedule="exp", rho_min=0.2, tau=4.0, k_min=3, share="group"),
    "group-pages": dict(schedule="linear", k_start=12.0, mu=0.7, k_min=4, metric="additive",
                        beta=0.2, clamp=True, vsum="max", share="group"),
}

WORKLOADS = {
    "llama-4k": wl.LLAMA_32K.replace(name="llama-4k", Hq=8, Hkv=2, S=4096),
    "qwen-3k": wl.QWEN_64K.replace(name="qwen-3k", Hq=7, Hkv=1, S=3072, tau=6.0),
    "bf16-d64-blk64": wl.LLAMA_32K.replace(name="bf16-d64-blk64", Hq=4, Hkv=2, S=2560, D=64,
                                           block=64, tau=8.0),
    "f32-d128-blk128": wl.TINY.replace(name="f32-d128-blk128", Hq=4, Hkv=2, S=2048, D=128,
                                       block=128),
}

CASES = ([(m, "llama-4k") for m in METHODS] +
         [(m, w) for m in ("pages", "group-product") for w in WORKLOADS if w != "llama-4k"])


def _method(name):
    return S.make_method(**METHODS[name])


def _oracle_kwargs(name):
    d = METHODS[name]
    return dict(rho_min=d.get("rho_min", 1.0), tau=d.get("tau", 1.0), k_min=d["k_min"],
                schedule=d.get("schedule", "exp"), k_start=d.get("k_start", 0.0),
                mu=d.get("mu", 1.0), metric_form=d.get("metric", "product"),
                beta=d.get("beta", 0.0), clamp=d.get("clamp", True), vsum=d.get("vsum", "mean"),
                share=d.get("share", "head"))


def _oracle_budget(name, nb):
    d = _oracle_kwargs(name)
    if d["schedule"] == "linear":
        return oracle.budget_linear(nb, d["k_start"], d["mu"], d["k_min"])
    return oracle.budget(nb, d["rho_min"], d["tau"], d["k_min"])


def _oracle_metric(name, qbar, kbar, vnorm):
    """Per-head metric [B, Hq, T]; for group sharing the group metric replicated per head."""
    d = _oracle_kwargs(name)
    if d["metric_form"] == "additive":
        m = oracle.metric_additive(qbar, kbar, vnorm, d["beta"], d["clamp"])
    else:
        m = oracle.metric(qbar, kbar, vnorm)
    if d["share"] == "group":
        G = qbar.shape[1] // kbar.shape[1]
        m = np.repeat(oracle.metric_group(m, G), G, axis=1)
    return m


def _oracle_select(name, m, kk, off, G):
    if _oracle_kwargs(name)["share"] == "group":
        return oracle.select_group(m[:, ::G], kk, off, G)
    return oracle.select(m, kk, off)


def inputs(w):
    q, k, v = wl.make_inputs(w, "cpu")
    return (q, k, v), (q.to(DEV), k.to(DEV), v.to(DEV))


@pytest.mark.parametrize("wname", list(WORKLOADS))
def test_pool_vmax(wname):
    w = WORKLOADS[wname]
    cpu, dev = inputs(w)
    qbar, kbar, vnorm = S.stem_pool(*dev, w.block, method=_method("pages"))
    torch.cuda.synchronize()
    rq, rk, rn = oracle.pool(*cpu, w.block, "max")
    for got, ref, x in ((qbar, rq, cpu[0]), (kbar, rk, cpu[1])):
        atol = 1e-6 * float(x.float().abs().max())
        np.testing.assert_allclose(got.double().cpu().numpy(), ref, rtol=0, atol=atol)
    # one row's float32 sum of D squares, then a correctly rounded sqrt
    np.testing.assert_allclose(vnorm.double().cpu().numpy(), rn, rtol=2e-6)


@pytest.mark.parametrize("mname,wname", CASES)
def test_select_from_oracle_pooling(mname, wname):
    w = WORKLOADS[wname]
    d = _oracle_kwargs(mname)
    cpu, _ = inputs(w)
    rq, rk, rn = oracle.pool(*cpu, w.block, d["vsum"])
    q32, k32, n32 = (torch.from_numpy(x).float() for x in (rq, rk, rn))
    m = _oracle_metric(mname, q32.double().numpy(), k32.double().numpy(), n32.double().numpy())
    kk, off = _oracle_budget(mname, w.nb)
    ref_idx, ref_cnt = _oracle_select(mname, m, kk, off, w.Hq // w.Hkv)
    sel_idx, sel_cnt, m_gpu = S.stem_select(q32.to(DEV), k32.to(DEV), n32.to(DEV), 0.0, 0.0, 0,
                                            with_metric=True, method=_method(mname))
    torch.cuda.synchronize()
    additive = d["metric_form"] == "additive"
    res = parity.compare_selection(sel_idx, sel_cnt, ref_idx, ref_cnt, m, kk, off,
                                   additive=additive)
    assert not res["violations"], res["violations"][:5]
    assert res["tie_swaps"] <= max(1, res["rows"] // 100), res
    mg = m_gpu.double().cpu().numpy()
    if additive:  # float32 scores: |error| ~ 1e-7 * (|s| + |beta e|)
        np.testing.assert_allclose(mg, m, rtol=0, atol=2e-5 * max(1.0, float(np.abs(m).max())))
    else:
        np.testing.assert_allclose(mg, m, rtol=2e-5, atol=1e-30)
    if _oracle_kwargs(mname)["share"] == "group":  # every head of a group keeps the same list
        G = w.Hq // w.Hkv
        si = sel_idx.cpu().numpy()[:, :, :int(off[-1])]
        for h in range(w.Hq):
            assert np.array_equal(si[:, h], si[:, (h // G) * G])


@pytest.mark.parametrize("mname,wname", CASES)
def test_end_to_end(mname, wname):
    w = WORKLOADS[wname]
    cpu, dev = inputs(w)
    ref = oracle.prefill(*cpu, w.block, **_oracle_kwargs(mname))
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    out, sel_idx, sel_cnt = S.stem_prefill_ex(*dev, w.block, 0.0, 0.0, 0, status=status,
                                              method=_method(mname))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    res = parity.compare_selection(sel_idx, sel_cnt, ref["sel_idx"], ref["sel_cnt"], ref["m"],
                                   ref["k"], ref["off"],
                                   additive=_oracle_kwargs(mname)["metric_form"] == "additive")
    assert not res["violations"], res["violations"][:5]
    assert res["tie_swaps"] <= max(1, res["rows"] // 100), res
    rows = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)]
    parity.assert_prefill_out(out, cpu, w.block, ref["out"], rows, res, sel_idx, sel_cnt,
                              ref["off"], w.torch_dtype, f"{mname}/{wname}")


def test_stage_calls_with_method_match_the_full_path():
    """pool_m -> select_m -> sparse_attn_m reproduce stem_prefill_ex(method) bit for bit."""
    w = WORKLOADS["llama-4k"]
    _, dev = inputs(w)
    m = _method("pages")
    out, sel_idx, sel_cnt = S.stem_prefill_ex(*dev, w.block, 0.0, 0.0, 0, method=m)
    qbar, kbar, vnorm = S.stem_pool(*dev, w.block, method=m)
    si, sc, _ = S.stem_select(qbar, kbar, vnorm, 0.0, 0.0, 0, method=m)
    o2 = S.stem_sparse_attn(*dev, w.block, 0.0, 0.0, 0, si, sc, method=m)
    torch.cuda.synchronize()
    assert torch.equal(si, sel_idx) and torch.equal(sc, sel_cnt)
    assert torch.equal(o2, out)


def test_host_api_with_method():
    w = WORKLOADS["llama-4k"]
    cpu, dev = inputs(w)
    m = _method("pages")
    out_d, si_d, sc_d = S.stem_prefill_ex(*dev, w.block, 0.0, 0.0, 0, method=m)
    torch.cuda.synchronize()
    out_h, si_h, sc_h = (torch.empty_like(x, device="cpu").pin_memory()
                         for x in (out_d, si_d, sc_d))
    S.stem_prefill_host(*(t.pin_memory() for t in cpu), w.block, 0.0, 0.0, 0, out_h, si_h, sc_h,
                        method=m)
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(si_h, si_d.cpu())
    assert torch.equal(sc_h, sc_d.cpu())
