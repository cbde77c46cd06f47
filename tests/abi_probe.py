"""Invalid-argument probes of the C ABI, run in a subprocess with CUDA_VISIBLE_DEVICES=''.

Every call here must be rejected by host-side validation before anything touches CUDA; with
the devices hidden, a validation bug could not launch a kernel anyway. Prints one JSON object
{case: return code}.
"""

import ctypes
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
assert os.environ.get("CUDA_VISIBLE_DEVICES") == "", "run with CUDA_VISIBLE_DEVICES=''"

from block_sparse_causal_pooling_b200 import stem as S  # noqa: E402

L = S.lib()
FAKE = 0x7F0000000000  # 256-byte aligned, never dereferenced


def base(**kw):
    a = S.stem_args_t()
    a.q = a.k = a.v = FAKE
    a.out = FAKE + 0x100
    a.sel_idx = FAKE + 0x200
    a.sel_cnt = FAKE + 0x300
    a.B, a.Hq, a.Hkv, a.S, a.D, a.block = 1, 4, 2, 1024, 128, 128
    a.rho_min, a.tau, a.k_min, a.dtype = 0.25, 4.0, 2, 0
    a.workspace = FAKE + 0x1000
    a.workspace_bytes = 1 << 30
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def ex(**kw):
    return L.stem_prefill_ex(ctypes.byref(base(**kw)), None)


res = {
    "hq_not_multiple": ex(Hq=3),
    "hkv_zero": ex(Hkv=0),
    "d_96": ex(D=96),
    "block_32": ex(block=32),
    "negative_S": ex(S=-128),
    "negative_B": ex(B=-1),
    "dtype_7": ex(dtype=7),
    "rho_zero": ex(rho_min=0.0),
    "rho_above_one": ex(rho_min=1.5),
    "rho_nan": ex(rho_min=float("nan")),
    "tau_zero": ex(tau=0.0),
    "tau_inf": ex(tau=float("inf")),
    "kmin_zero": ex(k_min=0),
    "q_null": ex(q=None),
    "out_null": ex(out=None),
    "q_misaligned": ex(q=FAKE + 8),
    "sel_idx_misaligned": ex(sel_idx=FAKE + 2),
    "status_misaligned": ex(status=FAKE + 2),
    "workspace_null": ex(workspace=None),
    "workspace_small": ex(workspace_bytes=1024),
    "workspace_misaligned": ex(workspace=FAKE + 16),
    "nb_too_large": ex(S=(S.STEM_MAX_NB + 1) * 128),
    "empty_B": ex(B=0, q=None, k=None, v=None, out=None, sel_idx=None, sel_cnt=None),
    "empty_S": ex(S=0, q=None, k=None, v=None, out=None, sel_idx=None, sel_cnt=None),
    "ex_null_args": L.stem_prefill_ex(None, None),
    "host_null_args": L.stem_prefill_host(None),
    "host_bad_block": L.stem_prefill_host(ctypes.byref(base(block=96))),
    "simple_bad_block": L.stem_prefill(FAKE, FAKE, FAKE, 1, 4, 2, 1024, 128, 96, 0.25, 4.0, 2,
                                       FAKE, FAKE, FAKE),
    "simple_bad_rho": L.stem_prefill(FAKE, FAKE, FAKE, 1, 4, 2, 1024, 128, 128, -0.1, 4.0, 2,
                                     FAKE, FAKE, FAKE),
    "pool_bad_dtype": L.stem_pool(FAKE, FAKE, FAKE, 5, 1, 4, 2, 1024, 128, 128, FAKE, FAKE,
                                  FAKE, None),
    "pool_null_out": L.stem_pool(FAKE, FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128, None, FAKE,
                                 FAKE, None),
    "pool_misaligned_qbar": L.stem_pool(FAKE, FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128, FAKE + 4,
                                        FAKE, FAKE, None),
    "select_bad_kmin": L.stem_select(FAKE, FAKE, FAKE, 1, 4, 2, 8, 128, 0.25, 4.0, 0, FAKE,
                                     FAKE, None, FAKE, 1 << 20, None),
    "select_nb_too_large": L.stem_select(FAKE, FAKE, FAKE, 1, 4, 2, S.STEM_MAX_NB + 1, 128,
                                         0.25, 4.0, 2, FAKE, FAKE, None, FAKE, 1 << 30, None),
    "select_no_workspace": L.stem_select(FAKE, FAKE, FAKE, 1, 4, 2, 8, 128, 0.25, 4.0, 2, FAKE,
                                         FAKE, None, None, 0, None),
    "attn_bad_hq": L.stem_sparse_attn(FAKE, FAKE, FAKE, 0, 1, 5, 2, 1024, 128, 128, 0.25, 4.0,
                                      2, FAKE, FAKE, FAKE, FAKE, 1 << 20, None, None),
    "attn_small_workspace": L.stem_sparse_attn(FAKE, FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128,
                                               0.25, 4.0, 2, FAKE, FAKE, FAKE, FAKE, 16, None,
                                               None),
    "budget_bad_tau": L.stem_budget(8, 0.5, -1.0, 2, None, None),
    "static_bad_kmin": L.stem_select_static(FAKE, FAKE, FAKE, 1, 4, 2, 8, 128, 0.25, 4.0, 0,
                                            FAKE, FAKE, None),
    "static_nb_too_large": L.stem_select_static(FAKE, FAKE, FAKE, 1, 4, 2, S.STEM_MAX_NB + 1,
                                                128, 0.25, 4.0, 2, FAKE, FAKE, None),
    "static_null_out": L.stem_select_static(FAKE, FAKE, FAKE, 1, 4, 2, 8, 128, 0.25, 4.0, 2,
                                            None, FAKE, None),
    "capacity_bad_rho": L.stem_sel_capacity(8, 0.0, 4.0, 2),
}

# method-parameterised calls: an invalid stem_method_t field is rejected the same way
BAD_MU = S.make_method("linear", k_start=8.0, mu=0.0, k_min=2)
BAD_BETA = S.make_method("exp", rho_min=0.25, tau=4.0, k_min=2, metric="additive", beta=-1.0)
BAD_VSUM = S.make_method("exp", rho_min=0.25, tau=4.0, k_min=2)
BAD_VSUM.vsum = 7
GOOD = S.make_method("linear", k_start=8.0, mu=0.7, k_min=2, metric="additive", beta=0.2)
BAD_SHARE = S.make_method("exp", rho_min=0.25, tau=4.0, k_min=2)
BAD_SHARE.share = 3
GROUP = S.make_method("exp", rho_min=0.25, tau=4.0, k_min=2, share="group")
M = lambda m: ctypes.byref(m)  # noqa: E731
def varlen(cu, method=GOOD, **kw):
    a = S.stem_varlen_args_t()
    a.q = a.k = a.v = FAKE
    a.out, a.sel_idx, a.sel_cnt = FAKE + 0x100, FAKE + 0x200, FAKE + 0x300
    arr = (ctypes.c_int32 * len(cu))(*cu)
    a.nseq, a.cu_seqlens = len(cu) - 1, arr
    a.Hq, a.Hkv, a.D, a.block, a.dtype = 4, 2, 128, 128, 0
    a.method = ctypes.pointer(method) if method is not None else None
    a.workspace, a.workspace_bytes = FAKE + 0x1000, 1 << 30
    for key, val in kw.items():
        setattr(a, key, val)
    return L.stem_prefill_varlen(ctypes.byref(a), None)


res.update({
    "varlen_decreasing_cu": varlen([0, 300, 200]),
    "varlen_cu0_nonzero": varlen([5, 300]),
    "varlen_no_method": varlen([0, 300], method=None),
    "varlen_bad_hq": varlen([0, 300], Hq=3),
    "varlen_q_null": varlen([0, 300], q=None),
    "varlen_small_workspace": varlen([0, 300], workspace_bytes=64),
    "varlen_all_empty": varlen([0, 0, 0], q=None, k=None, v=None, out=None, sel_idx=None,
                               sel_cnt=None),
    "method_bad_mu": ex(method=ctypes.pointer(BAD_MU)),
    "method_bad_beta": ex(method=ctypes.pointer(BAD_BETA)),
    "method_bad_vsum": ex(method=ctypes.pointer(BAD_VSUM)),
    "method_bad_share": ex(method=ctypes.pointer(BAD_SHARE)),
    "group_nb_too_large": ex(S=1025 * 128, method=ctypes.pointer(GROUP)),
    "method_overrides_bad_rho": ex(rho_min=-1.0, method=ctypes.pointer(BAD_MU)),
    "host_method_bad": L.stem_prefill_host(ctypes.byref(base(method=ctypes.pointer(BAD_BETA)))),
    "pool_m_bad_vsum": L.stem_pool_m(FAKE, FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128, M(BAD_VSUM),
                                     FAKE, FAKE, FAKE, None),
    "pool_m_null_method": L.stem_pool_m(FAKE, FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128, None,
                                        FAKE, FAKE, FAKE, None),
    "select_m_bad_mu": L.stem_select_m(FAKE, FAKE, FAKE, 1, 4, 2, 8, 128, M(BAD_MU), FAKE, FAKE,
                                       None, FAKE, 1 << 20, None),
    "select_m_null_method": L.stem_select_m(FAKE, FAKE, FAKE, 1, 4, 2, 8, 128, None, FAKE, FAKE,
                                            None, FAKE, 1 << 20, None),
    "select_m_no_workspace": L.stem_select_m(FAKE, FAKE, FAKE, 1, 4, 2, 8, 128, M(GOOD), FAKE,
                                             FAKE, None, None, 0, None),
    "attn_m_bad_beta": L.stem_sparse_attn_m(FAKE, FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128,
                                            M(BAD_BETA), FAKE, FAKE, FAKE, FAKE, 1 << 20, None,
                                            None),
    "attn_m_bad_block": L.stem_sparse_attn_m(FAKE, FAKE, FAKE, 0, 1, 4, 2, 1000, 128, 96, M(GOOD),
                                          FAKE, FAKE, FAKE, FAKE, 1 << 20, None, None),
})

# anti-diagonal scoring: stride rules and the estimator's entry points
AD = S.make_method("exp", rho_min=0.25, tau=4.0, k_min=2, score="antidiag", stride=16)
def ad(**kw):
    m = S.stem_method_t.from_buffer_copy(AD)
    for key, val in kw.items():
        setattr(m, key, val)
    return m


res.update({
    "ad_stride_not_pow2": ex(method=ctypes.pointer(ad(stride=12))),
    "ad_stride_zero": ex(method=ctypes.pointer(ad(stride=0))),
    "ad_stride_above_block": ex(method=ctypes.pointer(ad(stride=256))),
    "ad_too_many_groups": ex(method=ctypes.pointer(ad(stride=2))),
    "ad_S_not_multiple": ex(S=1000, method=ctypes.pointer(ad())),
    "ad_f32": ex(dtype=1, method=ctypes.pointer(ad())),
    "ad_bad_score": ex(method=ctypes.pointer(ad(score=5))),
    # the pooled method's workspace lacks the estimator's regions
    "ad_small_workspace": ex(workspace_bytes=L.stem_workspace_size(1, 4, 2, 1024, 128, 128),
                             method=ctypes.pointer(ad())),
    "ad_host_bad_stride": L.stem_prefill_host(ctypes.byref(base(method=ctypes.pointer(ad(stride=3))))),
    "ad_varlen_bad_S": varlen([0, 1000], method=ad()),
    "antidiag_m_null_method": L.stem_antidiag_m(FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128, None,
                                                FAKE, FAKE, 1 << 30, None, None),
    "antidiag_m_bad_stride": L.stem_antidiag_m(FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128,
                                               M(ad(stride=48)), FAKE, FAKE, 1 << 30, None, None),
    "antidiag_m_f32": L.stem_antidiag_m(FAKE, FAKE, 1, 1, 4, 2, 1024, 128, 128, M(AD), FAKE,
                                        FAKE, 1 << 30, None, None),
    "antidiag_m_null_p": L.stem_antidiag_m(FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128, M(AD), None,
                                           FAKE, 1 << 30, None, None),
    "antidiag_m_small_workspace": L.stem_antidiag_m(FAKE, FAKE, 0, 1, 4, 2, 1024, 128, 128,
                                                    M(AD), FAKE, FAKE, 4096, None, None),
    "antidiag_m_q_misaligned": L.stem_antidiag_m(FAKE + 8, FAKE, 0, 1, 4, 2, 1024, 128, 128,
                                                 M(AD), FAKE, FAKE, 1 << 30, None, None),
    "antidiag_m_empty": L.stem_antidiag_m(None, None, 0, 1, 4, 2, 0, 128, 128, M(AD), None,
                                          None, 0, None, None),
    "select_p_null_method": L.stem_select_p_m(FAKE, FAKE, 1, 4, 2, 8, None, FAKE, FAKE, None,
                                              FAKE, 1 << 20, None),
    "select_p_bad_mu": L.stem_select_p_m(FAKE, FAKE, 1, 4, 2, 8, M(BAD_MU), FAKE, FAKE, None,
                                         FAKE, 1 << 20, None),
    "select_p_no_workspace": L.stem_select_p_m(FAKE, FAKE, 1, 4, 2, 8, M(AD), FAKE, FAKE, None,
                                               None, 0, None),
    "select_p_nb_too_large": L.stem_select_p_m(FAKE, FAKE, 1, 4, 2, S.STEM_MAX_NB + 1, M(AD),
                                               FAKE, FAKE, None, FAKE, 1 << 30, None),
    "select_p_null_vnorm": L.stem_select_p_m(FAKE, None, 1, 4, 2, 8, M(AD), FAKE, FAKE, None,
                                             FAKE, 1 << 20, None),
})
print(json.dumps(res))
