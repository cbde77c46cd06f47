"""stem_select_static, the allocation-free selection entry point, against stem_select.

Callers that cannot allocate device memory (an application whose own allocator owns every
device buffer, a plugin that may not allocate behind it) use stem_select_static: its scratch,
the budget plan, lives in a fixed device array inside the library. This test calls it through
the C ABI twice in a row, on two different problems (so the second call runs on an array that
still holds the first call's plan), and checks each result against the workspace-based
stem_select on the same inputs. It lives in its own file so pytest collects it last.
"""

import pytest
import torch

from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl
from tests import parity

pytestmark = pytest.mark.gpu


def test_static_selection_matches_workspace_selection_twice():
    import oracle

    cases = [
        wl.LLAMA_32K.replace(name="a", Hq=8, Hkv=2, S=96 * 128, rho_min=0.1, tau=16.0, k_min=4),
        wl.QWEN_64K.replace(name="b", Hq=7, Hkv=1, S=40 * 128, rho_min=0.3, tau=5.0, k_min=3),
    ]
    for w in cases:
        q, k, v = wl.make_inputs(w, "cuda:0")
        qbar, kbar, vnorm = S.stem_pool(q, k, v, w.block)
        ref_idx, ref_cnt, _ = S.stem_select(qbar, kbar, vnorm, w.rho_min, w.tau, w.k_min)
        lib = S.lib()
        cap = S.stem_sel_capacity(w.nb, w.rho_min, w.tau, w.k_min)
        sel_idx = torch.full((w.B, w.Hq, cap), -1, dtype=torch.int32, device="cuda:0")
        sel_cnt = torch.full((w.B, w.Hq, w.nb), -1, dtype=torch.int32, device="cuda:0")
        rc = lib.stem_select_static(qbar.data_ptr(), kbar.data_ptr(), vnorm.data_ptr(), w.B,
                                    w.Hq, w.Hkv, w.nb, w.D, w.rho_min, w.tau, w.k_min,
                                    sel_idx.data_ptr(), sel_cnt.data_ptr(),
                                    S._stream(None))
        assert rc == 0, S.strerror(rc)
        torch.cuda.synchronize()
        # the same kernel on the same inputs: identical lists (tighter than the tie tolerance)
        assert torch.equal(sel_idx, ref_idx) and torch.equal(sel_cnt, ref_cnt)
        # and a valid selection by the parity rules against the oracle
        cpu = [t.cpu() for t in (q, k, v)]
        ref = oracle.prefill(*cpu, w.block, w.rho_min, w.tau, w.k_min, rows=[])
        res = parity.compare_selection(sel_idx, sel_cnt, ref["sel_idx"], ref["sel_cnt"],
                                       ref["m"], ref["k"], ref["off"])
        assert not res["violations"], res["violations"][:3]
