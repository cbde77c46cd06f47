"""The (batch, kv-head group) partition on the GPU: every rank's segments, run one after
another on one device through stem_prefill_ex on contiguous views, reassemble the unsharded
call bit for bit (CSR and output). On several GPUs each rank runs only its own segments; here
the ranks take turns, which needs no cross-rank waiting (the segments are independent calls).
"""

import pytest
import torch

from block_sparse_causal_pooling_b200 import partition as P
from block_sparse_causal_pooling_b200 import stem as S
from block_sparse_causal_pooling_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = [
    (wl.LLAMA_32K.replace(name="part-llama", Hq=16, Hkv=4, S=8192), 2),
    (wl.LLAMA_32K.replace(name="part-llama8", Hq=32, Hkv=8, S=4096), 8),
    (wl.LLAMA_32K.replace(name="part-b3", B=3, Hq=4, Hkv=2, S=3000, tau=6.0), 4),
    (wl.QWEN_64K.replace(name="part-qwen", Hq=28, Hkv=4, S=4096, tau=6.0), 3),
]


@pytest.mark.parametrize("w,world", CASES, ids=[f"{w.name}-n{n}" for w, n in CASES])
def test_segments_reassemble_the_whole_call(w, world):
    q, k, v = wl.make_inputs(w, DEV)
    ref_out, ref_si, ref_sc = S.stem_prefill_ex(q, k, v, w.block, w.rho_min, w.tau, w.k_min)
    out, si, sc = S.alloc_outputs(q, k, w.block, w.rho_min, w.tau, w.k_min)
    out.fill_(7.0)
    si.fill_(-1)
    sc.fill_(-1)
    calls = 0
    for rank in range(world):
        for vq, vk, vv, vo, vsi, vsc in P.rank_views(q, k, v, out, si, sc, rank, world):
            status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
            S.stem_prefill_ex(vq, vk, vv, w.block, w.rho_min, w.tau, w.k_min, vo, vsi, vsc,
                              status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            calls += 1
    assert calls >= world
    assert torch.equal(si, ref_si) and torch.equal(sc, ref_sc)
    assert torch.equal(out, ref_out)
