"""Seeded synthetic inputs for Stem block-sparse causal prefill.

This module draws Q, K, V tensors and holds the workload table. It contains none
of the method's arithmetic (no pooling, scoring, selection or attention), so the
CUDA path and the CPU oracle can both take their inputs from it without sharing
any computation.

The recipes restate the workloads named for the method ("Stem: Rethinking Causal
Information Flow in Sparse Attention", arXiv 2603.06274): Llama-3-8B-shaped and
Qwen2.5-7B-shaped single attention layers at 32K-128K tokens, with rotary
position embedding on Q and K, a planted attention sink at token 0, a few
high-norm V rows and, for the Qwen shape, heavy-tailed Q/K entries. The pages
evaluate on LongBench and RULER with trained weights; neither is available, so
these tensors stand in for them.

Drawing: a ``torch.Generator`` on the target device, seeded once per workload.
All values are drawn in fp32 and rounded once (round-to-nearest-even) to the
workload dtype, so every consumer reads identical bits.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

BASE_SEED = 20260306


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic prefill problem and its Stem budget parameters."""

    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    D: int
    block: int
    dtype: str  # "bf16" or "f32"
    rho_min: float
    tau: float
    k_min: int
    rope_theta: Optional[float]  # None: no rotary embedding
    sink_scale: float = 8.0  # K row of token 0 multiplied by this
    v_outlier_rows: Optional[int] = None  # absolute count per (b, kv-head)
    v_outlier_frac: float = 0.0  # or a fraction of S per (b, kv-head)
    v_outlier_scale: float = 5.0
    heavy_tail_frac: float = 0.0  # fraction of Q/K entries replaced by Student-t
    heavy_tail_nu: float = 3.0
    seed: int = BASE_SEED

    @property
    def nb(self) -> int:
        return -(-self.S // self.block)  # a partial last block counts

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def n_v_outliers(self) -> int:
        if self.v_outlier_rows is not None:
            return min(self.v_outlier_rows, self.S)
        return int(round(self.v_outlier_frac * self.S))

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _llama(name, S, rho_min, tau, k_min, seed, B=1):
    return Workload(name=name, B=B, Hq=32, Hkv=8, S=S, D=128, block=128, dtype="bf16",
                    rho_min=rho_min, tau=tau, k_min=k_min, rope_theta=5e5,
                    v_outlier_frac=0.005, seed=seed)


# The five workloads. Index i is seeded with BASE_SEED + i.
TINY = Workload(name="tiny", B=1, Hq=2, Hkv=2, S=1024, D=64, block=64, dtype="f32",
                rho_min=0.25, tau=4.0, k_min=2, rope_theta=None, v_outlier_rows=16,
                seed=BASE_SEED + 0)
LLAMA_32K = _llama("llama3-8b-32k", 32768, 0.1, 32.0, 4, BASE_SEED + 1)
LLAMA_128K = _llama("llama3-8b-128k", 131072, 0.05, 64.0, 8, BASE_SEED + 2)
QWEN_64K = Workload(name="qwen2.5-7b-64k", B=1, Hq=28, Hkv=4, S=65536, D=128, block=128,
                    dtype="bf16", rho_min=0.1, tau=48.0, k_min=4, rope_theta=1e6,
                    v_outlier_frac=0.0, heavy_tail_frac=0.02, seed=BASE_SEED + 3)
SWEEP_RHO = (0.05, 0.1, 0.2, 0.5, 1.0)
SWEEP_128K = tuple(_llama(f"llama3-8b-128k-rho{r}", 131072, r, 64.0, 8, BASE_SEED + 4)
                   for r in SWEEP_RHO)
SWEEP_B4_16K = tuple(_llama(f"llama3-8b-b4-16k-rho{r}", 16384, r, 64.0, 8, BASE_SEED + 4, B=4)
                     for r in SWEEP_RHO)

WORKLOADS = {w.name: w for w in (TINY, LLAMA_32K, LLAMA_128K, QWEN_64K) + SWEEP_128K + SWEEP_B4_16K}


def apply_rope(x: torch.Tensor, theta: float, chunk: int = 8192) -> torch.Tensor:
    """Rotate-half rotary embedding at positions 0..S-1, in place, fp32.

    x: [B, H, S, D] fp32. Frequencies theta^(-2m/D) for m in [0, D/2), angle
    position * frequency; pairs (x[m], x[m + D/2]) rotate together.
    """
    B, H, S, D = x.shape
    half = D // 2
    inv = theta ** (-torch.arange(0, half, dtype=torch.float64, device=x.device) * 2.0 / D)
    for s0 in range(0, S, chunk):
        s1 = min(S, s0 + chunk)
        pos = torch.arange(s0, s1, dtype=torch.float64, device=x.device)
        ang = torch.outer(pos, inv)
        cos = torch.cos(ang).to(torch.float32)
        sin = torch.sin(ang).to(torch.float32)
        a = x[:, :, s0:s1, :half]
        b = x[:, :, s0:s1, half:]
        a2 = a * cos - b * sin
        b2 = b * cos + a * sin
        a.copy_(a2)
        b.copy_(b2)
    return x


def _student_t_(x: torch.Tensor, frac: float, nu: float, g: torch.Generator) -> None:
    """Replace a random `frac` of the entries of x by Student-t(nu) draws, in place.

    t = Z / sqrt(chi2_nu / nu) with chi2_nu a sum of nu squared standard normals
    (nu must be an integer here).
    """
    n_nu = int(nu)
    assert n_nu == nu and n_nu >= 1
    mask = torch.rand(x.shape, generator=g, device=x.device) < frac
    cnt = int(mask.sum().item())
    if cnt == 0:
        return
    z = torch.randn(cnt, generator=g, device=x.device)
    chi = torch.randn(cnt, n_nu, generator=g, device=x.device).square().sum(dim=1)
    x[mask] = z / torch.sqrt(chi / nu)


def make_inputs(w: Workload, device: str | torch.device = "cpu"):
    """Draw (q, k, v) for workload `w` on `device`, contiguous [B, H, S, D].

    Recipe, in this order:
      1. Q [B,Hq,S,D], K [B,Hkv,S,D], V [B,Hkv,S,D] ~ N(0, 1) in fp32;
      2. if heavy_tail_frac > 0: that fraction of Q and K entries replaced by
         Student-t(nu) draws;
      3. if rope_theta: rotary embedding on Q and K;
      4. K[:, :, 0, :] *= sink_scale (position 0 is the identity rotation, so the
         order of 3 and 4 is immaterial);
      5. per (b, kv-head): n_v_outliers() distinct V rows, chosen uniformly,
         multiplied by v_outlier_scale;
      6. one round-to-nearest-even conversion to the workload dtype.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    q = torch.randn((w.B, w.Hq, w.S, w.D), generator=g, device=dev, dtype=torch.float32)
    k = torch.randn((w.B, w.Hkv, w.S, w.D), generator=g, device=dev, dtype=torch.float32)
    v = torch.randn((w.B, w.Hkv, w.S, w.D), generator=g, device=dev, dtype=torch.float32)
    if w.heavy_tail_frac > 0:
        _student_t_(q, w.heavy_tail_frac, w.heavy_tail_nu, g)
        _student_t_(k, w.heavy_tail_frac, w.heavy_tail_nu, g)
    if w.rope_theta:
        apply_rope(q, w.rope_theta)
        apply_rope(k, w.rope_theta)
    if w.S > 0:
        k[:, :, 0, :] *= w.sink_scale
    n_out = w.n_v_outliers()
    if n_out > 0:
        for b in range(w.B):
            for h in range(w.Hkv):
                rows = torch.randperm(w.S, generator=g, device=dev)[:n_out]
                v[b, h, rows, :] *= w.v_outlier_scale
    dt = w.torch_dtype
    return q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous()


def effective_flops(sel_count_total: int, block: int, D: int) -> float:
    """Effective attention FLOPs: 4*block^2*D per selected (b, q-head, i, j) pair
    (two block x block x D products, QK^T and PV, diagonal tile counted in full)."""
    return 4.0 * block * block * D * float(sel_count_total)


def causal_pairs(nb: int) -> int:
    return nb * (nb + 1) // 2


def sample_rows(w: Workload, n_random: int = 61, seed: int = 7, heads=None):
    """Deterministic sample of (b, h, i) query blocks for full-size parity checks:
    blocks 0, 1 and nb-1 plus `n_random` distinct random blocks per head."""
    import random

    rng = random.Random(seed)
    nb = w.nb
    heads = range(w.Hq) if heads is None else heads
    rows = []
    for b in range(w.B):
        for h in heads:
            fixed = {0, min(1, nb - 1), nb - 1}
            pool = [i for i in range(nb) if i not in fixed]
            extra = rng.sample(pool, min(n_random, len(pool)))
            for i in sorted(fixed | set(extra)):
                rows.append((b, h, i))
    return rows


__all__ = [
    "Workload", "WORKLOADS", "TINY", "LLAMA_32K", "LLAMA_128K", "QWEN_64K", "SWEEP_128K",
    "SWEEP_B4_16K", "SWEEP_RHO", "make_inputs", "apply_rope", "effective_flops",
    "causal_pairs", "sample_rows", "BASE_SEED",
]
