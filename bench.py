"""Benchmark of Stem block-sparse causal prefill on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one pass of the whole hot path (block pooling, budget, metric + top-k selection,
block-sparse attention) over one batch of synthetic input, through the library's C ABI
(stem_prefill_ex). Default workload: the Llama-3-8B-shaped layer at S = 131072 (B 1, Hq 32,
Hkv 8, D 128, block 128, rho_min 0.05, tau 64, k_min 8), bf16.

Metric: effective TFLOP/s = 4*block^2*D FLOP per kept (b, q-head, query block, key block) pair
divided by the step time (whole job: summed over ranks); the step latency is ms_per_step.
Timing: CUDA events on the launching stream, W >= 3 warm-up steps, barrier + synchronize on
both sides of exactly K timed steps, max over ranks. Inputs (1.61 GB) are larger than the
126 MB L2, so no flush runs between steps. Per-stage durations come from four events the
library records around its kernels inside the timed steps.

N > 1 (torchrun): one problem split across the ranks by (batch, kv-head group) (partition.py):
every rank builds the same seeded inputs and runs only its contiguous share of the (b, kv head)
units, through the same C-ABI call on views of its heads; no data-path collective (a query
head's pooling, selection and attention read only its own kv head); strong scaling, value =
the whole problem's effective FLOPs over the slowest rank's time. --replicas instead runs an
independent problem per rank (seed + rank), weak scaling.

--impl reference: the CPU oracle (oracle/), as it stands, on this host's cores, on a bounded
sample of the same workload per step (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_causal_pooling_b200 import workloads as wl  # noqa: E402

METRIC = "Stem prefill attention latency (ms) & effective TFLOP/s at S=128K, % of BF16 peak"
# library kernels per call: pooling, head-pair schedule, attention, and two per chunk of heads for
# the selection (scores, then the selection from them); select_chunks() counts the chunks
KERNELS_PER_CALL = 3
SCORE_CAP = 128 << 20  # most bytes of score triangles the workspace holds
# DRAM bytes (read + write) of one attention launch at the 128K workload, from the ncu capture in
# profiles/attn_sm100_dram_llama3-8b-128k.md; reported only while the kernel sources still hash
# to the revision that capture measured.
ATTN_TRAFFIC = {"workload": "llama3-8b-128k", "bytes": 1616291840 + 1018593792,
                "sources_sha256": "c3109ce70917af63022b2abe8b312a05f35b3bc096546960d6d91ef4cf73f62f"}
# The same for the anti-diagonal estimator (stride 16) at that workload: its three kernels (the
# partials, each query group's row statistics, then the merge into p), from the capture in
# profiles/antidiag_sm100_llama3-8b-128k.md.
AD_TRAFFIC = {"workload": "llama3-8b-128k", "stride": 16,
              "bytes": 1411807744 + 673798656 + 9449216 + 688407808 + 45303040,
              "sources_sha256": "2006ed9beacf780952bfedd0ae35d62ed920b342b2ea5cae5737a2825706b83f"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=wl.LLAMA_128K.name, choices=sorted(wl.WORKLOADS))
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--method", choices=["default", "pages", "group", "antidiag"],
                   default="default",
                   help="default: exponential budget, product metric, mean V norms; pages: the "
                        "pages' linear budget (mu 0.7) with the additive metric (beta 0.2, "
                        "clamped) and max-pooled V norms, k_start set for the default's mean "
                        "budget; group: the default with one selection per kv-head group; "
                        "antidiag: the default with block probabilities by anti-diagonal "
                        "sampling (--stride tokens per group)")
    p.add_argument("--stride", type=int, default=16)
    p.add_argument("--replicas", action="store_true",
                   help="N > 1: an independent problem per rank (weak scaling) instead of one "
                        "problem split across the ranks by kv-head group")
    p.add_argument("--no-context", action="store_true",
                   help="skip the context timing of dense causal attention (torch SDPA)")
    return p.parse_args()


def _sources_sha(files):
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "block_sparse_causal_pooling_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def attn_traffic(workload_name):
    if (workload_name == ATTN_TRAFFIC["workload"] and
            _sources_sha(("attn_sm100.cu", "attn_common.cuh", "pairs.cu", "sm100.cuh")) ==
            ATTN_TRAFFIC["sources_sha256"]):
        return ATTN_TRAFFIC["bytes"]
    return None


def antidiag_traffic(workload_name, stride):
    if (workload_name == AD_TRAFFIC["workload"] and stride == AD_TRAFFIC["stride"] and
            _sources_sha(("antidiag_sm100.cu", "sm100.cuh")) == AD_TRAFFIC["sources_sha256"]):
        return AD_TRAFFIC["bytes"]
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime

        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return world, rank, local


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        # nvidia-smi numbers GPUs physically; select ours by UUID
        try:
            self.gpu = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:  # noqa: BLE001
            self.gpu = str(device.index or 0)
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile

        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags)
                          if f.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle (reference arm)


def method_params(w, name, stride=16):
    """Method parameters of a bench run (None: the library's default). "pages": the pages' own
    forms with their ablation optimum (mu 0.7, beta 0.2); k_start gives the linear budget the
    same mean as the workload's default budget, 2 * mean / (1 + mu), to one decimal."""
    if name == "default":
        return None
    if name == "group":
        return dict(schedule="exp", rho_min=w.rho_min, tau=w.tau, k_min=w.k_min, share="group")
    if name == "antidiag":
        return dict(schedule="exp", rho_min=w.rho_min, tau=w.tau, k_min=w.k_min,
                    score="antidiag", stride=stride)
    from block_sparse_causal_pooling_b200 import stem as S

    kk, _ = S.stem_budget(w.nb, w.rho_min, w.tau, w.k_min)
    mu = 0.7
    k_start = round(2.0 * float(kk.double().mean()) / (1.0 + mu), 1)
    return dict(schedule="linear", k_start=k_start, mu=mu, k_min=w.k_min, metric="additive",
                beta=0.2, clamp=True, vsum="max")


def oracle_sample_step(w, q, k, v, rows, mp=None):
    """The oracle as it stands on one kv-head group: pooling, metric, selection for every query
    block of the group's heads, then exact attention for the listed rows. Returns (effective
    FLOP of the listed rows, seconds for attention + selection prorated to those rows).
    mp: method parameters (method_params) or None for the default."""
    import numpy as np

    import oracle

    G = w.Hq // w.Hkv
    qs, ks, vs = q[:, :G].contiguous(), k[:, :1].contiguous(), v[:, :1].contiguous()
    if mp is not None and mp.get("score") == "antidiag":
        # block probabilities of the sampled rows only (the estimator's cost grows with i);
        # the other rows get uniform placeholders, so their selections are valid but unused
        t0 = time.perf_counter()
        kk, off = oracle.budget(w.nb, w.rho_min, w.tau, w.k_min)
        _, _, vn = oracle.pool(qs, ks, vs, w.block)
        pr = oracle.antidiag(qs, ks, w.block, mp["stride"], rows=rows)
        p = np.ones((1, G, w.nb * (w.nb + 1) // 2))
        for (_, h, i), r in zip(rows, pr):
            p[0, h, i * (i + 1) // 2:i * (i + 1) // 2 + i + 1] = r[:i + 1]
        si, sc = oracle.select(oracle.metric_from_p(p, vn), kk, off)
        t1 = time.perf_counter()
        oracle.attention(qs, ks, vs, w.block, si, sc, off, rows)
        t2 = time.perf_counter()
        flop = sum(wl.effective_flops(int(kk[i]), w.block, w.D) for (_, _, i) in rows)
        return flop, t2 - t0, dict(select_s=t1 - t0, attn_s=t2 - t1)
    t0 = time.perf_counter()
    if mp is None or mp.get("schedule") == "exp":
        kk, off = oracle.budget(w.nb, w.rho_min, w.tau, w.k_min)
    else:
        kk, off = oracle.budget_linear(w.nb, mp["k_start"], mp["mu"], mp["k_min"])
    qb, kb, vn = oracle.pool(qs, ks, vs, w.block, "mean" if mp is None else mp.get("vsum", "mean"))
    if mp is not None and mp.get("metric") == "additive":
        m = oracle.metric_additive(qb, kb, vn, mp["beta"], mp["clamp"])
    else:
        m = oracle.metric(qb, kb, vn)
    if mp is not None and mp.get("share") == "group":
        si, sc = oracle.select_group(oracle.metric_group(m, G), kk, off, G)
    else:
        si, sc = oracle.select(m, kk, off)
    t1 = time.perf_counter()
    oracle.attention(qs, ks, vs, w.block, si, sc, off, rows)
    t2 = time.perf_counter()
    flop = sum(wl.effective_flops(int(kk[i]), w.block, w.D) for (_, _, i) in rows)
    share = len(rows) / float(G * w.nb)
    return flop, (t2 - t1) + (t1 - t0) * share, dict(select_s=t1 - t0, attn_s=t2 - t1)


def cpu_inputs(w, seed_offset=0):
    wr = w.replace(seed=w.seed + seed_offset, Hq=w.Hq // w.Hkv, Hkv=1)
    return wl.make_inputs(wr, "cpu")


def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle

    w = wl.WORKLOADS[args.workload]
    mp = method_params(w, args.method, args.stride)
    q, k, v = cpu_inputs(w)
    G = w.Hq // w.Hkv
    import random

    rng = random.Random(7)
    n_rows = max(4, oracle.threads())  # the oracle parallelises over query blocks
    samples = []
    for step in range(args.warmup + args.steps):
        rows = [(0, rng.randrange(G), rng.randrange(w.nb)) for _ in range(n_rows)]
        flop, sec, _ = oracle_sample_step(w, q, k, v, rows, mp)
        if step >= args.warmup:
            samples.append((flop, sec))
    flop = sum(f for f, _ in samples)
    sec = sum(s for _, s in samples)
    value = flop / sec / 1e12
    sample = (f"per step: pooling + metric + selection of one kv-head group ({G} q-heads x "
              f"{w.nb} query blocks, time prorated to the sampled rows) + exact attention of "
              f"{n_rows} random query blocks (seed 7)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sec / len(samples), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, mp),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ multi-rank helpers


def select_chunks(B: int, Hq: int, Hkv: int, nb: int) -> int:
    """Chunks of heads the selection stage runs in: the workspace region it shares with the
    head-pair schedule holds every head's score triangle up to SCORE_CAP bytes, and at least
    the schedule's size (as laid out by the library's stem_workspace_size)."""
    tri = 4 * nb * (nb + 1) // 2
    G = Hq // Hkv
    sched = 256 + 4 * B * Hkv * ((G + 1) // 2) * (nb * (nb + 1) // 2)
    region = -(-max(sched, min(tri * B * Hq, SCORE_CAP)) // 256) * 256
    per = max(1, region // tri)
    return -(-(B * Hq) // per)


def launches_per_call(w, views, mp=None) -> int:
    """Library kernels one stem_prefill_ex call launches, per segment view."""
    n = 0
    for vs in views:
        B, Hq, Hkv = vs[0].shape[0], vs[0].shape[1], vs[1].shape[1]
        if mp is not None and mp.get("score") == "antidiag":
            n += KERNELS_PER_CALL + 4  # estimator, row statistics, merge, selection from p
        elif mp is not None and mp.get("share") == "group" and Hq != Hkv:
            n += KERNELS_PER_CALL + 1  # one fused group-selection kernel
        else:
            n += KERNELS_PER_CALL + 2 * select_chunks(B, Hq, Hkv, w.nb)
    return n


def rank_workload(w, rank: int):
    """--replicas: each rank runs its own independent problem of the same shape (weak
    scaling)."""
    return w.replace(seed=w.seed + rank)


def sum_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's value (timing is the max over ranks)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flop_per_rank: float, world: int, seconds: float) -> float:
    """Throughput of the whole job: every rank's effective FLOPs over the slowest rank's time
    (replicas: every rank does flop_per_rank)."""
    return world * flop_per_rank / seconds / 1e12


# ------------------------------------------------------------------ GPU path


class RawEvents:
    """cudaEvent_t handles through the CUDA runtime torch already loaded. The library records
    them itself (inside stem_prefill_ex), which torch.cuda.Event does not track."""

    def __init__(self):
        import ctypes

        self.ct = ctypes
        self.rt = ctypes.CDLL("libcudart.so.12")
        self.made = []

    def create(self) -> int:
        ev = self.ct.c_void_p()
        rc = self.rt.cudaEventCreate(self.ct.byref(ev))
        if rc != 0:
            raise RuntimeError(f"cudaEventCreate failed ({rc})")
        self.made.append(ev.value)
        return ev.value

    def elapsed_ms(self, a: int, b: int) -> float:
        ms = self.ct.c_float()
        rc = self.rt.cudaEventElapsedTime(self.ct.byref(ms), self.ct.c_void_p(a),
                                          self.ct.c_void_p(b))
        if rc != 0:
            raise RuntimeError(f"cudaEventElapsedTime failed ({rc})")
        return ms.value

    def destroy(self):
        for e in self.made:
            self.rt.cudaEventDestroy(self.ct.c_void_p(e))
        self.made = []


L2_BYTES = 126 * 2 ** 20


def config_of(w, mp=None):
    elt = 2 if w.dtype == "bf16" else 4
    in_bytes = w.B * (w.Hq + 2 * w.Hkv) * w.S * w.D * elt
    l2 = (f"inputs (Q+K+V, {in_bytes / 1e6:.0f} MB) larger than the 126 MB L2; no flush"
          if in_bytes > L2_BYTES else
          f"inputs (Q+K+V, {in_bytes / 1e6:.1f} MB) fit in L2; not flushed (a parity-size "
          f"workload, not a timing one)")
    c = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "D": w.D,
         "block": w.block, "rho_min": w.rho_min, "tau": w.tau, "k_min": w.k_min,
         "input_dtype": w.dtype, "l2": l2}
    if mp is not None:
        c.pop("rho_min")
        c.pop("tau")
        c["method"] = dict(mp)
    return c


def run_ours(args, world, rank, local):
    from block_sparse_causal_pooling_b200 import stem as S

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = wl.WORKLOADS[args.workload]
    mp = method_params(w, args.method, args.stride)
    meth = None if mp is None else S.make_method(**mp)
    from block_sparse_causal_pooling_b200 import partition

    replicas = args.replicas and world > 1
    q, k, v = wl.make_inputs(rank_workload(w, rank) if replicas else w, dev)
    out, sel_idx, sel_cnt = S.alloc_outputs(q, k, w.block, w.rho_min, w.tau, w.k_min, meth)
    ws = S.alloc_workspace(q, k, w.block, meth)  # large enough for any segment of the problem
    if meth is None:
        kk, _ = S.stem_budget(w.nb, w.rho_min, w.tau, w.k_min)
    else:
        kk, _ = S.stem_budget_m(w.nb, meth)
    pairs = w.B * w.Hq * int(kk.sum())
    flop = wl.effective_flops(pairs, w.block, w.D)  # the whole problem
    # this rank's calls: the whole problem (one rank, or replicas), else its segments
    views = ([(q, k, v, out, sel_idx, sel_cnt)] if (world == 1 or replicas) else
             list(partition.rank_views(q, k, v, out, sel_idx, sel_cnt, rank, world)))
    rank_pairs = sum(t[0].shape[0] * t[0].shape[1] for t in views) * int(kk.sum())
    stream = torch.cuda.current_stream(dev)

    K, W = args.steps, args.warmup
    raw = RawEvents()
    ev = [[[raw.create() for _ in range(4)] for _ in views] for _ in range(K)]
    args_warm = [S.make_args(*t[:3], w.block, w.rho_min, w.tau, w.k_min, *t[3:], ws, method=meth)
                 for t in views]
    call_args = [[S.make_args(*t[:3], w.block, w.rho_min, w.tau, w.k_min, *t[3:], ws,
                              events=ev[s][c], method=meth) for c, t in enumerate(views)]
                 for s in range(K)]
    lib = S.lib()
    hstream = S.ctypes.c_void_p(stream.cuda_stream)

    def step(calls):
        for a in calls:
            rc = lib.stem_prefill_ex(S.ctypes.byref(a), hstream)
            if rc != 0:
                raise S.StemError(rc, "stem_prefill_ex")

    for _ in range(W):
        step(args_warm)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clocks:
        torch.cuda.synchronize(dev)
        start.record(stream)
        for s in range(K):
            step(call_args[s])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(stop)
    stage_ms = {"pool": [], "select": [], "attn": []}
    for s in range(K):  # a step's stage time: summed over this rank's calls
        stage_ms["pool"].append(sum(raw.elapsed_ms(e[0], e[1]) for e in ev[s]))
        stage_ms["select"].append(sum(raw.elapsed_ms(e[1], e[2]) for e in ev[s]))
        stage_ms["attn"].append(sum(raw.elapsed_ms(e[2], e[3]) for e in ev[s]))
    raw.destroy()
    ms = max_over_ranks(total_ms / K, world, dev)
    clk = clocks.summary()
    # the pooling kernel alone with a cold L2 (a 256 MB buffer written before each launch), so
    # its bandwidth counts no bytes left in L2 by the previous step's attention
    pool_cold_ms = pool_cold(S, views, w, meth, stream)

    # end to end through the host-buffer entry point: pinned inputs in, output + CSR back (this
    # rank's share of the problem)
    e2e = None
    if args.e2e_steps > 0:
        hviews = [tuple(t.cpu().pin_memory() for t in vs[:3]) +
                  (torch.empty(vs[3].shape, dtype=q.dtype).pin_memory(),
                   torch.empty(vs[4].shape, dtype=torch.int32).pin_memory(),
                   torch.empty(vs[5].shape, dtype=torch.int32).pin_memory()) for vs in views]

        def host_step():
            for hq, hk, hv, hout, hsi, hsc in hviews:
                S.stem_prefill_host(hq, hk, hv, w.block, w.rho_min, w.tau, w.k_min, hout, hsi,
                                    hsc, method=meth)

        host_step()
        if world > 1:
            torch.distributed.barrier()
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            host_step()
        e2e_s = max_over_ranks((time.perf_counter() - t0) / args.e2e_steps, world, dev)
        h2d = sum_over_ranks(sum(t.numel() * t.element_size() for hv_ in hviews
                                 for t in hv_[:3]), world, dev)
        d2h = sum_over_ranks(sum(t.numel() * t.element_size() for hv_ in hviews
                                 for t in hv_[3:]), world, dev)
        e2e = {"value": (whole_job_tflops(flop, world, e2e_s) if replicas else
                         flop / e2e_s / 1e12), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": 1e3 * e2e_s}

    if rank != 0:
        return
    pk, pk_kind = peaks()
    attn_ms = statistics.mean(stage_ms["attn"])
    pool_ms = statistics.mean(stage_ms["pool"])
    sel_ms = statistics.mean(stage_ms["select"])
    long_region = total_ms > 1000.0
    peak_tf = pk["bf16_tflops_sustained"] if long_region else pk["bf16_tflops"]
    # the dominant kernel's rate on this rank: its own share of the kept pairs
    achieved = wl.effective_flops(rank_pairs, w.block, w.D) / (attn_ms * 1e-3) / 1e12
    elt = 2 if w.dtype == "bf16" else 4
    share = rank_pairs / pairs  # this rank's fraction of the (b, head) units
    # the captured traffic is that of one launch over the whole problem: a rank that runs a
    # share of it, or several calls per step, has no captured figure
    whole = share == 1.0 and len(views) == 1
    pool_bytes = share * (w.B * (w.Hq + 2 * w.Hkv) * w.S * w.D * elt +
                          4 * (w.B * (w.Hq + w.Hkv) * w.nb * w.D + w.B * w.Hkv * w.nb))
    line = {
        "metric": METRIC,
        "value": (whole_job_tflops(flop, world, ms * 1e-3) if replicas else
                  flop / (ms * 1e-3) / 1e12), "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak" if (replicas or world == 1) else "strong", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": f"synthetic, seeded ({w.name}: N(0,1) Q/K/V, RoPE theta {w.rope_theta}, K row 0 "
                f"x{w.sink_scale}, {w.n_v_outliers()} V rows per kv-head x{w.v_outlier_scale}, "
                f"heavy-tail fraction {w.heavy_tail_frac})",
        "config": dict(config_of(w, mp), kept_pairs=pairs, effective_tflop=flop / 1e12,
                       parallelism=(f"replicas x{world}" if replicas else
                                    f"kv-head-group partition over {world} rank(s), "
                                    f"{len(views)} call(s) per step on rank 0"),
                       causal_exact_tflop=causal_exact_flops(w, kk) / 1e12,
                       causal_fraction=int(kk.sum()) / (w.nb * (w.nb + 1) / 2)),
        "roofline": {"kernel": "sparse_attn", "bound": "tensor", "achieved": achieved,
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved / peak_tf,
                     "traffic": attn_traffic(w.name) if mp is None and whole else None,
                     "peak_source": f"{pk_kind} {'sustained' if long_region else 'burst'} "
                                    "bf16 dense"},
        "kernels": {
            "pool": {"ms": pool_ms, "bound": "hbm", "bytes": pool_bytes,
                     "GB/s": pool_bytes / (pool_ms * 1e-3) / 1e9,
                     "frac": pool_bytes / (pool_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                     "cold_l2": {"ms": pool_cold_ms,
                                 "GB/s": pool_bytes / (pool_cold_ms * 1e-3) / 1e9,
                                 "frac": pool_bytes / (pool_cold_ms * 1e-3) / 1e9 /
                                 pk["hbm_gbs"],
                                 "how": f"stem_pool alone, {POOL_COLD_REPS} launches, each "
                                        "after writing a 256 MB buffer (L2 is 126 MB)"}},
            "select": select_roofline(w, sel_ms, share, kk, clk, pk),
            "attn": {"ms": attn_ms, "tflops": achieved},
        },
        "clocks": clk,
        "gpu_launches": launches_per_call(w, views, mp) * K,
    }
    if mp is not None and mp.get("score") == "antidiag":
        # the estimator: 2 * stride*D FLOP per causal (query group, key group) pair; its time is
        # the "select" stage, which also holds the selection from p (a lower bound on its rate)
        nred = w.S // mp["stride"]
        ad_flop = share * w.B * w.Hq * 2.0 * mp["stride"] * w.D * nred * (nred + 1) / 2
        ad_tf = ad_flop / (sel_ms * 1e-3) / 1e12
        ad_bytes = share * (2 * w.B * (w.Hq + w.Hkv) * w.S * w.D +
                            4 * w.B * w.Hq * w.nb * (w.nb + 1) // 2)  # Q, K read; p written
        ad_gbs = ad_bytes / (sel_ms * 1e-3) / 1e9
        line["kernels"]["select"] = {
            "ms": sel_ms, "what": "antidiag estimator + selection from p", "bound": "tensor",
            "flop": ad_flop, "tflops": ad_tf, "peak": peak_tf,
            "peak_unit": "TFLOP/s bf16 dense", "frac": ad_tf / peak_tf,
            "bytes": ad_bytes, "GB/s": ad_gbs, "hbm_frac": ad_gbs / pk["hbm_gbs"],
            "traffic": antidiag_traffic(w.name, mp["stride"]) if whole else None,
            "peak_derivation": "the attention roofline's peak"}

    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_context:
        line["context"] = dense_context(q, k, v, ms)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, mp)
        line["cpu_baseline"]["extrapolated_full_workload_s"] = (
            flop / (line["cpu_baseline"]["value"] * 1e12))
    print(json.dumps(line), flush=True)


POOL_COLD_REPS = 5
# fp32 lanes per SM (4 sub-partitions x 32) and FLOP per fused multiply-add
FP32_LANES_PER_SM = 128
SM_COUNT = 148


def pool_cold(S, views, w, meth, stream):
    """Mean duration (ms) of the pooling stage of this rank's calls with L2 flushed first."""
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=stream.device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    bufs = [S.stem_pool(*vs[:3], w.block, stream=stream, method=meth) for vs in views]
    times = []
    for _ in range(POOL_COLD_REPS):
        t = 0.0
        for vs, b in zip(views, bufs):
            flush.fill_(1)
            e0.record(stream)
            S.stem_pool(*vs[:3], w.block, *b, stream=stream, method=meth)
            e1.record(stream)
            torch.cuda.synchronize(stream.device)
            t += e0.elapsed_time(e1)
        times.append(t)
    return statistics.mean(times)


def select_roofline(w, sel_ms, share, kk, clk, pk):
    """Roofline entry of the metric + top-k stage. Its arithmetic is the pooled score, 2*D FLOP
    per causal (query block, key block) pair per query head, on the fp32 lanes (the bound the
    kernel is designed against); the peak is 2 FLOP x 128 lanes x 148 SMs x the median SM clock
    under load. Its bytes are the pooled inputs read and the CSR written."""
    pairs_causal = share * w.B * w.Hq * w.nb * (w.nb + 1) / 2
    flop = 2.0 * w.D * pairs_causal
    cap = int(kk.sum())
    bytes_ = share * (4 * w.B * (w.Hq + w.Hkv) * w.nb * w.D + 4 * w.B * w.Hkv * w.nb +
                      4 * w.B * w.Hq * (cap + w.nb))
    mhz = clk.get("sm_mhz") or 1965.0
    peak = 2.0 * FP32_LANES_PER_SM * SM_COUNT * mhz * 1e6 / 1e12
    tf = flop / (sel_ms * 1e-3) / 1e12
    gbs = bytes_ / (sel_ms * 1e-3) / 1e9
    return {"ms": sel_ms, "bound": "alu", "flop": flop, "tflops": tf,
            "peak": peak, "peak_unit": "TFLOP/s fp32 FMA", "frac": tf / peak,
            "bytes": bytes_, "GB/s": gbs, "hbm_frac": gbs / pk["hbm_gbs"],
            "peak_derivation": f"2 x {FP32_LANES_PER_SM} fp32 lanes x {SM_COUNT} SMs x "
                               f"{mhz:.0f} MHz (median SM clock under load)"}


def causal_exact_flops(w, kk):
    """FLOPs of the kept pairs counting only causal (query, key) token pairs: the diagonal
    block of every row is half a tile plus its diagonal; a partial last block counts its rows."""
    full = wl.effective_flops(1, w.block, w.D)  # one whole tile
    total = 0.0
    for i in range(w.nb):
        n = min(w.block, w.S - i * w.block)
        off_diag = int(kk[i]) - 1
        total += off_diag * full * n / w.block + full * n * (n + 1) / 2 / (w.block * w.block)
    return w.B * w.Hq * total


def dense_context(q, k, v, sparse_ms):
    """Context, not a target: dense causal attention by torch's scaled_dot_product_attention
    (a library kernel) at the same shape, against the step time."""
    try:
        G = q.shape[1] // k.shape[1]
        fn = torch.nn.functional.scaled_dot_product_attention
        run = lambda: fn(q, k, v, is_causal=True, enable_gqa=G > 1)  # noqa: E731
        run()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(3):
            run()
        b.record()
        torch.cuda.synchronize()
        dense_ms = a.elapsed_time(b) / 3
        return {"dense_causal_sdpa_ms": dense_ms, "speedup_vs_dense": dense_ms / sparse_ms,
                "what": "torch scaled_dot_product_attention, is_causal, same Q/K/V (library "
                        "kernel; not a baseline of this metric)"}
    except Exception as e:  # noqa: BLE001
        return {"dense_causal_sdpa_ms": None, "error": str(e)[:200]}


def cpu_baseline(w, mp=None):
    """The oracle, as it stands, on a bounded sample: one kv-head group's selection plus exact
    attention of 64 query blocks per q-head (blocks 0, 1, nb-1 and 61 random, seed 7)."""
    import oracle

    q, k, v = cpu_inputs(w)
    G = w.Hq // w.Hkv
    wg = w.replace(Hq=G, Hkv=1)
    rows = wl.sample_rows(wg, n_random=61, seed=7)
    flop, sec, parts = oracle_sample_step(w, q, k, v, rows, mp)
    if mp is not None and mp.get("score") == "antidiag":
        sample = (f"one kv-head group ({G} q-heads): V pooling, anti-diagonal block "
                  f"probabilities (stride {mp['stride']}) and selection of {len(rows)} query "
                  f"blocks ({parts['select_s']:.2f} s) + their exact fp64 attention "
                  f"({parts['attn_s']:.2f} s)")
    else:
        sample = (f"one kv-head group ({G} q-heads): pooling, metric and selection of all "
                  f"{w.nb} query blocks ({parts['select_s']:.2f} s, prorated to the sampled "
                  f"rows) + exact fp64 attention of {len(rows)} query blocks "
                  f"({parts['attn_s']:.2f} s)")
    return {"value": flop / sec / 1e12, "unit": "TFLOP/s", "cores": oracle.threads(),
            "kind": "oracle", "sample": sample}


def main():
    args = parse()
    world, rank, local = dist_init(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
