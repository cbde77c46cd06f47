// Block-sparse causal attention on the Blackwell tensor cores (tcgen05 + TMEM + TMA), bf16 in,
// fp32 accumulation, block = 128.
//
// Computes, for every query token of query block i, exact softmax attention over every token of
// the kept key blocks of row (b, h, i), token-causal inside block i ("Stem: Rethinking Causal
// Information Flow in Sparse Attention", gist.science/es "Resumen tecnico" 2 "Implementacion"
// step 3; gist.science/it 2.C step 3; gist.science/nl "Implementatie" step 3; gist.science/fr
// 2.C step 3).
//
// Work item: two GQA sibling heads A and B at one query block, which keep the same number of key
// blocks; a step schedule (pairs.cu) pairs their lists so a block both keep is one K/V tile.
//
// Persistent kernel, one CTA per SM, 10 warps. Work items are claimed at run time from a global
// counter in heavy-first order (the producer claims, the other roles read the claimed indices
// from a ring in shared memory), so the CTAs finish together.
//   warp 0      TMA producer: claims items; Q_A, Q_B (one tile each) and K/V tiles into a 4-slot
//               ring of 128B-swizzled shared-memory tiles (boxes of 128 rows x 64 columns),
//               filled in the order the products first use them.
//   warp 1      allocates the 512 TMEM columns; lane 0 issues every tcgen05.mma:
//                 S_T = Q_T K^T     (M 128, N 128, K = D; A and B K-major in shared memory)
//                 O_T += P_T V      (A = P read from TMEM over the first half of S_T, B = V
//                                    MN-major in shared memory)
//               in the order P V_A(c), S_A(c+1), P V_B(c), S_B(c+1), so one head's products run
//               while the softmax works on the other head; one commit per S, none per P V.
//   warps 2-9   softmax, two threads per query row (warps w and w+4 share TMEM lanes
//               32*(w%4).. and take 64 columns each; tcgen05.ld 32x32b): row max (halves
//               exchanged through shared memory at a barrier of the warp pair that also makes
//               both warps agree on going on, so an abort cannot strand one), exp2 with the
//               1/sqrt(D) scale folded in; P packed to bf16 and stored over the first half of
//               S_T (tcgen05.st); the per-thread partial row sums add the bf16 values that
//               enter P V, in fp32. Only an item's first step takes the exact row max; later steps
//               use it as the reference and fall back to the exact max, an O rescale in TMEM
//               and a recompute only when a partial row sum reaches 2^16 (exact: the final
//               1/l uses the same reference as P). At an item's end: O * (1/l) -> bf16 ->
//               global (streaming stores).
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,256+D) O_B [384,384+D).
//
// Synchronisation is by mbarriers, plus the warp-pair barrier above. Every mbarrier wait is
// bounded by the global nanosecond timer: on expiry the CTA records STEM_ERR_TIMEOUT in the
// status word, every role leaves its loop, the MMA thread drains its issued products, the
// producer drains its issued copies (both bounded), TMEM is freed and the kernel returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <type_traits>
#include <atomic>
#include <mutex>

#include "sm100.cuh"
#include "stem.h"
#include "stem_internal.h"


namespace stem {

// Test switch (stem_test_withhold_q): when set, the producer of every CTA skips its first Q
// tile, so the MMA thread's bounded wait for it expires and the whole CTA takes the abort path.
std::atomic<int> g_withhold_q{0};

cudaError_t launch_attn_bf16_mma(const void* q, const void* k, const void* v, int B, int Hq,
                                 int Hkv, int S, int D, int block, PlanDev plan, int64_t cap,
                                 const int32_t* sel_idx, void* out, cudaStream_t st);

namespace {

using namespace sm100;

constexpr int kM = 128;             // query rows per tile (= block)
constexpr int kN = 128;             // keys per kept block
constexpr int kSlots = 4;           // K/V ring slots
constexpr int kThreads = 320;       // 10 warps
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kItemRing = 8;                       // claimed work items in flight
constexpr int kItemReaders = 1 + kSoftmaxThreads;  // MMA thread and softmax threads

template <int D>
struct Cfg {
  static constexpr uint32_t kTile = kM * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int kBoxes = D / 64;          // 128B-swizzled boxes of 64 columns
  static constexpr int kKSteps = D / 16;         // MMA k-steps of QK^T
};

struct __align__(8) Bars {
  uint64_t q_full[2], q_empty[2];            // per tile (A, B)
  uint64_t kv_full[kSlots], kv_empty[kSlots];
  uint64_t s_full[2], p_full[2];             // per tile
  uint64_t o_full[2], o_empty[2];            // per tile
  uint64_t iq_full[kItemRing], iq_empty[kItemRing];  // claimed items, producer -> readers
  int64_t iq[kItemRing];                     // item index, or -1: none left
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
  float xch[2][2][kM];  // [parity][half][row] partial row maxima of the two halves
  float xl[2][2][kM];   // [tile][half][row] partial row sums (epilogue)
};

// ---------------------------------------------------------------- PTX helpers

// Bounded wait for the phase of parity `parity` of barrier b. Returns false (after recording
// the timeout) if it expired or another role already aborted.
__device__ __noinline__ bool wait_bar_slow(uint64_t* b, uint32_t parity, Bars* bars,
                                           int32_t* status) {
  const uint64_t t0 = gtimer();
  while (true) {
    if (mbar_try(b, parity)) return true;
    if (bars->abort) return false;
    if (gtimer() - t0 > kWaitNs) {
      bars->abort = 1;
      if (status) atomicExch(status, STEM_ERR_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_bar(uint64_t* b, uint32_t parity, Bars* bars,
                                         int32_t* status) {
  return mbar_try(b, parity) || wait_bar_slow(b, parity, bars, status);
}
// Barrier of the two warps that share TMEM lanes, which also agree on whether to go on: both
// get the AND of their flags, so a warp that gave up (a timed-out wait) takes its partner with
// it instead of leaving it at the barrier. Both warps make the same sequence of these calls.
__device__ __forceinline__ bool pair_and(int id, bool go) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "barrier.cta.red.and.pred b, %2, 64, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(go)), "r"(id)
      : "memory");
  return r != 0;
}
// Two fp32 lanes per instruction (sm_100 f32x2 arithmetic).
struct f2 {
  float x, y;
};
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 r;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Products of one group issued back to back from one asm block. Every descriptor is a base
// word plus an immediate offset, so the issuing thread spends one add per product between
// tcgen05.mma instructions: its instructions between products leave the tensor pipe idle (the
// MMA queue does not hide them), so they are kept to these.
//
// S group: S = Q K^T over the D/16 k-steps, both operands K-major 128B-swizzled tiles in shared
// memory (boxes of 128 rows x 64 columns, 16 KB apart; a k-step is 32 bytes): k-step kk is at
// descriptor offset (kk / 4) * 1024 + (kk % 4) * 2. The first product overwrites D.
// operands: %0 d, %1 a_lo, %2 b_lo, %3 hi, %4 idesc
#define STEM_MMA_SS(OFF)                                                                   \
  "add.u32 x, %1, " #OFF ";\n\tadd.u32 y, %2, " #OFF ";\n\t"                               \
  "mov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"                                        \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, pt;\n\t"
__device__ __forceinline__ void mma_s8(uint32_t d, uint32_t alo, uint32_t blo, uint32_t hi,
                                       uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b32 x, y;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 pf, %4, %4;\n\tsetp.eq.b32 pt, %4, %4;\n\t"
      "mov.b64 a, {%1, %3};\n\tmov.b64 b, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, pf;\n\t"
      STEM_MMA_SS(2) STEM_MMA_SS(4) STEM_MMA_SS(6) STEM_MMA_SS(1024) STEM_MMA_SS(1026)
      STEM_MMA_SS(1028) STEM_MMA_SS(1030) "}" ::"r"(d), "r"(alo), "r"(blo), "r"(hi), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ void mma_s4(uint32_t d, uint32_t alo, uint32_t blo, uint32_t hi,
                                       uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b32 x, y;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 pf, %4, %4;\n\tsetp.eq.b32 pt, %4, %4;\n\t"
      "mov.b64 a, {%1, %3};\n\tmov.b64 b, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, pf;\n\t"
      STEM_MMA_SS(2) STEM_MMA_SS(4) STEM_MMA_SS(6) "}" ::"r"(d), "r"(alo), "r"(blo), "r"(hi),
      "r"(idesc)
      : "memory");
}
#undef STEM_MMA_SS
// P V group: O += P V over the 128 keys, A = P from TMEM (bf16 pairs, 8 columns per k-step of
// 16 keys: keys 16kk.. at column a0 + kPCol[kk]), B = V MN-major in shared memory (16 key rows
// of 128 bytes per k-step: descriptor offset kk * 128). acc0 = 0 starts O afresh.
// operands: %0 d, %1 a0, %2 b_lo, %3 hi, %4 idesc, %5 acc0
#define STEM_MMA_TS(COL, OFF)                                                              \
  "add.u32 x, %1, " #COL ";\n\tadd.u32 y, %2, " #OFF ";\n\tmov.b64 b, {y, %3};\n\t"       \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], [x], b, %4, pt;\n\t"
__device__ __forceinline__ void mma_pv8(uint32_t d, uint32_t a0, uint32_t blo, uint32_t hi,
                                        uint32_t idesc, uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, pt;\n\t.reg .b32 x, y;\n\t.reg .b64 b;\n\t"
      "setp.ne.b32 p0, %5, 0;\n\tsetp.eq.b32 pt, %4, %4;\n\t"
      "mov.b64 b, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b, %4, p0;\n\t"
      STEM_MMA_TS(8, 128) STEM_MMA_TS(16, 256) STEM_MMA_TS(24, 384) STEM_MMA_TS(32, 512)
      STEM_MMA_TS(40, 640) STEM_MMA_TS(48, 768) STEM_MMA_TS(56, 896)
      "}" ::"r"(d), "r"(a0), "r"(blo), "r"(hi), "r"(idesc), "r"(acc0)
      : "memory");
}
#undef STEM_MMA_TS

// Work item t -> (b, g, i, head pair): kv-head-group-major, query blocks in the plan's
// heavy-first order, the ceil(G/2) head pairs of a group adjacent. Tile A is head g*G + 2p,
// tile B head g*G + 2p + 1 (absent when G is odd and this is the group's last pair).
struct Item {
  int b, g, p, i, hA, hB;  // hB < 0: single tile
};
__device__ __forceinline__ Item decode(int64_t t, int G, int nb, int Hkv, const int32_t* order) {
  const int P = (G + 1) >> 1;
  const int64_t per_group = static_cast<int64_t>(P) * nb;
  const int64_t bg = t / per_group;
  const int rem = static_cast<int>(t % per_group);
  Item it;
  it.i = order[rem / P];
  it.b = static_cast<int>(bg / Hkv);
  it.g = static_cast<int>(bg % Hkv);
  it.p = rem % P;
  it.hA = it.g * G + 2 * it.p;
  it.hB = (2 * it.p + 1 < G) ? it.hA + 1 : -1;
  return it;
}

// The k(i) steps of a head pair come from the schedule written by the pairing kernel: entry t
// is blockA | blockB << 16 (blockB 0xFFFF: no head B). Shared blocks first, then lone pairs;
// online softmax does not depend on the order of a row's blocks, and the diagonal is recognised
// by its index. Indices are clamped to [0, i], so no entry can send a load outside the head.
__device__ __forceinline__ const uint32_t* sched_row(const uint32_t* sched, const Item& it,
                                                     int Hkv, int G, int64_t cap,
                                                     const PlanDev& plan) {
  const int P = (G + 1) >> 1;
  const int64_t gp = (static_cast<int64_t>(it.b) * Hkv + it.g) * P + it.p;
  return sched + gp * cap + plan.off[it.i];
}
__device__ __forceinline__ void sched_step(uint32_t e, int i, int& ba, int& bb) {
  ba = min(static_cast<int>(e & 0xFFFFu), i);
  const uint32_t hb = e >> 16;
  bb = hb == 0xFFFFu ? -1 : min(static_cast<int>(hb), i);
}

// Global step sequence of one CTA: its work items (stride gridDim.x) and, inside each, the k(i)
// steps of the head pair's schedule. Producer and MMA thread walk the same sequence with one step of
// lookahead; the softmax warps walk it item by item.
struct Step {
  int n;  // item count of this CTA so far
  bool first, last;
  Item it;
  int ba, bb;  // key blocks of tiles A and B (bb < 0: no tile B)
  __device__ __forceinline__ bool has_b() const { return it.hB >= 0; }
  __device__ __forceinline__ bool shared() const { return bb == ba; }
};
// Work items are claimed at run time, in the heavy-first order of their indices: the producer
// takes the next index from a global counter (set to 0 by the pairing kernel) when it starts
// an item and hands it to the MMA thread and the softmax threads through a ring in shared
// memory (-1: none left). A CTA that finishes its items early takes more, so the CTAs end
// together instead of by a fixed round-robin share.
__device__ __forceinline__ bool claim_item(Bars* bars, unsigned long long* counter,
                                           int64_t items, int64_t n, int32_t* status,
                                           int64_t* t) {
  int64_t v = static_cast<int64_t>(atomicAdd(counter, 1ull));
  if (v >= items) v = -1;
  const int q = static_cast<int>(n % kItemRing);
  if (!wait_bar(&bars->iq_empty[q], static_cast<uint32_t>(((n / kItemRing) & 1) ^ 1), bars,
                status))
    return false;
  bars->iq[q] = v;
  mbar_arrive(&bars->iq_full[q]);
  *t = v;
  return true;
}
// The n-th claimed item of this CTA (every reader calls this once per item, in order).
__device__ __forceinline__ bool read_item(Bars* bars, int64_t n, int32_t* status, int64_t* t) {
  const int q = static_cast<int>(n % kItemRing);
  if (!wait_bar(&bars->iq_full[q], static_cast<uint32_t>((n / kItemRing) & 1), bars, status))
    return false;
  *t = bars->iq[q];
  mbar_arrive(&bars->iq_empty[q]);
  return true;
}

struct Seq {
  int64_t t, items;
  int G, nb, Hkv, Hq;
  int64_t cap;
  PlanDev plan;
  const uint32_t* sched;
  Bars* bars;
  unsigned long long* counter;  // non-null: this walker claims items (the producer)
  int32_t* status;
  bool failed;  // a bounded wait on the item ring expired
  int n, j, cnt;
  Item it;
  const uint32_t* row;
  uint32_t e_next;  // schedule entry of the coming step, loaded one call ahead
  __device__ __forceinline__ void init(int64_t items_, int G_, int nb_, int Hkv_, int Hq_,
                                       int64_t cap_, PlanDev plan_, const uint32_t* sched_,
                                       Bars* bars_, unsigned long long* counter_,
                                       int32_t* status_) {
    items = items_; G = G_; nb = nb_; Hkv = Hkv_; Hq = Hq_; cap = cap_; plan = plan_;
    sched = sched_; bars = bars_; counter = counter_; status = status_;
    failed = false;
    n = -1; j = 0; cnt = 0;
  }
  __device__ __forceinline__ bool next(Step& s) {
    if (j >= cnt) {
      const int64_t ord = n + 1;
      const bool ok = counter ? claim_item(bars, counter, items, ord, status, &t)
                              : read_item(bars, ord, status, &t);
      if (!ok) {
        failed = true;
        return false;
      }
      if (t < 0) return false;
      ++n;
      it = decode(t, G, nb, Hkv, plan.order);
      cnt = plan.k[it.i];
      j = 0;
      row = sched_row(sched, it, Hkv, G, cap, plan);
      e_next = row[0];
    }
    // the entry of this step was loaded by the previous call; the next one is loaded now, so
    // its latency overlaps a step's work instead of stalling the caller
    const uint32_t e = e_next;
    if (j + 1 < cnt) e_next = row[j + 1];
    s.n = n;
    s.first = (j == 0);
    s.last = (j == cnt - 1);
    s.it = it;
    sched_step(e, it.i, s.ba, s.bb);
    ++j;
    return true;
  }
};

// Fill indices of the K/V tiles each step's products take, in the MMA thread's issue order:
// S_A(0), S_B(0), then for every step c with successor x: P V_A(c), S_A(x), P V_B(c), S_B(x).
// A block both heads keep is one tile. The MMA thread (which takes the tiles) and the release
// thread (which frees them) run this same recurrence, so both agree on every slot.
struct TileOrder {
  int32_t next = 0;
  int32_t kA = 0, kB = 0, vA = 0, vB = 0;  // tiles of the latest S_A, S_B, PV_A, PV_B
  // call in issue order: k_a(x0), k_b(x0); then per step c: v_a(), k_a(x), v_b(c), k_b(x)
  __device__ __forceinline__ void k_a() { kA = next++; }
  __device__ __forceinline__ void k_b(bool shared) { kB = shared ? kA : next++; }
  __device__ __forceinline__ void v_a() { vA = next++; }
  __device__ __forceinline__ void v_b(bool shared) { vB = shared ? vA : next++; }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, int Hq, int Hkv, int S, int nb,
                      int64_t items, PlanDev plan, int64_t cap, unsigned long long* counter,
                      const uint32_t* __restrict__ sched, __nv_bfloat16* __restrict__ out,
                      int32_t* status, int withhold_q) {
  using C = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* q_tiles = smem;                   // [tile A, tile B][kTile]
  unsigned char* kv_tiles = smem + 2 * C::kTile;   // [kSlots][kTile]
  Bars* bars = reinterpret_cast<Bars*>(kv_tiles + kSlots * C::kTile);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = Hq / Hkv;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], kSoftmaxThreads);
      mbar_init(&bars->o_full[s], 1);
      mbar_init(&bars->o_empty[s], kSoftmaxThreads);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int s = 0; s < kItemRing; ++s) {
      mbar_init(&bars->iq_full[s], 1);
      mbar_init(&bars->iq_empty[s], kItemReaders);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // TMEM allocation (warp-wide)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(&bars->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)));
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)));
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)));
      const uint64_t pol_kv = policy_evict_last(), pol_q = policy_evict_first();
      // The ring is filled in the order the MMA thread first uses tiles: for step c with
      // lookahead x: V(c, A), K(x, A), V(c, B), K(x, B); a block both heads keep is one tile.
      int64_t f = 0;
      int64_t slot_round[kSlots];
      for (int s = 0; s < kSlots; ++s) slot_round[s] = -1;
      int64_t q_loads[2] = {0, 0};
      bool ok = true;
      auto fill = [&](const CUtensorMap* map, const Step& st, int blk) -> bool {
        const int s = static_cast<int>(f % kSlots);
        const int64_t r = f / kSlots;
        if (!wait_bar(&bars->kv_empty[s], static_cast<uint32_t>((r & 1) ^ 1), bars, status))
          return false;
        mbar_expect_tx(&bars->kv_full[s], C::kTile);
        const int head = st.it.b * Hkv + st.it.g;
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(kv_tiles + s * C::kTile + x * (kN * 128), map, x * 64, blk * kN, head,
                      &bars->kv_full[s], pol_kv);
        slot_round[s] = r;
        ++f;
        return true;
      };
      auto load_q = [&](const Step& st, int tile) -> bool {
        if (withhold_q && tile == 0 && q_loads[0] == 0) return true;  // test switch: never sent
        const int64_t r = q_loads[tile];
        if (!wait_bar(&bars->q_empty[tile], static_cast<uint32_t>((r & 1) ^ 1), bars, status))
          return false;
        mbar_expect_tx(&bars->q_full[tile], C::kTile);
        const int h = tile == 0 ? st.it.hA : st.it.hB;
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(q_tiles + tile * C::kTile + x * (kM * 128), &tm_q, x * 64, st.it.i * kM,
                      st.it.b * Hq + h, &bars->q_full[tile], pol_q);
        ++q_loads[tile];
        return true;
      };
      auto start_step = [&](const Step& st) -> bool {  // Q at item start, then K of tile A
        if (st.first) {
          if (!load_q(st, 0)) return false;
          if (st.has_b() && !load_q(st, 1)) return false;
        }
        return fill(&tm_k, st, st.ba);
      };
      Seq seq;
      seq.init(items, G, nb, Hkv, Hq, cap, plan, sched, bars, counter, status);
      Step x;
      bool have = seq.next(x);
      if (seq.failed) ok = false;
      if (have) {
        ok = start_step(x);
        if (ok && x.has_b() && !x.shared()) ok = fill(&tm_k, x, x.bb);
      }
      while (have && ok) {
        const Step c = x;
        have = seq.next(x);
        if (seq.failed) {
          ok = false;
          break;
        }
        if (!(ok = fill(&tm_v, c, c.ba))) break;
        if (have && !(ok = start_step(x))) break;
        if (c.has_b() && !c.shared() && !(ok = fill(&tm_v, c, c.bb))) break;
        if (have && x.has_b() && !x.shared() && !(ok = fill(&tm_k, x, x.bb))) break;
      }
      if (!ok) {  // abort: let issued copies land before the CTA can exit
        for (int s = 0; s < kSlots; ++s)
          if (slot_round[s] >= 0) drain_bar(&bars->kv_full[s], slot_round[s] & 1);
        for (int tl = 0; tl < 2; ++tl)
          if (q_loads[tl] > 0) drain_bar(&bars->q_full[tl], (q_loads[tl] - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per head step T of step c (lookahead x): the waits for P_T(c) and the V tile of c (and,
    // at an item's first step, the epilogue's release of O_T) are tested together, so their
    // latencies overlap, then P V_T(c) goes out; then the wait for the K tile of x (and, when
    // x starts an item, its Q tile) and S_T(x), with one commit after the S group. Bookkeeping
    // is 32-bit: phase bits and tile numbers (tile f sits in slot f % kSlots, fill round
    // f / kSlots).
    if (lane == 0) {
      constexpr uint32_t idesc_s = instr_desc(kM, kN, false);
      constexpr uint32_t idesc_o = instr_desc(kM, D, true);
      constexpr uint32_t kTileU = C::kTile >> 4;  // a tile's size in descriptor units
      const uint32_t hi = smem_desc_hi(1024);
      const uint32_t q_lo = smem_desc_lo(su32(q_tiles), 16);
      const uint32_t k_lo = smem_desc_lo(su32(kv_tiles), 16);
      const uint32_t v_lo = smem_desc_lo(su32(kv_tiles), kN * 128);
      uint32_t qph = 0;  // bit T: parity of the next q_full[T] wait
      uint32_t pph = 0;  // bit T: parity of the next p_full[T] wait
      uint32_t oph = 0;  // bit T: items finished on tile T, mod 2 (o_empty waits take the other)
      bool ok = true;
      TileOrder order;
      auto kv_try = [&](int32_t f) {
        return mbar_try(&bars->kv_full[f % kSlots], static_cast<uint32_t>(f / kSlots) & 1u);
      };
      auto kv_wait = [&](int32_t f) {
        return wait_bar(&bars->kv_full[f % kSlots], static_cast<uint32_t>(f / kSlots) & 1u, bars,
                        status);
      };
      auto s_group = [&](int tl, int32_t f) {
        const uint32_t a = q_lo + tl * kTileU, b = k_lo + static_cast<uint32_t>(f % kSlots) * kTileU;
        if constexpr (C::kKSteps == 8) {
          mma_s8(tmem + tl * 128, a, b, hi, idesc_s);
        } else {
          static_assert(C::kKSteps == 4, "D 128 or 64");
          mma_s4(tmem + tl * 128, a, b, hi, idesc_s);
        }
        tc_commit(&bars->s_full[tl]);
      };
      auto pv_group = [&](int tl, int32_t f, bool first) {
        static_assert(kN / 16 == 8, "one P V group is 8 products of 16 keys");
        mma_pv8(tmem + 256 + tl * 128, tmem + tl * 128,
                v_lo + static_cast<uint32_t>(f % kSlots) * kTileU, hi, idesc_o, first ? 0u : 1u);
      };
      Seq seq;
      seq.init(items, G, nb, Hkv, Hq, cap, plan, sched, bars, nullptr, status);
      Step x;
      bool have = seq.next(x);
      if (seq.failed) ok = false;
      if (have) {  // S of the first step
        order.k_a();
        ok = wait_bar(&bars->q_full[0], 0, bars, status) && kv_wait(order.kA);
        if (ok) {
          tc_fence_after();
          s_group(0, order.kA);
        }
        qph ^= 1u;
        if (ok && x.has_b()) {
          order.k_b(x.shared());
          ok = wait_bar(&bars->q_full[1], 0, bars, status) && (x.shared() || kv_wait(order.kB));
          if (ok) {
            tc_fence_after();
            s_group(1, order.kB);
          }
          qph ^= 2u;
        }
      }
      while (have && ok) {
        const Step c = x;
        have = seq.next(x);
        if (seq.failed) {
          ok = false;
          break;
        }
        // ---------------- head A: P V_A(c), then S_A(x)
        order.v_a();
        {
          bool r = mbar_try(&bars->p_full[0], pph & 1u) & kv_try(order.vA);
          if (c.first) r &= mbar_try(&bars->o_empty[0], (oph & 1u) ^ 1u);
          if (!r) {
            ok = wait_bar(&bars->p_full[0], pph & 1u, bars, status) && kv_wait(order.vA) &&
                 (!c.first || wait_bar(&bars->o_empty[0], (oph & 1u) ^ 1u, bars, status));
            if (!ok) break;
          }
          pph ^= 1u;
        }
        tc_fence_after();
        pv_group(0, order.vA, c.first);
        if (c.last) {
          tc_commit(&bars->o_full[0]);
          oph ^= 1u;
        }
        if (have) {
          order.k_a();
          const bool qx = x.first;
          bool r = kv_try(order.kA);
          if (qx) r &= mbar_try(&bars->q_full[0], qph & 1u);
          if (!r) {
            ok = kv_wait(order.kA) && (!qx || wait_bar(&bars->q_full[0], qph & 1u, bars, status));
            if (!ok) break;
          }
          if (qx) qph ^= 1u;
          tc_fence_after();
          s_group(0, order.kA);
        }
        // ---------------- head B: P V_B(c) when step c has a head B, then S_B(x) when step x
        // has one (independently: an item without head B can be followed by one with it)
        const bool xb = have && x.has_b();
        if (c.has_b()) {
          order.v_b(c.shared());
          const bool wv = !c.shared();
          bool r = mbar_try(&bars->p_full[1], (pph >> 1) & 1u);
          if (wv) r &= kv_try(order.vB);
          if (c.first) r &= mbar_try(&bars->o_empty[1], ((oph >> 1) & 1u) ^ 1u);
          if (!r) {
            ok = wait_bar(&bars->p_full[1], (pph >> 1) & 1u, bars, status) &&
                 (!wv || kv_wait(order.vB)) &&
                 (!c.first ||
                  wait_bar(&bars->o_empty[1], ((oph >> 1) & 1u) ^ 1u, bars, status));
            if (!ok) break;
          }
          pph ^= 2u;
          tc_fence_after();
          pv_group(1, order.vB, c.first);
          // no S_B follows this P V to cover it: release its V slot from here
          if (!xb) tc_commit(&bars->kv_empty[order.vB % kSlots]);
          if (c.last) {
            tc_commit(&bars->o_full[1]);
            oph ^= 2u;
          }
        }
        if (xb) {
          order.k_b(x.shared());
          const bool qx = x.first, wk = !x.shared();
          bool r = true;
          if (wk) r &= kv_try(order.kB);
          if (qx) r &= mbar_try(&bars->q_full[1], (qph >> 1) & 1u);
          if (!r) {
            ok = (!wk || kv_wait(order.kB)) &&
                 (!qx || wait_bar(&bars->q_full[1], (qph >> 1) & 1u, bars, status));
            if (!ok) break;
          }
          if (qx) qph ^= 2u;
          tc_fence_after();
          s_group(1, order.kB);
        }
      }
      // make sure every issued product has completed before TMEM is released
      tc_commit(&bars->drain);
      drain_bar(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    constexpr int kH = kN / 2;          // key columns per thread
    constexpr int kDH = D / 2;          // output columns per thread
    const int sub = warp & 3;           // TMEM sub-partition of this warp
    const int half = (warp - 2) >> 2;   // 0: columns [0, 64), 1: [64, 128)
    const int row = sub * 32 + lane;    // query row within the tile
    const int bar_id = 1 + sub;         // named barrier of the warp pair (sub, sub + 4)
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const float sl2 = 1.4426950408889634f * rsqrtf(static_cast<float>(D));
    // per-tile state lives in scalars (passed by reference) so it stays in registers
    int64_t steps_a = 0, steps_b = 0, outs_a = 0, outs_b = 0;
    int xp = 0;  // exchange-slot parity
    float m_a = 0.f, m_b = 0.f, l_a = 0.f, l_b = 0.f;
    bool ok = true;
    // The release thread frees ring slots and Q tiles: when S_T of a step is complete, so is
    // every product issued before it (K of this step unless head B still needs it, V of the
    // previous step, Q after the item's last S).
    const bool releaser = (warp == 2 && lane == 0);
    auto release = [&](int64_t tile) {
      if (tile >= 0) mbar_arrive(&bars->kv_empty[tile % kSlots]);
    };
    // one step of tile tl on key block blk; returns false on abort
    // Row max of this thread's half of S (log2 units, scale folded in) agreed with the partner
    // half through shared memory; both warps of the pair call it at the same point.
    auto pair_max = [&](const uint32_t* sr, bool& ok) -> float {
      float mx[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) mx[e] = __uint_as_float(sr[e]);
#pragma unroll
      for (int c = 4; c < kH; c += 2)
        mx[(c >> 1) & 3] =
            max3(mx[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
      float mt = max3(mx[0], mx[1], fmaxf(mx[2], mx[3]));
      bars->xch[xp][half][row] = mt;
      ok = pair_and(bar_id, true);
      mt = fmaxf(mt, bars->xch[xp][half ^ 1][row]) * sl2;  // both halves alike
      xp ^= 1;
      return mt;
    };
    // P = exp2(S * sl2 - m_run) packed to bf16 over column pairs [C0, C1) of this thread's
    // half; adds to the partial row sums the bf16 values that enter P V (mixed-precision adds
    // take each half of a packed pair as it is), so the normaliser and the products see the
    // same P and a row that one key dominates returns that key's V row.
    auto exp_pack = [&](const uint32_t* sr, float m_run, uint32_t* p, f2* sum, auto c0,
                        auto c1) {
      const f2 scl{sl2, sl2}, neg{-m_run, -m_run};
#pragma unroll
      for (int c = decltype(c0)::value; c < decltype(c1)::value; ++c) {
        const f2 x = fma2(f2{__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])}, scl, neg);
        const f2 e{ex2(x.x), ex2(x.y)};
        p[c] = pack_bf16(e.x, e.y);
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
            : "+f"(sum[c & 1].x), "+f"(sum[c & 1].y)
            : "r"(p[c]));
      }
    };
    auto exp_all = [&](const uint32_t* sr, float m_run, uint32_t* p) -> float {
      f2 sum[2] = {f2{0.f, 0.f}, f2{0.f, 0.f}};
      exp_pack(sr, m_run, p, sum, std::integral_constant<int, 0>{},
               std::integral_constant<int, kH / 2>{});
      return (sum[0].x + sum[0].y) + (sum[1].x + sum[1].y);
    };
    auto diag_mask = [&](uint32_t* sr, auto c0, auto c1) {
#pragma unroll
      for (int c = decltype(c0)::value; c < decltype(c1)::value; ++c)
        if (half * kH + c > row) sr[c] = __float_as_uint(-INFINITY);
    };
    // One step of tile tl on key block blk; returns false on abort.
    //
    // The exponentials use the row's running reference max m_run. The first step of an item
    // sets it to the exact row max; later steps form P against it without looking for their
    // own max, and only if some row's partial sum reaches 2^16 (a score that grew by ~10 in
    // log2 units, or an overflow) does the pair take the exact max, rescale O and recompute.
    // The result is exact either way: the final 1/l uses the same reference as P.
    //
    // Barriers of the warp pair per step, the same sequence on both warps: [first step: max
    // exchange] check; if the check fails: agree on going on, then the max exchange. A warp
    // that gives up joins every barrier its partner will meet with "stop".
    auto step = [&](int tl, int blk, int qi, bool first, int64_t& nsteps, float& m_run,
                    float& lsum, int64_t rel_k, int64_t rel_v, bool rel_q) -> bool {
      const int64_t r = nsteps++;
      bool w = wait_bar(&bars->s_full[tl], static_cast<uint32_t>(r & 1), bars, status);
      if (!__all_sync(0xffffffffu, w)) {
        pair_and(bar_id, false);  // [first: the max exchange | the check]
        if (!first) pair_and(bar_id, false);  // the agreement after a failed check
        return false;
      }
      if (releaser) {
        release(rel_k);
        release(rel_v);
        if (rel_q) mbar_arrive(&bars->q_empty[tl]);
      }
      tc_fence_after();
      const uint32_t s_addr = tmem + tl * 128 + lane_off;
      uint32_t sr[kH];
      uint32_t p[kH / 2];
      bool ok = true;
#pragma unroll
      for (int c = 0; c < kH / 32; ++c) TC_LD32(s_addr + half * kH + 32 * c, (sr + 32 * c));
      tc_wait_ld_r32(sr);
      tc_wait_ld_r32(sr + 32);
      if (blk == qi) {  // the diagonal block: token-causal
        diag_mask(sr, std::integral_constant<int, 0>{}, std::integral_constant<int, kH>{});
      }
      if (first) {
        m_run = pair_max(sr, ok);
        if (!ok) return false;
        lsum = 0.f;
      }
      float part = exp_all(sr, m_run, p);
      const bool small = part < 65536.0f;  // false for inf and NaN too
      if (!pair_and(bar_id, __all_sync(0xffffffffu, small))) {
        if (!pair_and(bar_id, true)) return false;
        // a row's scores grew past the reference (never on a first step, whose reference is
        // the exact max): the warp rescales its part of O_T (each row by its own factor, 1
        // where the max did not grow) and recomputes P. The previous P V of this tile is
        // complete: this S was issued after it and s_full tracks every earlier product.
        const float mt = pair_max(sr, ok);
        if (!ok) return false;
        const float m_new = fmaxf(m_run, mt);
        const float alpha = ex2(m_run - m_new);
        m_run = m_new;
        lsum *= alpha;
        const uint32_t o_addr = tmem + 256 + tl * 128 + half * kDH + lane_off;
#pragma unroll 1
        for (int c = 0; c < kDH / 32; ++c) {
          uint32_t o[32];
          TC_LD32(o_addr + 32 * c, o);
          tc_wait_ld_r32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          TC_ST32(o_addr + 32 * c, o);
        }
        tc_wait_st();
        part = exp_all(sr, m_run, p);
      }
      // P over S_T columns [0, 64): this half's keys go to columns half*32 .. +32 (both halves
      // finished reading S before the pair's check barrier above)
      TC_ST32(s_addr + half * (kH / 2), p);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[tl]);
      lsum += part;
      return true;
    };
    auto epilogue = [&](int tl, const Item& it, int64_t& nouts, float lsum) -> bool {
      const int64_t r = nouts++;
      bool w = wait_bar(&bars->o_full[tl], static_cast<uint32_t>(r & 1), bars, status);
      w = __all_sync(0xffffffffu, w);
      bars->xl[tl][half][row] = lsum;
      if (!pair_and(bar_id, w)) return false;
      const float inv = 1.0f / (lsum + bars->xl[tl][half ^ 1][row]);
      tc_fence_after();
      const int h = tl == 0 ? it.hA : it.hB;
      __nv_bfloat16* dst = out + ((static_cast<int64_t>(it.b) * Hq + h) * S +
                                  static_cast<int64_t>(it.i) * kM + row) * D + half * kDH;
      const bool valid = static_cast<int64_t>(it.i) * kM + row < S;  // partial last block
      const uint32_t o_addr = tmem + 256 + tl * 128 + half * kDH + lane_off;
#pragma unroll
      for (int c = 0; c < kDH / 32; ++c) {
        uint32_t o[32];
        TC_LD32(o_addr + 32 * c, o);
        tc_wait_ld_r32(o);
        uint4 pk[4];
        uint32_t* wv = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          wv[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
        if (valid) {
#pragma unroll
          for (int e = 0; e < 4; ++e) __stcs(d4 + e, pk[e]);  // evict-first: keep K/V in L2
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->o_empty[tl]);
      return true;
    };
    TileOrder order;  // replica of the MMA thread's tile numbering
    bool have_prev = false, prev_has_b = false, prev_shared = false;
    for (int64_t n = 0; ok; ++n) {
      int64_t t = -1;
      const bool got = read_item(bars, n, status, &t);
      // both warps of a pair go on together (a failed read takes the partner out too)
      if (!pair_and(bar_id, __all_sync(0xffffffffu, got))) {
        ok = false;
        break;
      }
      if (t < 0) break;
      const Item it = decode(t, G, nb, Hkv, plan.order);
      const int cnt = plan.k[it.i];
      const uint32_t* srow = sched_row(sched, it, Hkv, G, cap, plan);
      uint32_t e_next = srow[0];  // loaded one step ahead, as in Seq
      for (int j = 0; j < cnt && ok; ++j) {
        const uint32_t e = e_next;
        if (j + 1 < cnt) e_next = srow[j + 1];
        Step x;
        x.it = it;
        sched_step(e, it.i, x.ba, x.bb);
        const bool has_b = x.has_b(), shared = x.shared();
        if (have_prev) order.v_a();
        order.k_a();
        if (have_prev && prev_has_b) order.v_b(prev_shared);
        if (has_b) order.k_b(shared);
        const int64_t rka = (has_b && shared) ? -1 : order.kA;
        const int64_t rva = (have_prev && !(prev_has_b && prev_shared)) ? order.vA : -1;
        ok = step(0, x.ba, it.i, j == 0, steps_a, m_a, l_a, rka, rva, j == cnt - 1);
        if (ok && has_b) {
          const int64_t rvb = (have_prev && prev_has_b) ? order.vB : -1;
          ok = step(1, x.bb, it.i, j == 0, steps_b, m_b, l_b, order.kB, rvb, j == cnt - 1);
        }
        have_prev = true;
        prev_has_b = has_b;
        prev_shared = shared;
      }
      if (!ok) break;
      ok = epilogue(0, it, outs_a, l_a);
      if (ok && it.hB >= 0) ok = epilogue(1, it, outs_b, l_b);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// ---------------------------------------------------------------- host side

// 3-D view [heads, S, D] of a bf16 tensor, boxes of 64 columns x 128 tokens x 1 head, 128B
// swizzle. Token rows past S are outside the view: a box over a partial last block reads them
// as 0 instead of the next head's first rows.
bool make_map(CUtensorMap* m, const void* base, uint64_t heads, int S, int D) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), heads};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S) * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_sm100(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                         int S, PlanDev plan, int64_t cap, const int32_t* sel_idx,
                         uint32_t* sched, void* out, int32_t* status, cudaStream_t st) {
  const int nb = (S + kM - 1) / kM;
  const int G = Hq / Hkv;
  const int64_t items = static_cast<int64_t>(B) * Hkv * nb * ((G + 1) / 2);  // head pairs
  if (items == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, static_cast<uint64_t>(B) * Hq, S, D) ||
      !make_map(&tk, k, static_cast<uint64_t>(B) * Hkv, S, D) ||
      !make_map(&tv, v, static_cast<uint64_t>(B) * Hkv, S, D))
    return cudaErrorInvalidValue;
  // one CTA per SM: each CTA takes all 512 TMEM columns
  const size_t smem = std::max<size_t>(1024 + (2 + kSlots) * Cfg<D>::kTile + sizeof(Bars),
                                       120 * 1024);
  auto kern = attn_sm100_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // the pairing kernel sets the work counter (the region's first bytes) to 0 and writes the
  // schedule after it
  e = launch_pairs(sel_idx, B, Hq, Hkv, nb, plan, cap, sched, st);
  if (e != cudaSuccess) return e;
  auto* counter = reinterpret_cast<unsigned long long*>(sched);
  const int64_t grid = std::min<int64_t>(items, sm_count());
  kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(
      tq, tk, tv, Hq, Hkv, S, nb, items, plan, cap, counter, pairs_schedule(sched),
      static_cast<__nv_bfloat16*>(out), status, g_withhold_q.load());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bf16(const void* q, const void* k, const void* v, int B, int Hq,
                             int Hkv, int S, int D, int block, PlanDev plan, int64_t cap,
                             const int32_t* sel_idx, const int32_t*, uint32_t* sched, void* out,
                             int32_t* status, cudaStream_t st) {
  if (block == 128 && D == 128)
    return launch_sm100<128>(q, k, v, B, Hq, Hkv, S, plan, cap, sel_idx, sched, out, status, st);
  if (block == 128 && D == 64)
    return launch_sm100<64>(q, k, v, B, Hq, Hkv, S, plan, cap, sel_idx, sched, out, status, st);
  return launch_attn_bf16_mma(q, k, v, B, Hq, Hkv, S, D, block, plan, cap, sel_idx, out, st);
}

}  // namespace stem

extern "C" int stem_test_withhold_q(int on) { return stem::g_withhold_q.exchange(on ? 1 : 0); }
