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
// Persistent kernel, one CTA per SM, 12 warps. Work items are claimed at run time from a global
// counter in heavy-first order (the producer claims, the other roles read the claimed indices
// from a ring in shared memory), so the CTAs finish together.
//   warp 0      TMA producer: claims items; Q_A, Q_B (one tile each) and K/V tiles into a ring
//               of 128B-swizzled shared-memory tiles (boxes of 128 rows x 64 columns), filled
//               in the order the products use them.
//   warp 1      allocates the 512 TMEM columns; lane 0 issues every tcgen05.mma:
//                 S_T = Q_T K^T     (M 128, N 128, K = D; A and B K-major in shared memory)
//                 O_T += P_T V      (A = P K-major in shared memory, B = V MN-major)
//               S_T of the next step goes out as soon as the softmax has read S_T of this step
//               into registers, so it runs while the softmax works: a head is no serial chain
//               of softmax, P V and the next S.
//   warps 2-3   idle (they complete the first warpgroup, which hands its registers over).
//   warps 4-7   softmax of head A, warps 8-11 of head B: one thread per query row (warp w reads
//               TMEM lanes 32*(w%4)..), all 128 key columns (tcgen05.ld 32x32b): row max,
//               exp2 with the 1/sqrt(D) scale folded in, P packed to bf16 and written to the
//               head's P tile in shared memory (the layout a TMA box of Q has), row sums over
//               the bf16 values that enter P V, in fp32. The running reference max moves only
//               when a row's max exceeds it by more than 8 (log2 units): then O's row is
//               rescaled in TMEM; otherwise P stays below 2^8 and the reference is kept (exact
//               either way: the final 1/l uses the same reference as P). At an item's end:
//               O * (1/l) -> bf16, staged in the head's P tile (free until the next item's
//               first P) and copied out by each warp with coalesced streaming stores.
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,256+D) O_B [384,384+D).
//
// Synchronisation is by mbarriers only. Every mbarrier wait is bounded by the global
// nanosecond timer: on expiry the CTA records STEM_ERR_TIMEOUT in the status word, every role
// leaves its loop, the MMA thread drains its issued products, the producer drains its issued
// copies (both bounded), TMEM is freed and the kernel returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "attn_common.cuh"
#include "sm100.cuh"
#include "stem.h"
#include "stem_internal.h"


namespace stem {

// Test switch (stem_test_withhold_q): when set, the producer of every CTA skips its first Q
// tile, so the MMA thread's bounded wait for it expires and the whole CTA takes the abort path.
std::atomic<int> g_withhold_q{0};

cudaError_t launch_attn_bf16_b64(const void* q, const void* k, const void* v, int B, int Hq,
                                 int Hkv, int S, int D, PlanDev plan, int64_t cap,
                                 const int32_t* sel_idx, uint32_t* sched, void* out,
                                 int32_t* status, cudaStream_t st);

namespace {

using namespace sm100;

constexpr int kM = 128;             // query rows per tile (= block)
template <int D>
struct Cfg {
  static constexpr uint32_t kTile = kM * D * 2;   // bytes of a 128 x D bf16 tile
  static constexpr uint32_t kPTile = kM * kN * 2; // bytes of a 128 x 128 bf16 P tile
  static constexpr int kBoxes = D / 64;           // 128B-swizzled boxes of 64 columns
  static constexpr int kKSteps = D / 16;          // MMA k-steps of QK^T
  static constexpr int kSlots = D == 128 ? 3 : 4; // what fits beside Q and P
  static constexpr size_t kSmem =
      1024 + 2 * kTile + 2 * kPTile + kSlots * static_cast<size_t>(kTile) + sizeof(Bars);
};
static_assert(Cfg<128>::kSmem <= 232448, "shared memory of the D = 128 kernel");
static_assert(Cfg<64>::kSmem <= 232448, "shared memory of the D = 64 kernel");

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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, int Hq, int Hkv, int S, int nb,
                      int64_t items, PlanDev plan, int64_t cap, unsigned long long* counter,
                      const uint32_t* __restrict__ sched, __nv_bfloat16* __restrict__ out,
                      int32_t* status, int withhold_q) {
  using C = Cfg<D>;
  constexpr int kSlots = C::kSlots;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* q_tiles = smem;                        // [tile A, tile B][kTile]
  unsigned char* p_tiles = smem + 2 * C::kTile;         // [tile A, tile B][kPTile]
  unsigned char* kv_tiles = p_tiles + 2 * C::kPTile;    // [kSlots][kTile]
  Bars* bars = reinterpret_cast<Bars*>(kv_tiles + kSlots * C::kTile);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = Hq / Hkv;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], kGroupThreads);
      mbar_init(&bars->p_full[s], kGroupThreads);
      mbar_init(&bars->pv_done[s], 1);
      mbar_init(&bars->o_empty[s], kGroupThreads);
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

  // Registers: the launch gives every thread 168 (12 warps; a scheduler holds three). The
  // producer / MMA warpgroup needs few and gives them to the two softmax warpgroups, whose
  // threads each hold a row of 128 scores and its 64 packed P words: 4 x 32 x 72 +
  // 8 x 32 x 216 = 384 x 168.
  if (warp < 4) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 72;" ::: "memory");
   if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)));
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)));
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)));
      const uint64_t pol_kv = policy_evict_last(), pol_q = policy_evict_first();
      // The ring is filled in the order the MMA thread uses tiles: per step c with successor
      // x, K(x, A), K(x, B), V(c, A), V(c, B) inside an item, V before K when x starts the
      // next item; a block both heads keep is one tile.
      int64_t f = 0;
      int64_t slot_round[kMaxSlots];
      for (int s = 0; s < kMaxSlots; ++s) slot_round[s] = -1;
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
      auto fill_k = [&](const Step& st) -> bool {  // Q at an item's start, then the K tiles
        if (st.first) {
          if (!load_q(st, 0)) return false;
          if (st.has_b() && !load_q(st, 1)) return false;
        }
        if (!fill(&tm_k, st, st.ba)) return false;
        return !(st.has_b() && !st.shared()) || fill(&tm_k, st, st.bb);
      };
      auto fill_v = [&](const Step& st) -> bool {
        if (!fill(&tm_v, st, st.ba)) return false;
        return !(st.has_b() && !st.shared()) || fill(&tm_v, st, st.bb);
      };
      Seq seq;
      seq.init(items, G, nb, Hkv, Hq, cap, plan, sched, bars, counter, status);
      Step x;
      bool have = seq.next(x);
      if (seq.failed) ok = false;
      if (have) ok = fill_k(x);
      while (have && ok) {
        const Step c = x;
        have = seq.next(x);
        if (seq.failed) {
          ok = false;
          break;
        }
        if (have && !x.first)
          ok = fill_k(x) && fill_v(c);
        else
          ok = fill_v(c) && (!have || fill_k(x));
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
    // Inside an item, per step c with successor x: S_A(x), S_B(x), P V_A(c), P V_B(c). S_T(x)
    // waits for its K tile, its Q tile when x starts an item and the softmax's read of the
    // previous S_T (s_free); P V_T(c) for P_T(c), its V tile and, at an item's first step,
    // the epilogue's read of O_T. When x starts the next item, P V of c goes first. A tile
    // is released by a commit after the last product that reads it.
    if (lane == 0) {
      constexpr uint32_t idesc_s = instr_desc(kM, kN, false);
      constexpr uint32_t idesc_o = instr_desc(kM, D, true);
      constexpr uint32_t kTileU = C::kTile >> 4;    // a tile's size in descriptor units
      constexpr uint32_t kPTileU = C::kPTile >> 4;
      const uint32_t hi = smem_desc_hi(1024);
      const uint32_t q_lo = smem_desc_lo(su32(q_tiles), 16);
      const uint32_t p_lo = smem_desc_lo(su32(p_tiles), 16);
      const uint32_t k_lo = smem_desc_lo(su32(kv_tiles), 16);
      const uint32_t v_lo = smem_desc_lo(su32(kv_tiles), kN * 128);
      int32_t f = 0;               // K/V tiles taken, in fill order
      int32_t nq[2] = {0, 0};      // Q tiles taken per tile (q_full phases)
      int32_t ns[2] = {0, 0};      // S products issued per tile
      int32_t np[2] = {0, 0};      // P V groups issued per tile (p_full phases)
      int32_t no[2] = {0, 0};      // items started per tile (o_empty phases)
      bool ok = true;
      auto kv_try = [&](int32_t t) {
        return mbar_try(&bars->kv_full[t % kSlots], static_cast<uint32_t>(t / kSlots) & 1u);
      };
      auto kv_wait = [&](int32_t t) {
        return wait_bar(&bars->kv_full[t % kSlots], static_cast<uint32_t>(t / kSlots) & 1u, bars,
                        status);
      };
      auto issue_s = [&](const Step& s, int tl, int32_t kt, bool wait_k, bool release_k) -> bool {
        const uint32_t qp = static_cast<uint32_t>(nq[tl]) & 1u;
        const uint32_t sp = static_cast<uint32_t>(ns[tl] - 1) & 1u;
        bool r = !wait_k || kv_try(kt);
        if (s.first) r &= mbar_try(&bars->q_full[tl], qp);
        if (ns[tl] > 0) r &= mbar_try(&bars->s_free[tl], sp);
        if (!r && !((!wait_k || kv_wait(kt)) &&
                    (!s.first || wait_bar(&bars->q_full[tl], qp, bars, status)) &&
                    (ns[tl] == 0 || wait_bar(&bars->s_free[tl], sp, bars, status))))
          return false;
        if (s.first) ++nq[tl];
        ++ns[tl];
        tc_fence_after();
        const uint32_t a = q_lo + tl * kTileU;
        const uint32_t b = k_lo + static_cast<uint32_t>(kt % kSlots) * kTileU;
        if constexpr (C::kKSteps == 8) {
          mma_s8(tmem + tl * 128, a, b, hi, idesc_s);
        } else {
          static_assert(C::kKSteps == 4, "D 128 or 64");
          mma_s4(tmem + tl * 128, a, b, hi, idesc_s);
        }
        tc_commit(&bars->s_full[tl]);
        if (s.last) tc_commit(&bars->q_empty[tl]);
        if (release_k) tc_commit(&bars->kv_empty[kt % kSlots]);
        return true;
      };
      auto issue_pv = [&](const Step& c, int tl, int32_t vt, bool wait_v,
                          bool release_v) -> bool {
        const uint32_t pp = static_cast<uint32_t>(np[tl]) & 1u;
        const uint32_t op = static_cast<uint32_t>(no[tl] - 1) & 1u;
        const bool wo = c.first && no[tl] > 0;
        bool r = mbar_try(&bars->p_full[tl], pp);
        if (wait_v) r &= kv_try(vt);
        if (wo) r &= mbar_try(&bars->o_empty[tl], op);
        if (!r && !(wait_bar(&bars->p_full[tl], pp, bars, status) &&
                    (!wait_v || kv_wait(vt)) &&
                    (!wo || wait_bar(&bars->o_empty[tl], op, bars, status))))
          return false;
        if (c.first) ++no[tl];
        ++np[tl];
        tc_fence_after();
        static_assert(kN / 16 == 8, "one P V group is 8 products of 16 keys");
        mma_pv8(tmem + 256 + tl * 128, p_lo + tl * kPTileU,
                v_lo + static_cast<uint32_t>(vt % kSlots) * kTileU, hi, idesc_o,
                c.first ? 0u : 1u);
        tc_commit(&bars->pv_done[tl]);
        if (release_v) tc_commit(&bars->kv_empty[vt % kSlots]);
        return true;
      };
      auto s_step = [&](const Step& s) -> bool {
        const bool sh = s.has_b() && s.shared();
        const int32_t ka = f++;
        if (!issue_s(s, 0, ka, true, !sh)) return false;
        if (!s.has_b()) return true;
        const int32_t kb = sh ? ka : f++;
        return issue_s(s, 1, kb, !sh, true);
      };
      auto pv_step = [&](const Step& c) -> bool {
        const bool sh = c.has_b() && c.shared();
        const int32_t va = f++;
        if (!issue_pv(c, 0, va, true, !sh)) return false;
        if (!c.has_b()) return true;
        const int32_t vb = sh ? va : f++;
        return issue_pv(c, 1, vb, !sh, true);
      };
      Seq seq;
      seq.init(items, G, nb, Hkv, Hq, cap, plan, sched, bars, nullptr, status);
      Step x;
      bool have = seq.next(x);
      if (seq.failed) ok = false;
      if (have) ok = s_step(x);
      while (have && ok) {
        const Step c = x;
        have = seq.next(x);
        if (seq.failed) {
          ok = false;
          break;
        }
        if (have && !x.first)
          ok = s_step(x) && pv_step(c);
        else
          ok = pv_step(c) && (!have || s_step(x));
      }
      // make sure every issued product has completed before TMEM is released
      tc_commit(&bars->drain);
      drain_bar(&bars->drain, 0);
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;" ::: "memory");
    // ------------------------------------------------------------ softmax + epilogue
    const int tl = (warp - 4) >> 2;     // 0: head A (warps 4-7), 1: head B (warps 8-11)
    const int sub = warp & 3;           // TMEM sub-partition of this warp
    const int row = sub * 32 + lane;    // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t s_addr = tmem + tl * 128 + lane_off;
    const uint32_t o_addr = tmem + 256 + tl * 128 + lane_off;
    const uint32_t p_row = su32(p_tiles + tl * C::kPTile) + static_cast<uint32_t>(row) * 128;
    const uint32_t swz = static_cast<uint32_t>(row & 7);
    const float sl2 = 1.4426950408889634f * rsqrtf(static_cast<float>(D));
    int32_t ns = 0;       // S_T tiles read
    int32_t np = 0;       // P_T tiles written (each followed by one P V_T group)
    int32_t pv_seen = 0;  // P V_T groups known complete
    float m_run = 0.f, lsum = 0.f;
    bool ok = true;
    // Until the latest P V_T has completed: P_T may then be rewritten and O_T is final.
    auto pv_wait = [&]() -> bool {
      if (pv_seen >= np) return true;
      const bool w = wait_bar(&bars->pv_done[tl], static_cast<uint32_t>(np - 1) & 1u, bars,
                              status);
      if (!__all_sync(0xffffffffu, w)) return false;
      pv_seen = np;
      return true;
    };
    // One step of this head on key block blk; returns false on abort.
    auto step = [&](int blk, int qi, bool first) -> bool {
      const bool w = wait_bar(&bars->s_full[tl], static_cast<uint32_t>(ns) & 1u, bars, status);
      if (!__all_sync(0xffffffffu, w)) return false;
      ++ns;
      tc_fence_after();
      uint32_t sr[kN];
      TC_LD32(s_addr, sr);
      TC_LD32(s_addr + 32, (sr + 32));
      TC_LD32(s_addr + 64, (sr + 64));
      TC_LD32(s_addr + 96, (sr + 96));
      tc_wait_ld_r32(sr);
      tc_wait_ld_r32(sr + 32);
      tc_wait_ld_r32(sr + 64);
      tc_wait_ld_r32(sr + 96);
      tc_fence_before();
      mbar_arrive(&bars->s_free[tl]);  // the next S_T may overwrite these columns
      if (blk == qi) {  // the diagonal block: token-causal
#pragma unroll
        for (int c = 0; c < kN; ++c)
          if (c > row) sr[c] = __float_as_uint(-INFINITY);
      }
      float mq[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) mq[e] = __uint_as_float(sr[e]);
#pragma unroll
      for (int c = 4; c < kN; c += 2)
        mq[(c >> 1) & 3] =
            max3(mq[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
      const float mx = max3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * sl2;
      if (first) {
        m_run = mx;
        lsum = 0.f;
      } else {
        const bool need = mx > m_run + kRescale;
        if (__any_sync(0xffffffffu, need)) {
          // rows whose max moved past the reference take the new max and rescale their row
          // of O_T (complete once the latest P V_T is); the others multiply by 1
          if (!pv_wait()) return false;
          const float alpha = need ? ex2(m_run - mx) : 1.0f;
          if (need) m_run = mx;
          lsum *= alpha;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            TC_LD32(o_addr + 32 * c, o);
            tc_wait_ld_r32(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            TC_ST32(o_addr + 32 * c, o);
          }
          tc_wait_st();
        }
      }
      // P = exp2(S * sl2 - m_run) packed to bf16; the row sum adds the bf16 values that enter
      // P V (mixed-precision adds take each half of a packed pair as it is), so the
      // normaliser and the products see the same P and a row that one key dominates returns
      // that key's V row.
      uint32_t p[kN / 2];
      f2 sum[2] = {f2{0.f, 0.f}, f2{0.f, 0.f}};
      {
        const f2 scl{sl2, sl2}, neg{-m_run, -m_run};
#pragma unroll
        for (int c = 0; c < kN / 2; ++c) {
          const f2 x =
              fma2(f2{__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])}, scl, neg);
          p[c] = pack_bf16(ex2(x.x), ex2(x.y));
          asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
              "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
              : "+f"(sum[c & 1].x), "+f"(sum[c & 1].y)
              : "r"(p[c]));
        }
      }
      if (!pv_wait()) return false;  // the previous P V_T has read P_T
      // the row's 256 bytes in the 128B-swizzled K-major layout of a TMA box (two boxes of 64
      // keys, 16 KB apart; 16-byte chunk j of row r at r*128 + ((j ^ (r % 8)) * 16))
#pragma unroll
      for (int k = 0; k < kN / 8; ++k)
        st_shared_v4(p_row + (k >> 3) * (kM * 128) + (((k & 7) ^ swz) << 4), p[4 * k],
                     p[4 * k + 1], p[4 * k + 2], p[4 * k + 3]);
      fence_proxy_async_smem();  // the tensor cores read P through the async proxy
      tc_fence_before();         // and O_T after a rescale
      mbar_arrive(&bars->p_full[tl]);
      ++np;
      lsum += (sum[0].x + sum[0].y) + (sum[1].x + sum[1].y);
      return true;
    };
    // At the item's end: when its last P V is complete, O * (1/l) -> bf16 into P_T's buffer
    // (free until the next item's first P), each thread its own row in the 128B-swizzled
    // layout P uses; O_T is released. Each warp then copies out the 32 rows its own lanes
    // wrote (so a warp barrier orders it), two rows (512 contiguous bytes of the output) per
    // instruction for D 128, with streaming stores: a thread storing its own row would touch
    // 32 rows per warp instruction.
    auto epilogue = [&](const Item& it) -> bool {
      if (!pv_wait()) return false;
      const float inv = 1.0f / lsum;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        TC_LD32(o_addr + 32 * c, o);
        tc_wait_ld_r32(o);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = 4 * c + q;  // 16-byte chunk of the row
          st_shared_v4(p_row + (k >> 3) * (kM * 128) + (((k & 7) ^ swz) << 4), w[4 * q],
                       w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->o_empty[tl]);
      __syncwarp();
      const int h = tl == 0 ? it.hA : it.hB;
      constexpr int kChunks = D / 8;      // 16-byte chunks of a row
      constexpr int kRows = 32 / kChunks;  // rows per instruction
      const int cj = lane % kChunks, rr = lane / kChunks;
      const int64_t row0 = static_cast<int64_t>(it.i) * kM + sub * 32;  // the warp's first row
      uint4* dst = reinterpret_cast<uint4*>(
                       out + ((static_cast<int64_t>(it.b) * Hq + h) * S + row0) * D) + cj;
      const uint32_t src = su32(p_tiles + tl * C::kPTile) + (cj >> 3) * (kM * 128);
#pragma unroll 4
      for (int t = 0; t < 32 / kRows; ++t) {
        const int r = sub * 32 + t * kRows + rr;  // row within the tile
        const uint4 v = ld_shared_v4(src + r * 128 + (((cj & 7) ^ (r & 7)) << 4));
        if (row0 + t * kRows + rr < S)  // rows past S in a partial last block are not written
          __stcs(dst + (t * kRows + rr) * kChunks, v);  // evict-first: keep K/V in L2
      }
      return true;
    };
    for (int64_t n = 0; ok; ++n) {
      int64_t t = -1;
      if (!__all_sync(0xffffffffu, read_item(bars, n, status, &t))) {
        ok = false;
        break;
      }
      if (t < 0) break;
      const Item it = decode(t, G, nb, Hkv, plan.order);
      if (tl == 1 && it.hB < 0) continue;  // a lone head A
      const int cnt = plan.k[it.i];
      const uint32_t* srow = sched_row(sched, it, Hkv, G, cap, plan);
      uint32_t e_next = srow[0];  // loaded one step ahead, as in Seq
      for (int j = 0; j < cnt && ok; ++j) {
        const uint32_t e = e_next;
        if (j + 1 < cnt) e_next = srow[j + 1];
        int ba, bb;
        sched_step(e, it.i, ba, bb);
        ok = step(tl == 0 ? ba : bb, it.i, j == 0);
      }
      if (!ok) break;
      ok = epilogue(it);
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
  const size_t smem = std::max<size_t>(Cfg<D>::kSmem, 120 * 1024);
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
  if (block == 64)
    return launch_attn_bf16_b64(q, k, v, B, Hq, Hkv, S, D, plan, cap, sel_idx, sched, out,
                                status, st);
  return cudaErrorInvalidValue;
}

}  // namespace stem

extern "C" int stem_test_withhold_q(int on) { return stem::g_withhold_q.exchange(on ? 1 : 0); }
