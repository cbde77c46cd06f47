// Block-sparse causal attention at block 64 on the Blackwell tensor cores (tcgen05 + TMEM +
// TMA), bf16 in, fp32 accumulation.
//
// Computes, for every query token of query block i, exact softmax attention over every token of
// the kept key blocks of row (b, h, i), token-causal inside block i ("Stem: Rethinking Causal
// Information Flow in Sparse Attention", gist.science/es "Resumen tecnico" 2 "Implementacion"
// step 3; gist.science/it 2.C step 3; gist.science/nl "Implementatie" step 3; gist.science/fr
// 2.C step 3).
//
// A tensor-core tile has 128 query rows; a block holds 64. A tile therefore stacks the query
// block i of two GQA sibling heads (a head pair: rows 0-63 the first head, rows 64-127 the
// second), which keep the same number k(i) of key blocks. The pairing kernel's step schedule
// (pairs.cu) gives, per step, the key block of each head of the pair; the step's K/V tile holds
// both blocks (keys 0-63 the first head's, 64-127 the second's) or, when both heads keep the same
// block or the pair has one head, that block alone. So S = Q K^T is a 128 x 128 product whose two
// cross quadrants are masked (each head's rows see only its own block), or a 128 x 64 product;
// P V then runs over 128 or 64 keys, and the masked entries of P are zero.
//
// Work item: the query block i of up to two head pairs of one kv-head group (tiles A and B).
// The kernel is the block-128 kernel's design (attn_sm100.cu) on these tiles: persistent, one CTA
// per SM, 12 warps (TMA producer, MMA issuer, two idle warps, one softmax warpgroup per tile with
// one thread per query row), P written to shared memory, the next S of a tile issued as soon as
// the softmax has read the current one, work items claimed at run time, bounded waits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "attn_common.cuh"
#include "sm100.cuh"
#include "stem.h"
#include "stem_internal.h"

namespace stem {
namespace {

constexpr int kM = 128;   // query rows per tile: two blocks
constexpr int kBlk = 64;  // tokens per block

template <int D>
struct Cfg64 {
  static constexpr uint32_t kTile = kM * D * 2;    // a 128 x D bf16 tile (two 64-row halves)
  static constexpr uint32_t kHalf = kBlk * D * 2;  // one block of rows
  static constexpr uint32_t kPTile = kM * kN * 2;  // a 128 x 128 bf16 P tile
  static constexpr int kBoxes = D / 64;            // 128B-swizzled boxes of 64 columns
  static constexpr int kKSteps = D / 16;           // MMA k-steps of QK^T
  static constexpr int kSlots = D == 128 ? 3 : 4;  // what fits beside Q and P
  static constexpr size_t kSmem =
      1024 + 2 * kTile + 2 * kPTile + kSlots * static_cast<size_t>(kTile) + sizeof(Bars);
};
static_assert(Cfg64<128>::kSmem <= 232448, "shared memory of the D = 128 kernel");

// Work item t -> (b, g, q, i): kv-head-group-major, query blocks in the plan's heavy-first
// order, the ceil(P/2) tile pairs of a group adjacent (P = ceil(G/2) head pairs). Tile A is head
// pair 2q, tile B head pair 2q + 1 (absent when P is odd and this is the group's last item); head
// pair p is heads g*G + 2p and g*G + 2p + 1 (the second absent when G is odd and p the last).
struct Item64 {
  int b, g, i;
  int pA, pB;        // head pairs (pB < 0: no tile B)
  int h[2][2];       // [tile][half] head, -1 when absent
};
__device__ __forceinline__ Item64 decode64(int64_t t, int G, int nb, int Hkv,
                                          const int32_t* order) {
  const int P = (G + 1) >> 1;
  const int Qd = (P + 1) >> 1;
  const int64_t per_group = static_cast<int64_t>(Qd) * nb;
  const int64_t bg = t / per_group;
  const int rem = static_cast<int>(t % per_group);
  Item64 it;
  it.i = order[rem / Qd];
  it.b = static_cast<int>(bg / Hkv);
  it.g = static_cast<int>(bg % Hkv);
  const int q = rem % Qd;
  it.pA = 2 * q;
  it.pB = 2 * q + 1 < P ? 2 * q + 1 : -1;
#pragma unroll
  for (int tl = 0; tl < 2; ++tl) {
    const int p = tl == 0 ? it.pA : it.pB;
    const int h0 = it.g * G + 2 * p;
    it.h[tl][0] = p >= 0 ? h0 : -1;
    it.h[tl][1] = (p >= 0 && 2 * p + 1 < G) ? h0 + 1 : -1;
  }
  return it;
}
__device__ __forceinline__ const uint32_t* sched_row64(const uint32_t* sched, const Item64& it,
                                                       int p, int Hkv, int G, int64_t cap,
                                                       const PlanDev& plan) {
  const int P = (G + 1) >> 1;
  const int64_t gp = (static_cast<int64_t>(it.b) * Hkv + it.g) * P + p;
  return sched + gp * cap + plan.off[it.i];
}

// One step of an item: the key blocks of the two halves of each tile (k[tile][1] < 0: the
// tile's second head keeps the same block or is absent; then the step's K/V tile of that tile
// is one block and its S has 64 columns).
struct Step64 {
  bool first, last;
  Item64 it;
  int k[2][2];
  __device__ __forceinline__ bool has_b() const { return it.pB >= 0; }
  __device__ __forceinline__ bool two(int tl) const { return k[tl][1] >= 0; }
};
__device__ __forceinline__ void split_entry(uint32_t e, int i, int* k) {
  int a, b;
  sched_step(e, i, a, b);
  k[0] = a;
  k[1] = (b >= 0 && b != a) ? b : -1;
}

struct Seq64 {
  int64_t t, items;
  int G, nb, Hkv;
  int64_t cap;
  PlanDev plan;
  const uint32_t* sched;
  Bars* bars;
  unsigned long long* counter;  // non-null: this walker claims items (the producer)
  int32_t* status;
  bool failed;
  int n, j, cnt;
  Item64 it;
  const uint32_t* row[2];
  uint32_t e_next[2];  // schedule entries of the coming step, loaded one call ahead
  __device__ __forceinline__ void init(int64_t items_, int G_, int nb_, int Hkv_, int64_t cap_,
                                       PlanDev plan_, const uint32_t* sched_, Bars* bars_,
                                       unsigned long long* counter_, int32_t* status_) {
    items = items_; G = G_; nb = nb_; Hkv = Hkv_; cap = cap_; plan = plan_;
    sched = sched_; bars = bars_; counter = counter_; status = status_;
    failed = false;
    n = -1; j = 0; cnt = 0;
  }
  __device__ __forceinline__ bool next(Step64& s) {
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
      it = decode64(t, G, nb, Hkv, plan.order);
      cnt = plan.k[it.i];
      j = 0;
      row[0] = sched_row64(sched, it, it.pA, Hkv, G, cap, plan);
      e_next[0] = row[0][0];
      if (it.pB >= 0) {
        row[1] = sched_row64(sched, it, it.pB, Hkv, G, cap, plan);
        e_next[1] = row[1][0];
      }
    }
    const uint32_t e0 = e_next[0], e1 = e_next[1];
    if (j + 1 < cnt) {
      e_next[0] = row[0][j + 1];
      if (it.pB >= 0) e_next[1] = row[1][j + 1];
    }
    s.first = (j == 0);
    s.last = (j == cnt - 1);
    s.it = it;
    split_entry(e0, it.i, s.k[0]);
    if (it.pB >= 0) split_entry(e1, it.i, s.k[1]);
    ++j;
    return true;
  }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_b64_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, int Hq, int Hkv, int S,
                          int nb, int64_t items, PlanDev plan, int64_t cap,
                          unsigned long long* counter, const uint32_t* __restrict__ sched,
                          __nv_bfloat16* __restrict__ out, int32_t* status, int withhold_q) {
  using C = Cfg64<D>;
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

  // Registers as in the block-128 kernel: 4 x 32 x 72 + 8 x 32 x 216 = 384 x 168.
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
      // x, K(x, A), K(x, B), V(c, A), V(c, B) inside an item, V before K when x starts the next
      // item. A K/V tile holds the key blocks of both halves of its Q tile (64 rows each), or
      // one block.
      int64_t f = 0;
      int64_t slot_round[kMaxSlots];
      for (int s = 0; s < kMaxSlots; ++s) slot_round[s] = -1;
      int64_t q_loads[2] = {0, 0};
      bool ok = true;
      auto fill = [&](const CUtensorMap* map, const Step64& st, int tl) -> bool {
        const int s = static_cast<int>(f % kSlots);
        const int64_t r = f / kSlots;
        if (!wait_bar(&bars->kv_empty[s], static_cast<uint32_t>((r & 1) ^ 1), bars, status))
          return false;
        const bool two = st.two(tl);
        mbar_expect_tx(&bars->kv_full[s], two ? 2 * C::kHalf : C::kHalf);
        const int head = st.it.b * Hkv + st.it.g;
        for (int hf = 0; hf < (two ? 2 : 1); ++hf)
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(kv_tiles + s * C::kTile + x * (kM * 128) + hf * (kBlk * 128), map,
                        x * 64, st.k[tl][hf] * kBlk, head, &bars->kv_full[s], pol_kv);
        slot_round[s] = r;
        ++f;
        return true;
      };
      // Q of a tile at an item's start: block i of its pair's first head into rows 0-63, of the
      // second head (when there is one) into rows 64-127
      auto load_q = [&](const Step64& st, int tl) -> bool {
        if (withhold_q && tl == 0 && q_loads[0] == 0) return true;  // test switch: never sent
        const int64_t r = q_loads[tl];
        if (!wait_bar(&bars->q_empty[tl], static_cast<uint32_t>((r & 1) ^ 1), bars, status))
          return false;
        const bool two = st.it.h[tl][1] >= 0;
        mbar_expect_tx(&bars->q_full[tl], two ? 2 * C::kHalf : C::kHalf);
        for (int hf = 0; hf < (two ? 2 : 1); ++hf)
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(q_tiles + tl * C::kTile + x * (kM * 128) + hf * (kBlk * 128), &tm_q,
                        x * 64, st.it.i * kBlk, st.it.b * Hq + st.it.h[tl][hf],
                        &bars->q_full[tl], pol_q);
        ++q_loads[tl];
        return true;
      };
      auto fill_k = [&](const Step64& st) -> bool {  // Q at an item's start, then the K tiles
        if (st.first) {
          if (!load_q(st, 0)) return false;
          if (st.has_b() && !load_q(st, 1)) return false;
        }
        if (!fill(&tm_k, st, 0)) return false;
        return !st.has_b() || fill(&tm_k, st, 1);
      };
      auto fill_v = [&](const Step64& st) -> bool {
        if (!fill(&tm_v, st, 0)) return false;
        return !st.has_b() || fill(&tm_v, st, 1);
      };
      Seq64 seq;
      seq.init(items, G, nb, Hkv, cap, plan, sched, bars, counter, status);
      Step64 x;
      bool have = seq.next(x);
      if (seq.failed) ok = false;
      if (have) ok = fill_k(x);
      while (have && ok) {
        const Step64 c = x;
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
    // Per step c with successor x: S_A(x), S_B(x), P V_A(c), P V_B(c) (at an item boundary the
    // P V groups first), as in the block-128 kernel; S has 128 or 64 key columns and P V 128 or
    // 64 keys, by whether the tile's K/V tile holds one block or two.
    if (lane == 0) {
      constexpr uint32_t idesc_s2 = instr_desc(kM, 2 * kBlk, false);
      constexpr uint32_t idesc_s1 = instr_desc(kM, kBlk, false);
      constexpr uint32_t idesc_o = instr_desc(kM, D, true);
      constexpr uint32_t kTileU = C::kTile >> 4;    // a tile's size in descriptor units
      constexpr uint32_t kPTileU = C::kPTile >> 4;
      const uint32_t hi = smem_desc_hi(1024);
      const uint32_t q_lo = smem_desc_lo(su32(q_tiles), 16);
      const uint32_t p_lo = smem_desc_lo(su32(p_tiles), 16);
      const uint32_t k_lo = smem_desc_lo(su32(kv_tiles), 16);
      const uint32_t v_lo = smem_desc_lo(su32(kv_tiles), kM * 128);
      int32_t f = 0;
      int32_t nq[2] = {0, 0}, ns[2] = {0, 0}, np[2] = {0, 0}, no[2] = {0, 0};
      bool ok = true;
      auto kv_try = [&](int32_t t) {
        return mbar_try(&bars->kv_full[t % kSlots], static_cast<uint32_t>(t / kSlots) & 1u);
      };
      auto kv_wait = [&](int32_t t) {
        return wait_bar(&bars->kv_full[t % kSlots], static_cast<uint32_t>(t / kSlots) & 1u, bars,
                        status);
      };
      auto issue_s = [&](const Step64& s, int tl) -> bool {
        const int32_t kt = f++;
        const uint32_t qp = static_cast<uint32_t>(nq[tl]) & 1u;
        const uint32_t sp = static_cast<uint32_t>(ns[tl] - 1) & 1u;
        bool r = kv_try(kt);
        if (s.first) r &= mbar_try(&bars->q_full[tl], qp);
        if (ns[tl] > 0) r &= mbar_try(&bars->s_free[tl], sp);
        if (!r && !(kv_wait(kt) && (!s.first || wait_bar(&bars->q_full[tl], qp, bars, status)) &&
                    (ns[tl] == 0 || wait_bar(&bars->s_free[tl], sp, bars, status))))
          return false;
        if (s.first) ++nq[tl];
        ++ns[tl];
        tc_fence_after();
        const uint32_t a = q_lo + tl * kTileU;
        const uint32_t b = k_lo + static_cast<uint32_t>(kt % kSlots) * kTileU;
        const uint32_t idesc = s.two(tl) ? idesc_s2 : idesc_s1;
        if constexpr (C::kKSteps == 8) {
          mma_s8(tmem + tl * 128, a, b, hi, idesc);
        } else {
          static_assert(C::kKSteps == 4, "D 128 or 64");
          mma_s4(tmem + tl * 128, a, b, hi, idesc);
        }
        tc_commit(&bars->s_full[tl]);
        if (s.last) tc_commit(&bars->q_empty[tl]);
        tc_commit(&bars->kv_empty[kt % kSlots]);
        return true;
      };
      auto issue_pv = [&](const Step64& c, int tl) -> bool {
        const int32_t vt = f++;
        const uint32_t pp = static_cast<uint32_t>(np[tl]) & 1u;
        const uint32_t op = static_cast<uint32_t>(no[tl] - 1) & 1u;
        const bool wo = c.first && no[tl] > 0;
        bool r = mbar_try(&bars->p_full[tl], pp) & kv_try(vt);
        if (wo) r &= mbar_try(&bars->o_empty[tl], op);
        if (!r && !(wait_bar(&bars->p_full[tl], pp, bars, status) && kv_wait(vt) &&
                    (!wo || wait_bar(&bars->o_empty[tl], op, bars, status))))
          return false;
        if (c.first) ++no[tl];
        ++np[tl];
        tc_fence_after();
        const uint32_t vlo = v_lo + static_cast<uint32_t>(vt % kSlots) * kTileU;
        const uint32_t acc0 = c.first ? 0u : 1u;
        if (c.two(tl))
          mma_pv8(tmem + 256 + tl * 128, p_lo + tl * kPTileU, vlo, hi, idesc_o, acc0);
        else
          mma_pv4(tmem + 256 + tl * 128, p_lo + tl * kPTileU, vlo, hi, idesc_o, acc0);
        tc_commit(&bars->pv_done[tl]);
        tc_commit(&bars->kv_empty[vt % kSlots]);
        return true;
      };
      auto s_step = [&](const Step64& s) -> bool {
        return issue_s(s, 0) && (!s.has_b() || issue_s(s, 1));
      };
      auto pv_step = [&](const Step64& c) -> bool {
        return issue_pv(c, 0) && (!c.has_b() || issue_pv(c, 1));
      };
      Seq64 seq;
      seq.init(items, G, nb, Hkv, cap, plan, sched, bars, nullptr, status);
      Step64 x;
      bool have = seq.next(x);
      if (seq.failed) ok = false;
      if (have) ok = s_step(x);
      while (have && ok) {
        const Step64 c = x;
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
    const int tl = (warp - 4) >> 2;     // 0: tile A (warps 4-7), 1: tile B (warps 8-11)
    const int sub = warp & 3;           // TMEM sub-partition of this warp
    const int row = sub * 32 + lane;    // query row within the tile
    const int half = row >> 6;          // 0: the pair's first head, 1: its second
    const int r6 = row & 63;            // query row within the block
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t s_addr = tmem + tl * 128 + lane_off;
    const uint32_t o_addr = tmem + 256 + tl * 128 + lane_off;
    const uint32_t p_row = su32(p_tiles + tl * C::kPTile) + static_cast<uint32_t>(row) * 128;
    const uint32_t swz = static_cast<uint32_t>(row & 7);
    const float sl2 = 1.4426950408889634f * rsqrtf(static_cast<float>(D));
    int32_t ns = 0, np = 0, pv_seen = 0;
    float m_run = 0.f, lsum = 0.f;
    bool ok = true;
    auto pv_wait = [&]() -> bool {
      if (pv_seen >= np) return true;
      const bool w = wait_bar(&bars->pv_done[tl], static_cast<uint32_t>(np - 1) & 1u, bars,
                              status);
      if (!__all_sync(0xffffffffu, w)) return false;
      pv_seen = np;
      return true;
    };
    // One step of this tile; `two`: its K/V tile holds two blocks (keys 0-63 for the rows of
    // the first head, 64-127 for the second), else one block for all rows; blk: the key block
    // of this row's half. Each row reads, exponentiates and writes only its own block's 64
    // columns; with two blocks the other half of its P row is written as zeros. Returns false
    // on abort.
    constexpr int kC = kBlk;  // key columns of a row
    auto step = [&](bool two, int blk, int qi, bool first) -> bool {
      const bool w = wait_bar(&bars->s_full[tl], static_cast<uint32_t>(ns) & 1u, bars, status);
      if (!__all_sync(0xffffffffu, w)) return false;
      ++ns;
      tc_fence_after();
      const int c0 = two ? half * kBlk : 0;  // warp-uniform: a warp's rows share a half
      uint32_t sr[kC];
      TC_LD32(s_addr + c0, sr);
      TC_LD32(s_addr + c0 + 32, (sr + 32));
      tc_wait_ld_r32(sr);
      tc_wait_ld_r32(sr + 32);
      tc_fence_before();
      mbar_arrive(&bars->s_free[tl]);  // the next S_T may overwrite these columns
      if (blk == qi) {  // the diagonal block: token-causal
#pragma unroll
        for (int c = 0; c < kC; ++c)
          if (c > r6) sr[c] = __float_as_uint(-INFINITY);
      }
      float mq[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) mq[e] = __uint_as_float(sr[e]);
#pragma unroll
      for (int c = 4; c < kC; c += 2)
        mq[(c >> 1) & 3] =
            max3(mq[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
      const float mx = max3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * sl2;
      if (first) {
        m_run = mx;
        lsum = 0.f;
      } else {
        const bool need = mx > m_run + kRescale;
        if (__any_sync(0xffffffffu, need)) {
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
      // P against the reference max, packed to bf16; the row sum adds the bf16 values that
      // enter P V
      uint32_t p[kC / 2];
      f2 sum[2] = {f2{0.f, 0.f}, f2{0.f, 0.f}};
      {
        const f2 scl{sl2, sl2}, neg{-m_run, -m_run};
#pragma unroll
        for (int c = 0; c < kC / 2; ++c) {
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
      // the row's keys c0 .. c0+63 are box c0 / 64 of the P tile (16-byte chunk j of row r at
      // r*128 + ((j ^ (r % 8)) * 16)); with two blocks the other box of the row is zero
      const uint32_t own = p_row + static_cast<uint32_t>(c0 / kBlk) * (kM * 128);
#pragma unroll
      for (int k = 0; k < kC / 8; ++k)
        st_shared_v4(own + ((k ^ swz) << 4), p[4 * k], p[4 * k + 1], p[4 * k + 2], p[4 * k + 3]);
      if (two) {
        const uint32_t other = p_row + static_cast<uint32_t>(1 - c0 / kBlk) * (kM * 128);
#pragma unroll
        for (int k = 0; k < kC / 8; ++k) st_shared_v4(other + ((k ^ swz) << 4), 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full[tl]);
      ++np;
      lsum += (sum[0].x + sum[0].y) + (sum[1].x + sum[1].y);
      return true;
    };
    // At the item's end: O * (1/l) -> bf16 -> global for the rows of a present head.
    auto epilogue = [&](const Item64& it) -> bool {
      if (!pv_wait()) return false;
      const float inv = 1.0f / lsum;
      tc_fence_after();
      const int h = it.h[tl][half];
      const int64_t pos = static_cast<int64_t>(it.i) * kBlk + r6;
      const bool valid = h >= 0 && pos < S;  // partial last block, absent second head
      __nv_bfloat16* dst =
          out + ((static_cast<int64_t>(it.b) * Hq + (h >= 0 ? h : 0)) * S + pos) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
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
          for (int e = 0; e < 4; ++e) __stcs(d4 + e, pk[e]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->o_empty[tl]);
      return true;
    };
    for (int64_t n = 0; ok; ++n) {
      int64_t t = -1;
      if (!__all_sync(0xffffffffu, read_item(bars, n, status, &t))) {
        ok = false;
        break;
      }
      if (t < 0) break;
      const Item64 it = decode64(t, G, nb, Hkv, plan.order);
      if (tl == 1 && it.pB < 0) continue;  // no tile B in this item
      const int cnt = plan.k[it.i];
      const uint32_t* srow = sched_row64(sched, it, tl == 0 ? it.pA : it.pB, Hkv, G, cap, plan);
      uint32_t e_next = srow[0];  // loaded one step ahead, as in Seq64
      for (int j = 0; j < cnt && ok; ++j) {
        const uint32_t e = e_next;
        if (j + 1 < cnt) e_next = srow[j + 1];
        int k2[2];
        split_entry(e, it.i, k2);
        const bool two = k2[1] >= 0;
        ok = step(two, two ? k2[half] : k2[0], it.i, j == 0);
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

// 3-D view [heads, S, D] of a bf16 tensor, boxes of 64 columns x 64 tokens x 1 head, 128B
// swizzle. Token rows past S are outside the view: a box over a partial last block reads them
// as 0.
bool make_map64(CUtensorMap* m, const void* base, uint64_t heads, int S, int D) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), heads};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kBlk), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_b64(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                       int S, PlanDev plan, int64_t cap, const int32_t* sel_idx,
                       uint32_t* sched, void* out, int32_t* status, cudaStream_t st) {
  const int nb = (S + kBlk - 1) / kBlk;
  const int G = Hq / Hkv;
  const int P = (G + 1) / 2;
  const int64_t items = static_cast<int64_t>(B) * Hkv * nb * ((P + 1) / 2);
  if (items == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  if (!make_map64(&tq, q, static_cast<uint64_t>(B) * Hq, S, D) ||
      !make_map64(&tk, k, static_cast<uint64_t>(B) * Hkv, S, D) ||
      !make_map64(&tv, v, static_cast<uint64_t>(B) * Hkv, S, D))
    return cudaErrorInvalidValue;
  const size_t smem = std::max<size_t>(Cfg64<D>::kSmem, 120 * 1024);
  auto kern = attn_sm100_b64_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
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

cudaError_t launch_attn_bf16_b64(const void* q, const void* k, const void* v, int B, int Hq,
                                 int Hkv, int S, int D, PlanDev plan, int64_t cap,
                                 const int32_t* sel_idx, uint32_t* sched, void* out,
                                 int32_t* status, cudaStream_t st) {
  if (D == 128)
    return launch_b64<128>(q, k, v, B, Hq, Hkv, S, plan, cap, sel_idx, sched, out, status, st);
  if (D == 64)
    return launch_b64<64>(q, k, v, B, Hq, Hkv, S, plan, cap, sel_idx, sched, out, status, st);
  return cudaErrorInvalidValue;
}

}  // namespace stem
