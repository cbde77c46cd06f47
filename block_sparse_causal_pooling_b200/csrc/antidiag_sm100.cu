// Block probabilities by anti-diagonal sampling, on the Blackwell tensor cores (tcgen05 + TMEM +
// TMA), bf16 in, fp32 accumulation.
//
// Method ("Stem: Rethinking Causal Information Flow in Sparse Attention", gist.science/fr
// "Resume technique" 2.C step 1: the per-block metrics are computed with anti-diagonal sampling
// for efficiency). Tokens form groups of `stride` (sigma) consecutive tokens. Query group u and
// key group w span a sigma x sigma sub-tile of Q K^T / sqrt(D); the mean of its anti-diagonal
// samples stands for it:
//   a_uw = (1/sigma) sum_t Q[u sigma + t] . K[w sigma + sigma-1-t] / sqrt(D).
// Each query group takes a softmax over the key groups it sees causally (w <= u), and
//   p_ij = (1/n_i) sum_{u in block i} sum_{w in block j} softmax_w(a_u.)
// averages over the n_i query groups of block i the mass they put on block j.
//
// The sum over t and the feature dimension is one contraction of length sigma*D between
//   Q'[u] = Q[u sigma .. u sigma + sigma-1] read as one row of sigma*D elements, and
//   K'[w] = the same view of K with its sigma token chunks taken in reverse order,
// so a_uw = Q'[u] . K'[w] / (sigma sqrt(D)) is a plain GEMM over [S/sigma, sigma*D] views of
// the inputs: no copy is made. The reversal costs nothing: the k-step that reads chunk t of Q'
// reads chunk sigma-1-t of K', which is only a different TMA box coordinate.
//
// Persistent kernel, one CTA per SM, 10 warps. Work unit: (b, h, 128 consecutive query groups),
// claimed from a global counter in kv-head-major order (the units in flight share one kv head's
// K', which stays in L2) and handed to the other roles through a ring in shared memory.
//   warp 0    TMA producer: for every key tile (256 key groups, up to the unit's causal end) and
//             every k-step (64 of the sigma*D columns), the Q' box (128 x 64) and the K' box
//             (256 x 64) into a 4-stage ring of 128B-swizzled shared-memory tiles.
//   warp 1    allocates the 512 TMEM columns; lane 0 issues tcgen05.mma (M 128, N 256, K 16)
//             into one of two 256-column fp32 accumulators, so the epilogue of one key tile
//             overlaps the products of the next.
//   warps 2-5 tile epilogue, one query group (TMEM lane) per thread: online softmax over the
//             32-column chunks of each key tile in base 2 (running max m, running sum l), one
//             TMEM read per chunk; per key block the sum of exp2(a - m) over its key groups goes
//             to a scratch row, and each chunk's m (its snapshot) beside it. At the unit's end
//             m and l go to shared memory and the unit's scratch slot is handed over.
//   warps 6-9 fixup, while warps 2-5 work on the next unit (two scratch slots per CTA): each
//             value is rescaled to its row's final m and divided by l, the block's query groups
//             are summed with shuffles and p_ij is written.
// Q' tiles load with evict_last (a unit re-reads its Q' tile for every key tile); scratch and p
// move with streaming loads and stores, so that they do not push Q' and K' out of L2.
// Every mbarrier wait is bounded by the global nanosecond timer; on expiry the CTA records
// STEM_ERR_TIMEOUT, every role leaves its loop, issued products and copies are drained (bounded)
// and TMEM is freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "sm100.cuh"
#include "stem.h"
#include "stem_internal.h"

namespace stem {
namespace {

using namespace sm100;

constexpr int kAM = 128;              // query groups per tile (MMA M)
constexpr int kAN = 256;              // key groups per tile (MMA N)
constexpr int kStages = 4;            // shared-memory ring
constexpr int kAThreads = 320;        // 10 warps
constexpr int kEpiThreads = 128;      // warps 2-5
constexpr int kFixThreads = 128;      // warps 6-9
constexpr uint32_t kQBox = kAM * 128;  // 128 rows x 64 bf16
constexpr uint32_t kKBox = kAN * 128;  // 256 rows x 64 bf16
constexpr uint32_t kStageBytes = kQBox + kKBox;
constexpr uint32_t kTmemCols = 512;
constexpr int kUnitRing = 8;          // unit indices handed from the producer to the other roles
constexpr int kUnitReaders = 1 + kEpiThreads + kFixThreads;  // MMA thread, warps 2-9

struct __align__(8) ABars {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t unit_done[2], fix_done[2];  // per scratch slot: tiles done -> fixup done
  uint64_t uq_full[kUnitRing], uq_empty[kUnitRing];
  uint64_t drain;
  int64_t uq[kUnitRing];  // unit index, or -1: no more units
  uint32_t tmem_base;
  volatile int abort;
  float ml[2][2][kAM];  // [slot][running max m, running sum l][query group of the tile]
};

struct AdParams {
  int Hq, Hkv, nb, R;   // R = block / stride: groups per block (1 .. 32)
  int nred, nqt;        // groups per head, query tiles per head
  int ksteps, kparts;   // stride*D/64 k-steps; D/64 of them per token chunk
  int stride, D;
  int64_t units;        // B * Hq * nqt
  float scale_log2;     // log2(e) / (stride * sqrt(D))
  float* p;             // [B*Hq][nb*(nb+1)/2]
  unsigned long long* next_unit;  // work counter, 0 at launch
  float* scratch;       // [gridDim.x][2 slots][nb*128 + 8*nkt_max*128]
  int64_t scratch_per_slot;
  int32_t* status;
  int withhold;         // test switch: the first stage's copies are never sent
};

__device__ __noinline__ bool ad_wait_slow(uint64_t* b, uint32_t parity, ABars* bars,
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
__device__ __forceinline__ bool ad_wait(uint64_t* b, uint32_t parity, ABars* bars,
                                        int32_t* status) {
  return mbar_try(b, parity) || ad_wait_slow(b, parity, bars, status);
}

// Unit t -> (bh, qt). kv-head-major, so that the units in flight share one kv head's K' (which
// then stays in L2); inside a kv head the heaviest query tiles first (a tile's key range grows
// with qt), the G query heads of a tile next to each other. CTAs take units from a global
// counter, so the order is the order of issue, not a fixed assignment.
struct AUnit {
  int bh, qt, nkt, kvh;
};
__device__ __forceinline__ AUnit ad_unit(int64_t t, const AdParams& P) {
  const int G = P.Hq / P.Hkv;
  const int64_t per_kv = static_cast<int64_t>(G) * P.nqt;
  const int kvh = static_cast<int>(t / per_kv);  // b * Hkv + kv head
  const int r = static_cast<int>(t % per_kv);
  AUnit u;
  u.kvh = kvh;
  u.qt = P.nqt - 1 - r / G;
  u.bh = (kvh / P.Hkv) * P.Hq + (kvh % P.Hkv) * G + r % G;
  const int last = min(P.nred - 1, u.qt * kAM + kAM - 1);  // last query group of the tile
  u.nkt = last / kAN + 1;                                   // key tiles 0 .. (last / 256)
  return u;
}

// The n-th unit of this CTA from the ring (every reader calls this once per unit, in order).
__device__ __forceinline__ bool ad_next_unit(ABars* bars, int64_t n, int32_t* status,
                                             int64_t* t) {
  const int q = static_cast<int>(n % kUnitRing);
  if (!ad_wait(&bars->uq_full[q], static_cast<uint32_t>((n / kUnitRing) & 1), bars, status))
    return false;
  *t = bars->uq[q];
  mbar_arrive(&bars->uq_empty[q]);
  return true;
}

__global__ void __launch_bounds__(kAThreads, 1)
    antidiag_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k, AdParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  ABars* bars = reinterpret_cast<ABars*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->acc_full[s], 1);
      mbar_init(&bars->acc_empty[s], kEpiThreads);
      mbar_init(&bars->unit_done[s], kEpiThreads);
      mbar_init(&bars->fix_done[s], kFixThreads);
    }
    for (int s = 0; s < kUnitRing; ++s) {
      mbar_init(&bars->uq_full[s], 1);
      mbar_init(&bars->uq_empty[s], kUnitReaders);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
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
      // a unit re-reads its Q' tile for every key tile: keep it; K' tiles pass through
      const uint64_t pol_q = policy_evict_last(), pol_k = policy_evict_normal();
      int64_t f = 0;
      bool ok = true;
      for (int64_t n = 0; ok; ++n) {
        // claim the next unit and publish it to the other roles (-1: none left)
        int64_t t = static_cast<int64_t>(atomicAdd(P.next_unit, 1ull));
        if (t >= P.units) t = -1;
        const int q = static_cast<int>(n % kUnitRing);
        if (!(ok = ad_wait(&bars->uq_empty[q], static_cast<uint32_t>(((n / kUnitRing) & 1) ^ 1),
                           bars, P.status)))
          break;
        bars->uq[q] = t;
        mbar_arrive(&bars->uq_full[q]);
        if (t < 0) break;
        const AUnit u = ad_unit(t, P);
        const int kvh = u.kvh;
        for (int kt = 0; kt < u.nkt && ok; ++kt) {
          for (int ks = 0; ks < P.ksteps; ++ks) {
            const int s = static_cast<int>(f % kStages);
            const int64_t r = f / kStages;
            if (!(ok = ad_wait(&bars->empty[s], static_cast<uint32_t>((r & 1) ^ 1), bars,
                               P.status)))
              break;
            mbar_expect_tx(&bars->full[s], kStageBytes);
            if (P.withhold && f == 0) {  // test switch: the stage's bytes never arrive
              ++f;
              continue;
            }
            const int chunk = ks / P.kparts, part = ks % P.kparts;
            unsigned char* st = smem + s * kStageBytes;
            tma_load_3d(st, &tm_q, ks * 64, u.qt * kAM, u.bh, &bars->full[s], pol_q);
            tma_load_3d(st + kQBox, &tm_k, (P.stride - 1 - chunk) * P.D + part * 64, kt * kAN,
                        kvh, &bars->full[s], pol_k);
            ++f;
          }
        }
      }
      if (!ok) {  // abort: let the copies in flight land before the CTA can exit
        for (int64_t g = f - kStages < 0 ? 0 : f - kStages; g < f; ++g)
          drain_bar(&bars->full[g % kStages], static_cast<uint32_t>((g / kStages) & 1));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(kAM, kAN, false);
      const uint32_t base = su32(smem);
      int64_t f = 0, tiles = 0;
      bool ok = true;
      for (int64_t n = 0; ok; ++n) {
        int64_t t;
        if (!(ok = ad_next_unit(bars, n, P.status, &t)) || t < 0) break;
        const AUnit u = ad_unit(t, P);
        for (int kt = 0; kt < u.nkt && ok; ++kt) {
          const int buf = static_cast<int>(tiles & 1);
          const int64_t use = tiles >> 1;
          if (!(ok = ad_wait(&bars->acc_empty[buf], static_cast<uint32_t>((use & 1) ^ 1), bars,
                             P.status)))
            break;
          tc_fence_after();
          const uint32_t d_tm = tmem + buf * kAN;
          for (int ks = 0; ks < P.ksteps; ++ks) {
            const int s = static_cast<int>(f % kStages);
            if (!(ok = ad_wait(&bars->full[s], static_cast<uint32_t>((f / kStages) & 1), bars,
                               P.status)))
              break;
            tc_fence_after();
            const uint32_t qa = base + s * kStageBytes, ka = qa + kQBox;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(d_tm, smem_desc(qa + kk * 32, 16, 1024), smem_desc(ka + kk * 32, 16, 1024),
                     idesc, (ks | kk) != 0 ? 1u : 0u);
            tc_commit(&bars->empty[s]);  // the stage is free once these products are done
            ++f;
          }
          if (!ok) break;
          tc_commit(&bars->acc_full[buf]);
          ++tiles;
        }
      }
      tc_commit(&bars->drain);  // every issued product completes before TMEM is released
      drain_bar(&bars->drain, 0);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ tile epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int R = P.R;
    int64_t tiles = 0, n = 0;
    bool ok = true;
    for (; ok; ++n) {
      int64_t t;
      ok = __all_sync(0xffffffffu, ad_next_unit(bars, n, P.status, &t));
      if (!ok || t < 0) break;
      const AUnit un = ad_unit(t, P);
      const int slot = static_cast<int>(n & 1);
      // the slot's previous unit (n - 2) must be through its fixup before it is overwritten
      ok = __all_sync(0xffffffffu, ad_wait(&bars->fix_done[slot],
                                           static_cast<uint32_t>(((n >> 1) & 1) ^ 1), bars,
                                           P.status));
      if (!ok) break;
      float* esc = P.scratch + (2 * static_cast<int64_t>(blockIdx.x) + slot) * P.scratch_per_slot;
      float* msc = esc + static_cast<int64_t>(P.nb) * kAM;  // [nkt * 8 chunks][128] snapshots
      const int u = un.qt * kAM + row;  // this thread's query group
      float m_run = -INFINITY, l_run = 0.f;
      for (int kt = 0; kt < un.nkt; ++kt) {
        const int buf = static_cast<int>(tiles & 1);
        const int64_t use = tiles >> 1;
        // warp-uniform: the TMEM loads below are .sync.aligned
        ok = __all_sync(0xffffffffu,
                        ad_wait(&bars->acc_full[buf], static_cast<uint32_t>(use & 1), bars,
                                P.status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem + lane_addr + buf * kAN;
        // One pass per 32-column chunk: the exact running max over the columns seen so far,
        // exp2 against it, sums by tree. Each chunk's sums are stored with the max they were
        // taken against (its snapshot), so no column is read twice.
#pragma unroll 1
        for (int ch = 0; ch < kAN / 32; ++ch) {
          uint32_t r[32];
          TC_LD32(taddr + ch * 32, r);
          tc_wait_ld();
          const int lim = u - kt * kAN - ch * 32;  // columns c <= lim are visible (w <= u)
          float x[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = c <= lim ? __uint_as_float(r[c]) : -INFINITY;
          float mx[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) mx[c] = fmaxf(x[c], x[c + 16]);
#pragma unroll
          for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
            for (int c = 0; c < w; ++c) mx[c] = fmaxf(mx[c], mx[c + w]);
          // every row sees column 0 of its first chunk, so m_new is finite from there on
          const float m_new = fmaxf(m_run, mx[0] * P.scale_log2);
          l_run *= ex2(m_run - m_new);  // m_run = -inf before the first chunk: l_run stays 0
          float e[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) e[c] = ex2(fmaf(x[c], P.scale_log2, -m_new));  // -inf -> 0
          // tree sums: at level R the partial sums are the per-key-block sums (R | 32)
          const int jb = (kt * kAN + ch * 32) / R;  // key block of column 0 of the chunk
#pragma unroll
          for (int lv = 1; lv <= 32; lv <<= 1) {
            if (lv == R) {
#pragma unroll
              for (int c = 0; c < 32; c += lv) {
                const int j = jb + c / lv;  // the last tile may reach past block nb-1
                if (j < P.nb) __stcs(esc + static_cast<int64_t>(j) * kAM + row, e[c]);
              }
            }
            if (lv < 32) {
#pragma unroll
              for (int c = 0; c < 32; c += 2 * lv) e[c] += e[c + lv];
            }
          }
          l_run += e[0];
          __stcs(msc + (kt * (kAN / 32) + ch) * kAM + row, m_new);
          m_run = m_new;
        }
        tc_fence_before();
        mbar_arrive(&bars->acc_empty[buf]);
        ++tiles;
      }
      if (!ok) break;
      bars->ml[slot][0][row] = m_run;
      bars->ml[slot][1][row] = l_run;
      mbar_arrive(&bars->unit_done[slot]);  // releases the slot's scratch and m, l
    }
  } else {
    // ------------------------------------------------------------ fixup (warps 6-9)
    // The unit's block probabilities from its scratch slot, while the other warps work on the
    // next unit: each value is rescaled to its row's final m and divided by l, the block's
    // query groups are summed with shuffles and p_ij is written.
    const int fw = warp - 6;
    const int row = fw * 32 + lane;
    const int R = P.R;
    const int64_t tri = static_cast<int64_t>(P.nb) * (P.nb + 1) / 2;
    int64_t n = 0;
    for (;; ++n) {
      int64_t t;
      if (!__all_sync(0xffffffffu, ad_next_unit(bars, n, P.status, &t)) || t < 0) break;
      const AUnit un = ad_unit(t, P);
      const int slot = static_cast<int>(n & 1);
      if (!__all_sync(0xffffffffu, ad_wait(&bars->unit_done[slot],
                                           static_cast<uint32_t>((n >> 1) & 1), bars,
                                           P.status)))
        break;
      const float* esc =
          P.scratch + (2 * static_cast<int64_t>(blockIdx.x) + slot) * P.scratch_per_slot;
      const float* msc = esc + static_cast<int64_t>(P.nb) * kAM;
      const float m_run = bars->ml[slot][0][row], l_run = bars->ml[slot][1][row];
      const int u = un.qt * kAM + row;
      const bool valid = u < P.nred;
      const int i = u / R;                         // query block of this group
      const int n_i = min(R, P.nred - i * R);      // its query groups
      const float inv_l = 1.f / l_run;
      const int i_hi = min(P.nb - 1, (un.qt * kAM + fw * 32 + 31) / R);  // warp's last block
      float* prow = P.p + static_cast<int64_t>(un.bh) * tri + static_cast<int64_t>(i) * (i + 1) / 2;
      const float inv_n = 1.f / static_cast<float>(n_i);
      // eight key blocks per step, their loads issued together; every j <= i_hi lies in a tile
      // this unit processed, so the scratch entries read here are this unit's
      for (int j0 = 0; j0 <= i_hi; j0 += 8) {
        float ev[8], sv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = min(j0 + q, i_hi);
          ev[q] = __ldcs(esc + static_cast<int64_t>(j) * kAM + row);
          sv[q] = __ldcs(msc + ((j * R) >> 5) * kAM + row);  // snapshot of block j's chunk
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = j0 + q;
          float val = valid && j <= i ? ev[q] * ex2(sv[q] - m_run) * inv_l : 0.f;
          for (int o = 1; o < R; o <<= 1) val += __shfl_xor_sync(0xffffffffu, val, o);
          if (valid && j <= i && (lane & (R - 1)) == 0) __stcs(prow + j, val * inv_n);
        }
      }
      mbar_arrive(&bars->fix_done[slot]);  // the slot may be overwritten
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

// 3-D view [heads, S/stride, stride*D] of a bf16 [heads, S, D] tensor: one row per group of
// stride tokens. Boxes of 64 columns x `rows` groups x 1 head, 128B swizzle; groups past the
// last read 0.
bool make_group_map(CUtensorMap* m, const void* base, uint64_t heads, int S, int D, int stride,
                    int rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(stride) * D, static_cast<cuuint64_t>(S / stride),
                        heads};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(stride) * D * 2,
                           static_cast<cuuint64_t>(S) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int64_t antidiag_units(int B, int Hq, int S, int stride) {
  const int64_t nred = S / stride;
  return static_cast<int64_t>(B) * Hq * ((nred + kAM - 1) / kAM);
}

size_t antidiag_scratch_floats(int B, int Hq, int S, int block, int stride) {
  const int64_t nb = (S + block - 1) / block;
  const int64_t nred = S / stride;
  const int64_t nkt = (nred + kAN - 1) / kAN;
  const int64_t slots = std::min<int64_t>(antidiag_units(B, Hq, S, stride), kAdSlots);
  // the work counter (64 floats, keeping the rest 256-byte aligned), then two slots per CTA
  return static_cast<size_t>(64 + slots * 2 * (nb + (kAN / 32) * nkt) * kAM);
}

cudaError_t launch_antidiag(const void* q, const void* k, int B, int Hq, int Hkv, int S, int D,
                            int block, int stride, float* p, float* scratch, int32_t* status,
                            cudaStream_t st) {
  if (B * Hq == 0 || S == 0) return cudaSuccess;
  if ((D != 64 && D != 128) || stride < 1 || block % stride || S % stride ||
      block / stride > 32 || ((block / stride) & (block / stride - 1)))
    return cudaErrorInvalidValue;
  AdParams P;
  P.Hq = Hq;
  P.Hkv = Hkv;
  P.nb = (S + block - 1) / block;
  P.R = block / stride;
  P.nred = S / stride;
  P.nqt = (P.nred + kAM - 1) / kAM;
  P.kparts = D / 64;
  P.ksteps = stride * P.kparts;
  P.stride = stride;
  P.D = D;
  P.units = antidiag_units(B, Hq, S, stride);
  P.scale_log2 = static_cast<float>(1.4426950408889634 / (stride * std::sqrt(static_cast<double>(D))));
  P.p = p;
  P.next_unit = reinterpret_cast<unsigned long long*>(scratch);
  P.scratch = scratch + 64;
  P.scratch_per_slot = static_cast<int64_t>(P.nb + (kAN / 32) * ((P.nred + kAN - 1) / kAN)) * kAM;
  P.status = status;
  P.withhold = g_withhold_q.load();
  CUtensorMap tq, tk;
  if (!make_group_map(&tq, q, static_cast<uint64_t>(B) * Hq, S, D, stride, kAM) ||
      !make_group_map(&tk, k, static_cast<uint64_t>(B) * Hkv, S, D, stride, kAN))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + kStages * kStageBytes + sizeof(ABars);
  cudaError_t e = cudaFuncSetAttribute(antidiag_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>({P.units, static_cast<int64_t>(sm_count()),
                                          static_cast<int64_t>(kAdSlots)});
  e = cudaMemsetAsync(P.next_unit, 0, sizeof(unsigned long long), st);
  if (e != cudaSuccess) return e;
  antidiag_sm100_kernel<<<static_cast<unsigned>(grid), kAThreads, smem, st>>>(tq, tk, P);
  return cudaGetLastError();
}

}  // namespace stem
