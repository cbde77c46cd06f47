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
// Persistent kernel, one CTA per SM, 6 warps, then a merge kernel. Work unit: (b, h, 128 consecutive query groups,
// a part of at most four of their key tiles), claimed from a global counter in kv-head-major
// order with the parts of one query tile next to each other, and handed to the other roles
// through a ring in shared memory. The parts of a query tile run on different CTAs at once, so
// the CTAs in flight share few Q' tiles and one kv head's K', which then stay in L2.
//   warp 0    TMA producer: for every key tile of the part (256 key groups each, up to the
//             tile's causal end) and every k-step (64 of the sigma*D columns), the Q' box
//             (128 x 64) and the K' box (256 x 64) into a 4-stage ring of 128B-swizzled
//             shared-memory tiles.
//   warp 1    allocates the 512 TMEM columns; lane 0 issues tcgen05.mma (M 128, N 256, K 16)
//             into one of two 256-column fp32 accumulators, so the epilogue of one key tile
//             overlaps the products of the next.
//   warps 2-5 tile epilogue, one query group (TMEM lane) per thread: online softmax over the
//             32-column chunks of each key tile in base 2 (running max m, running sum l), one
//             TMEM read per chunk; per key block the sum of exp2(a - m) over its key groups
//             goes to the partials in global memory, and each chunk's m (its snapshot) beside
//             it; at the part's end its m and l.
// antidiag_merge_kernel, one CTA per (b, h, query block i): combines the parts' m and l of each
// of the block's query groups into the row's final max M and sum L, rescales every block sum to
// M and divides by L, sums the block's query groups with shuffles and writes p_ij; a
// bandwidth-bound pass over the partials.
// Q' tiles load with evict_last (a part re-reads its Q' tile for each of its key tiles); the
// partials move with streaming stores.
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
constexpr int kAThreads = 192;        // 6 warps
constexpr int kEpiThreads = 128;      // warps 2-5
constexpr uint32_t kQBox = kAM * 128;  // 128 rows x 64 bf16
constexpr uint32_t kKBox = kAN * 128;  // 256 rows x 64 bf16
constexpr uint32_t kStageBytes = kQBox + kKBox;
constexpr uint32_t kTmemCols = 512;
constexpr int kUnitRing = 8;          // unit indices handed from the producer to the other roles
constexpr int kUnitReaders = 1 + kEpiThreads;  // MMA thread, warps 2-5
#ifndef STEM_AD_PART_TILES
#define STEM_AD_PART_TILES 4
#endif
constexpr int kPartTiles = STEM_AD_PART_TILES;  // key tiles per part
constexpr int kMaxQt = 4096;          // query tiles per head the unit table holds

struct __align__(8) ABars {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t uq_full[kUnitRing], uq_empty[kUnitRing];
  uint64_t drain;
  int64_t uq[kUnitRing];  // unit index, or -1: no more units
  uint32_t tmem_base;
  volatile int abort;
};

struct AdParams {
  int Hq, Hkv, nb, R;   // R = block / stride: groups per block (1 .. 32)
  int nred, nqt;        // groups per head, query tiles per head
  int ksteps, kparts;   // stride*D/64 k-steps; D/64 of them per token chunk
  int stride, D;
  int maxparts;         // parts of the largest query tile
  int64_t units;        // B * Hq * (parts over all query tiles of a head)
  int64_t per_head;     // units of one head
  float scale_log2;     // log2(e) / (stride * sqrt(D))
  float* p;             // [B*Hq][nb*(nb+1)/2]
  unsigned long long* next_unit;  // work counter, 0 at launch
  // Partials, one triangle per head. e: the per-block sums of exp2(a - snapshot), for query
  // block i and key block j <= i the R groups of block i next to each other, entry
  // (i, j, u - i*R) at R*i*(i+1)/2 + j*R + (u - i*R), so a query block's partials are one
  // range. snap: per query group u and 32-group chunk c <= u/32 the snapshot max,
  // chunk-major: entry (c, u) at c*nred - 32*c*(c-1)/2 + (u - 32*c).
  float* e;             // [B*Hq][tri_e]
  float* snap;          // [B*Hq][tri_s]
  float* pm;            // [B*Hq][nqt][maxparts][128] each part's max m
  float* pl;            // the same for its sum l
  int64_t tri_e, tri_s;
  int32_t* status;
  int withhold;         // test switch: the first stage's copies are never sent
};

// Key tiles (256 groups) of query tile qt: up to its last query group.
__host__ __device__ __forceinline__ int ad_nkt(int qt, int nred) {
  const int last = min(nred - 1, qt * 128 + 127);
  return last / 256 + 1;
}
__host__ __device__ __forceinline__ int ad_nparts(int qt, int nred) {
  return (ad_nkt(qt, nred) + kPartTiles - 1) / kPartTiles;
}
// Offset of entry (j, u) in a block-major lower triangle with rows of `step` groups per index.
__host__ __device__ __forceinline__ int64_t ad_tri(int64_t j, int64_t u, int64_t nred,
                                                   int64_t step) {
  return j * nred - step * j * (j - 1) / 2 + (u - j * step);
}

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

// Unit t -> (bh, qt, part). kv-head-major, so that the units in flight share one kv head's K'
// (which then stays in L2); inside a kv head the heaviest query tiles first (a tile's key range
// grows with qt), the G query heads of a tile next to each other and each head's parts next to
// each other, so the parts of a tile run at once and share its Q' in L2. CTAs take units from a
// global counter, so the order is the order of issue, not a fixed assignment. cum[k] counts the
// units of one query head in the k heaviest query tiles (a table in shared memory).
struct AUnit {
  int bh, qt, kvh, part, nparts, kt0, kt1;
};
__device__ __forceinline__ AUnit ad_unit(int64_t t, const AdParams& P, const int* cum) {
  const int G = P.Hq / P.Hkv;
  const int64_t per_kv = static_cast<int64_t>(G) * P.per_head;
  const int kvh = static_cast<int>(t / per_kv);  // b * Hkv + kv head
  const int r = static_cast<int>(t % per_kv);
  // the k-th heaviest tile holds units [G*cum[k], G*cum[k+1]) of the kv head
  int lo = 0, hi = P.nqt - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (G * cum[mid] <= r) lo = mid; else hi = mid - 1;
  }
  AUnit u;
  u.kvh = kvh;
  u.qt = P.nqt - 1 - lo;
  u.nparts = ad_nparts(u.qt, P.nred);
  const int rr = r - G * cum[lo];
  u.part = rr % u.nparts;
  u.bh = (kvh / P.Hkv) * P.Hq + (kvh % P.Hkv) * G + rr / u.nparts;
  u.kt0 = u.part * kPartTiles;
  u.kt1 = min(ad_nkt(u.qt, P.nred), u.kt0 + kPartTiles);
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
  int* cum = reinterpret_cast<int*>(bars + 1);  // [nqt + 1], see ad_unit
  int* part_sum = cum + kMaxQt + 1;             // [kAThreads] scan scratch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the unit table: parts of the k heaviest query tiles of one head, as a chunked scan
  {
    const int per = (P.nqt + kAThreads - 1) / kAThreads;
    const int k0 = min(P.nqt, static_cast<int>(threadIdx.x) * per), k1 = min(P.nqt, k0 + per);
    int sum = 0;
    for (int k = k0; k < k1; ++k) sum += ad_nparts(P.nqt - 1 - k, P.nred);
    part_sum[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
      int run = 0;
      for (int t = 0; t < kAThreads; ++t) {
        const int v = part_sum[t];
        part_sum[t] = run;
        run += v;
      }
      cum[P.nqt] = run;
    }
    __syncthreads();
    int run = part_sum[threadIdx.x];
    for (int k = k0; k < k1; ++k) {
      cum[k] = run;
      run += ad_nparts(P.nqt - 1 - k, P.nred);
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->acc_full[s], 1);
      mbar_init(&bars->acc_empty[s], kEpiThreads);
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
      // a part re-reads its Q' tile for each of its key tiles: keep it; K' tiles pass through
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
        const AUnit u = ad_unit(t, P, cum);
        const int kvh = u.kvh;
        for (int kt = u.kt0; kt < u.kt1 && ok; ++kt) {
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
        const AUnit u = ad_unit(t, P, cum);
        for (int kt = u.kt0; kt < u.kt1 && ok; ++kt) {
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
      const AUnit un = ad_unit(t, P, cum);
      const int u = un.qt * kAM + row;  // this thread's query group
      const bool urow = u < P.nred;     // a group of the head (the last tile may run past)
      const int iu = u / R;             // its query block
      float* eh = P.e + static_cast<int64_t>(un.bh) * P.tri_e;
      const int64_t ebase = static_cast<int64_t>(R) * iu * (iu + 1) / 2 + (u - iu * R);
      float* sh = P.snap + static_cast<int64_t>(un.bh) * P.tri_s;
      float m_run = -INFINITY, l_run = 0.f;
      for (int kt = un.kt0; kt < un.kt1; ++kt) {
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
          const int col0 = kt * kAN + ch * 32;  // key group of column 0 of the chunk
          const int lim = u - col0;             // columns c <= lim are visible (w <= u)
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
          // every row sees column 0 of its part's first chunk (a part starts at a multiple of
          // 256 groups, at or before the tile's first group), so m_new is finite from there on
          const float m_new = fmaxf(m_run, mx[0] * P.scale_log2);
          l_run *= ex2(m_run - m_new);  // m_run = -inf before the first chunk: l_run stays 0
          float e[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) e[c] = ex2(fmaf(x[c], P.scale_log2, -m_new));  // -inf -> 0
          // tree sums: at level R the partial sums are the per-key-block sums (R | 32)
          const int jb = col0 / R;  // key block of column 0 of the chunk
#pragma unroll
          for (int lv = 1; lv <= 32; lv <<= 1) {
            if (lv == R) {
#pragma unroll
              for (int c = 0; c < 32; c += lv) {
                const int j = jb + c / lv;  // blocks past the row's own are not stored
                if (urow && j <= iu) __stcs(eh + ebase + j * R, e[c]);
              }
            }
            if (lv < 32) {
#pragma unroll
              for (int c = 0; c < 32; c += 2 * lv) e[c] += e[c + lv];
            }
          }
          l_run += e[0];
          const int cc = col0 / 32;  // the chunk's index among the row's chunks
          if (urow && cc <= u / 32) __stcs(sh + ad_tri(cc, u, P.nred, 32), m_new);
          m_run = m_new;
        }
        tc_fence_before();
        mbar_arrive(&bars->acc_empty[buf]);
        ++tiles;
      }
      if (!ok) break;
      const int64_t mi = ((static_cast<int64_t>(un.bh) * P.nqt + un.qt) * P.maxparts + un.part) *
                             kAM + row;
      __stcs(P.pm + mi, m_run);
      __stcs(P.pl + mi, l_run);
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

// p_ij of query block i of head bh from the estimator's partials: per query group u of the
// block, the parts' maxima and sums combine into M_u = max m and L_u = sum l * 2^(m - M_u);
// p_ij = (1/n_i) sum_u e_uj * 2^(snap_u,c(j) - M_u) / L_u, with c(j) the 32-group chunk that
// holds block j. One CTA per (bh, i), 256 threads; a warp takes 32/R blocks j at a time, one
// lane per (j, u), and sums the block's query groups with shuffles.
__global__ void __launch_bounds__(256)
    antidiag_merge_kernel(AdParams P) {
  const int i = blockIdx.x % P.nb;
  const int bh = blockIdx.x / P.nb;
  const int R = P.R;
  const int u0 = i * R;
  const int n_i = min(R, P.nred - u0);
  const int qt = u0 / kAM;  // a block's groups lie in one 128-group tile (R | 128)
  const int np = ad_nparts(qt, P.nred);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = 32 / R;  // blocks j per warp step
  const int uu = lane % R, jj = lane / R;
  const bool urow = uu < n_i;
  const int u = u0 + (urow ? uu : 0);
  const float* eh = P.e + static_cast<int64_t>(bh) * P.tri_e + static_cast<int64_t>(R) * i * (i + 1) / 2;
  const float* sh = P.snap + static_cast<int64_t>(bh) * P.tri_s;
  float* prow = P.p + static_cast<int64_t>(bh) * P.nb * (P.nb + 1) / 2 +
                static_cast<int64_t>(i) * (i + 1) / 2;
  const float inv_n = 1.f / static_cast<float>(n_i);
  // every lane loads its row's part maxima and sums together with its first partials (the
  // partials are read-only here: written by the estimator kernel before this one)
  const int64_t mb = (static_cast<int64_t>(bh) * P.nqt + qt) * P.maxparts * kAM + (u - qt * kAM);
  float pmv[8], plv[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    pmv[q] = q < np ? __ldg(P.pm + mb + q * kAM) : -INFINITY;
    plv[q] = q < np ? __ldg(P.pl + mb + q * kAM) : 0.f;
  }
  for (int q = 8; q < np; ++q) {  // more than eight parts: S/stride above 8192 * 8 groups
    const float mq = __ldg(P.pm + mb + q * kAM), lq = __ldg(P.pl + mb + q * kAM);
    const float mn = fmaxf(pmv[7], mq);
    plv[7] = plv[7] * ex2(pmv[7] - mn) + lq * ex2(mq - mn);
    pmv[7] = mn;
  }
  constexpr int kUn = 4;
  float ev[kUn], sv[kUn];
  auto load = [&](int jb) {
#pragma unroll
    for (int q = 0; q < kUn; ++q) {
      const int j = jb + q * 8 * per + jj;
      const bool in = j <= i && urow;
      ev[q] = in ? __ldg(eh + j * R + uu) : 0.f;  // the block's partials: one range
      sv[q] = in ? __ldg(sh + ad_tri((j * R) >> 5, u, P.nred, 32)) : 0.f;
    }
  };
  int jb = warp * per;
  if (jb <= i) load(jb);
  float M = pmv[0];
#pragma unroll
  for (int q = 1; q < 8; ++q) M = fmaxf(M, pmv[q]);
  float L = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q) L += plv[q] * ex2(pmv[q] - M);
  const float inv_l = 1.f / L;
  for (; jb <= i; jb += 8 * per * kUn) {
    float val[kUn];
#pragma unroll
    for (int q = 0; q < kUn; ++q) val[q] = ev[q] * ex2(sv[q] - M) * inv_l;
    if (jb + 8 * per * kUn <= i) load(jb + 8 * per * kUn);  // the next step's loads in flight
#pragma unroll
    for (int q = 0; q < kUn; ++q) {
      const int j = jb + q * 8 * per + jj;
      float v = val[q];
      for (int o = 1; o < R; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (j <= i && uu == 0) __stcs(prow + j, v * inv_n);
    }
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

namespace {

// Regions of the estimator's scratch (in floats, each 256-byte aligned): the work counter, the
// partials e and snap, and each part's m and l.
struct AdLayout {
  int64_t nb, nred, R, nqt, maxparts, tri_e, tri_s;
  int64_t e, snap, pm, pl, total;
};
int64_t align64(int64_t x) { return (x + 63) / 64 * 64; }
AdLayout ad_layout(int B, int Hq, int S, int block, int stride) {
  AdLayout L;
  L.nb = (S + block - 1) / block;
  L.nred = S / stride;
  L.R = block / stride;
  L.nqt = (L.nred + kAM - 1) / kAM;
  L.maxparts = L.nqt > 0 ? ad_nparts(static_cast<int>(L.nqt - 1), static_cast<int>(L.nred)) : 0;
  L.tri_e = L.R * L.nb * (L.nb + 1) / 2;
  const int64_t nch = (L.nred + 31) / 32;
  L.tri_s = nch * L.nred - 32 * nch * (nch - 1) / 2;
  const int64_t heads = static_cast<int64_t>(B) * Hq;
  int64_t o = 64;  // the work counter
  L.e = o;
  o += align64(heads * L.tri_e);
  L.snap = o;
  o += align64(heads * L.tri_s);
  L.pm = o;
  o += align64(heads * L.nqt * L.maxparts * kAM);
  L.pl = o;
  o += align64(heads * L.nqt * L.maxparts * kAM);
  L.total = o;
  return L;
}

}  // namespace

int64_t antidiag_units(int B, int Hq, int S, int stride) {
  const int nred = S / stride;
  const int nqt = (nred + kAM - 1) / kAM;
  int64_t per_head = 0;
  for (int qt = 0; qt < nqt; ++qt) per_head += ad_nparts(qt, nred);
  return static_cast<int64_t>(B) * Hq * per_head;
}

size_t antidiag_scratch_floats(int B, int Hq, int S, int block, int stride) {
  return static_cast<size_t>(ad_layout(B, Hq, S, block, stride).total);
}

cudaError_t launch_antidiag(const void* q, const void* k, int B, int Hq, int Hkv, int S, int D,
                            int block, int stride, float* p, float* scratch, int32_t* status,
                            cudaStream_t st) {
  if (B * Hq == 0 || S == 0) return cudaSuccess;
  if ((D != 64 && D != 128) || stride < 1 || block % stride || S % stride ||
      block / stride > 32 || ((block / stride) & (block / stride - 1)))
    return cudaErrorInvalidValue;
  const AdLayout L = ad_layout(B, Hq, S, block, stride);
  if (L.nqt > kMaxQt) return cudaErrorInvalidValue;
  AdParams P;
  P.Hq = Hq;
  P.Hkv = Hkv;
  P.nb = static_cast<int>(L.nb);
  P.R = static_cast<int>(L.R);
  P.nred = static_cast<int>(L.nred);
  P.nqt = static_cast<int>(L.nqt);
  P.kparts = D / 64;
  P.ksteps = stride * P.kparts;
  P.stride = stride;
  P.D = D;
  P.maxparts = static_cast<int>(L.maxparts);
  P.units = antidiag_units(B, Hq, S, stride);
  P.per_head = P.units / (static_cast<int64_t>(B) * Hq);
  P.scale_log2 = static_cast<float>(1.4426950408889634 / (stride * std::sqrt(static_cast<double>(D))));
  P.p = p;
  P.next_unit = reinterpret_cast<unsigned long long*>(scratch);
  P.e = scratch + L.e;
  P.snap = scratch + L.snap;
  P.pm = scratch + L.pm;
  P.pl = scratch + L.pl;
  P.tri_e = L.tri_e;
  P.tri_s = L.tri_s;
  P.status = status;
  P.withhold = g_withhold_q.load();
  CUtensorMap tq, tk;
  if (!make_group_map(&tq, q, static_cast<uint64_t>(B) * Hq, S, D, stride, kAM) ||
      !make_group_map(&tk, k, static_cast<uint64_t>(B) * Hkv, S, D, stride, kAN))
    return cudaErrorInvalidValue;
  const size_t smem =
      1024 + kStages * kStageBytes + sizeof(ABars) + sizeof(int) * (kMaxQt + 1 + kAThreads);
  cudaError_t e = cudaFuncSetAttribute(antidiag_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>({P.units, static_cast<int64_t>(sm_count()),
                                          static_cast<int64_t>(kAdSlots)});
  e = cudaMemsetAsync(P.next_unit, 0, sizeof(unsigned long long), st);
  if (e != cudaSuccess) return e;
  antidiag_sm100_kernel<<<static_cast<unsigned>(grid), kAThreads, smem, st>>>(tq, tk, P);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  antidiag_merge_kernel<<<static_cast<unsigned>(static_cast<int64_t>(B) * Hq * P.nb), 256, 0,
                          st>>>(P);
  return cudaGetLastError();
}

}  // namespace stem
