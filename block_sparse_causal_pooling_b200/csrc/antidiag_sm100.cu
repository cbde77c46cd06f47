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
// antidiag_rowstat_kernel, one thread per (b, h, query group u): combines the parts' m and l of
// the group into the row's final max M and sum L. antidiag_merge_kernel, one thread per p_ij:
// rescales the R block sums of block i's query groups to their M, divides by L, adds them and
// writes p_ij; a bandwidth-bound pass over the partials.
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
  float* pm;            // [B*Hq][nqt][maxparts][128] each part's max m; after the row
                        // statistics, part 0's entry holds the query group's final max M
  float* pl;            // the same for its sum l; part 0's entry then holds 1/L
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

// Per query group u of head bh: the parts' maxima and sums combine into the row's
// M_u = max m and L_u = sum l * 2^(m - M_u), written over part 0's entries as M_u and 1/L_u.
// One thread per (bh, u); consecutive threads take consecutive u (coalesced).
__global__ void __launch_bounds__(256) antidiag_rowstat_kernel(AdParams P, int64_t rows) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (t >= rows) return;
  const int64_t bh = t / P.nred;
  const int u = static_cast<int>(t - bh * P.nred);
  const int qt = u / kAM;
  const int np = ad_nparts(qt, P.nred);
  const int64_t mb = (bh * P.nqt + qt) * P.maxparts * kAM + (u - qt * kAM);
  float M = -INFINITY;
  for (int q = 0; q < np; ++q) M = fmaxf(M, P.pm[mb + q * kAM]);
  float L = 0.f;
  for (int q = 0; q < np; ++q) L += P.pl[mb + q * kAM] * ex2(P.pm[mb + q * kAM] - M);
  P.pm[mb] = M;
  P.pl[mb] = 1.0f / L;
}

// p_ij from the partials: p_ij = (1/n_i) sum_u e_uj * 2^(snap_u,c(j) - M_u) / L_u over the n_i
// query groups u of block i, with c(j) the 32-group chunk that holds block j. One thread per
// entry of a head's p triangle (entry g = i(i+1)/2 + j), so consecutive threads read
// consecutive runs of R partials (e holds entry g's R partials at R*g) and write consecutive p;
// the row's M_u and 1/L_u and the chunk's snapshots are R consecutive floats each, shared by
// the threads of a row or a chunk (served by L1). The grid strides over the heads' chunks of
// 256 entries.
template <int kR>
__global__ void __launch_bounds__(256) antidiag_merge_kernel(AdParams P, int64_t tri,
                                                             int64_t ctas_per_head,
                                                             int64_t chunks) {
  for (int64_t blk = blockIdx.x; blk < chunks; blk += gridDim.x) {
    const int64_t bh = blk / ctas_per_head;
    const int64_t g = (blk - bh * ctas_per_head) * 256 + threadIdx.x;
    if (g >= tri) continue;
    // i, j of entry g: the float root may be off by one either way; the integer tests fix it
    int i = static_cast<int>((sqrtf(8.0f * static_cast<float>(g) + 1.0f) - 1.0f) * 0.5f);
    while (static_cast<int64_t>(i) * (i + 1) / 2 > g) --i;
    while (static_cast<int64_t>(i + 1) * (i + 2) / 2 <= g) ++i;
    const int j = static_cast<int>(g - static_cast<int64_t>(i) * (i + 1) / 2);
    const int u0 = i * kR;
    const int n_i = min(kR, P.nred - u0);
    const int qt = u0 / kAM;  // a block's groups lie in one 128-group tile (R | 128)
    const int c = (j * kR) >> 5;
    const float* ep = P.e + bh * P.tri_e + kR * g;
    const float* sp = P.snap + bh * P.tri_s + ad_tri(c, u0, P.nred, 32);
    const int64_t mb = (bh * P.nqt + qt) * P.maxparts * kAM + (u0 - qt * kAM);
    const float* mp = P.pm + mb;
    const float* lp = P.pl + mb;
    float acc = 0.f;
    if (kR >= 4 && n_i == kR && (reinterpret_cast<uintptr_t>(sp) & 15) == 0) {
      // whole block, every run 16-byte aligned (e, M and 1/L always are; the snapshot run is
      // unless S/stride is not a multiple of 4)
#pragma unroll
      for (int q = 0; q < (kR >= 4 ? kR / 4 : 1); ++q) {
        const float4 e4 = __ldcs(reinterpret_cast<const float4*>(ep) + q);
        const float4 s4 = __ldg(reinterpret_cast<const float4*>(sp) + q);
        const float4 m4 = __ldg(reinterpret_cast<const float4*>(mp) + q);
        const float4 l4 = __ldg(reinterpret_cast<const float4*>(lp) + q);
        acc += (e4.x * ex2(s4.x - m4.x) * l4.x + e4.y * ex2(s4.y - m4.y) * l4.y) +
               (e4.z * ex2(s4.z - m4.z) * l4.z + e4.w * ex2(s4.w - m4.w) * l4.w);
      }
    } else {
      for (int uu = 0; uu < n_i; ++uu)
        acc += __ldcs(ep + uu) * ex2(__ldg(sp + uu) - __ldg(mp + uu)) * __ldg(lp + uu);
    }
    P.p[bh * tri + g] = acc * (1.0f / static_cast<float>(n_i));
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
  const int64_t rows = static_cast<int64_t>(B) * Hq * P.nred;
  antidiag_rowstat_kernel<<<static_cast<unsigned>((rows + 255) / 256), 256, 0, st>>>(P, rows);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t tri = static_cast<int64_t>(P.nb) * (P.nb + 1) / 2;
  const int64_t per_head = (tri + 255) / 256;
  const int64_t chunks = static_cast<int64_t>(B) * Hq * per_head;
  const unsigned gm = static_cast<unsigned>(std::min<int64_t>(chunks, int64_t{1} << 20));
  switch (P.R) {
    case 1: antidiag_merge_kernel<1><<<gm, 256, 0, st>>>(P, tri, per_head, chunks); break;
    case 2: antidiag_merge_kernel<2><<<gm, 256, 0, st>>>(P, tri, per_head, chunks); break;
    case 4: antidiag_merge_kernel<4><<<gm, 256, 0, st>>>(P, tri, per_head, chunks); break;
    case 8: antidiag_merge_kernel<8><<<gm, 256, 0, st>>>(P, tri, per_head, chunks); break;
    case 16: antidiag_merge_kernel<16><<<gm, 256, 0, st>>>(P, tri, per_head, chunks); break;
    default: antidiag_merge_kernel<32><<<gm, 256, 0, st>>>(P, tri, per_head, chunks); break;
  }
  return cudaGetLastError();
}

}  // namespace stem
