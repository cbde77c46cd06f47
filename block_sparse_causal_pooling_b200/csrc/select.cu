// Output-Aware Metric and variable-k top-k block selection, fused in one kernel.
//
// Method ("Stem: Rethinking Causal Information Flow in Sparse Attention"): rank the key blocks
// of each query block by routing probability times value magnitude (gist.science/es "Resumen
// tecnico" 2.B; gist.science/it 2.B; gist.science/nl OAM; gist.science/fr 2.B), keep the
// position-dependent number k(i) of them (es 2.A, it 2.A, nl TPD, fr 2.A), always including
// the initial (sink) block (es 1, shd-paper.top English abstract) and the diagonal block.
// On pooled blocks:
//   s_ij = qbar_i . kbar_j / sqrt(D),  m_ij = softmax_{j<=i}(s_ij) * n_j.
// Within row i, log m_ij = s_ij + ln n_j - logsumexp_j(s_ij), so ranking by
//   key_ij = s_ij + ln n_j
// ranks exactly like m_ij; the kernel ranks by key_ij in double (s_ij from a float32 dot
// product, ln n_j in double) and never materialises m unless asked for it.
//
// The pages' additive form (es 2.B, it 2.B, nl OAM, fr 2.B) ranks by
//   key_ij = s_ij + beta * e_j,   e_j = log(n_j^2) = 2 ln n_j, clamped at 0 (max(0, .)) on request,
// the same machinery with another per-column term (e_j is not evaluated when beta = 0).
//
// Kept set of row i: {0, i} plus the k(i)-2 largest key_ij over j in [1, i-1], larger first,
// equal keys to the lower j. Written ascending into the CSR slot of row (b, h, i).
//
// Two designs compute the same selection from the same scores:
//   split (the path's default, given scratch): score_tri_kernel writes s for the lower triangle
//     of a chunk of heads into scratch (a tiled float32 SIMT product, 64 x 64 tiles, 4 x 4
//     scores per thread), then select_s_kernel selects each row with one warp per row at high
//     occupancy; the chunk's triangle (tens of MB) stays in L2 between the two;
//   fused (no scratch; the allocation-free entry point): select_kernel, one CTA (8 warps) per
//     (b, h, R consecutive query blocks): phase 1 computes s for its R rows into shared memory,
//     phase 2 selects each row with one warp.
// Every score is the same float32 multiply-add chain over d ascending in both, so both designs
// select identically. The selection of a row: an exact radix select on the 64-bit
// order-preserving image of key_ij (8-bit digits, starting at the highest bit where the row's
// keys differ), then an ascending ballot compaction that takes the threshold ties lowest-j first.
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>

#include "stem_internal.h"

namespace stem {
namespace {

constexpr int kSelThreads = 256;
constexpr int kWarps = kSelThreads / 32;
constexpr int kTileJ = 64;

__device__ __forceinline__ uint64_t order_bits(double x) {
  // order-preserving map from double to uint64 (no NaNs expected)
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x + 0.0));  // -0 -> +0
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// The digit (0-255, taken from the largest) at which a count of `rem` keys is reached in a
// warp's 256-bin histogram, the number of keys in larger digits, and the digit's own count.
struct DigitPick {
  int digit, above, dcount;
};
__device__ __forceinline__ DigitPick pick_digit(const int* hist, int lane, int rem) {
  // lane l owns bins 255-8l .. 248-8l (descending)
  int cnt[8];
  int local = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    cnt[e] = hist[255 - 8 * lane - e];
    local += cnt[e];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int excl = incl - local;
  const bool owner = excl < rem && rem <= incl;
  int digit = 0, above = 0, dcount = 0;
  if (owner) {
    int run = excl;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (run + cnt[e] >= rem) {
        digit = 255 - 8 * lane - e;
        above = run;
        dcount = cnt[e];
        break;
      }
      run += cnt[e];
    }
  }
  const int src = __ffs(__ballot_sync(0xffffffffu, owner)) - 1;
  DigitPick r;
  r.digit = __shfl_sync(0xffffffffu, digit, src);
  r.above = __shfl_sync(0xffffffffu, above, src);
  r.dcount = __shfl_sync(0xffffffffu, dcount, src);
  __syncwarp();
  return r;
}

// Kept set of row i: {0, i} plus the k(i)-2 largest keys over j in [1, i-1] (equal keys: lower
// j first), written ascending to dst + t*dstride for t < ndst (the same list at every
// destination). One warp; key_bits(j) is the order-preserving image of column j's key; hist is
// the warp's 256-bin histogram.
template <typename KeyBits>
__device__ __forceinline__ void select_row(int i, int kk, KeyBits key_bits, int* hist, int lane,
                                           int32_t* dst, int64_t dstride, int ndst) {
  const unsigned lt_mask = (1u << lane) - 1u;
  if (i == 0) {
    if (lane == 0)
      for (int t = 0; t < ndst; ++t) dst[t * dstride] = 0;
    return;
  }
  const int need = kk - 2;  // picks among j in [1, i-1]
  if (need >= i - 1) {      // every causal block
    for (int j = lane; j <= i; j += 32)
      for (int t = 0; t < ndst; ++t) dst[t * dstride + j] = j;
    return;
  }
  if (need <= 0) {
    if (lane == 0)
      for (int t = 0; t < ndst; ++t) {
        dst[t * dstride] = 0;
        dst[t * dstride + 1] = i;
      }
    return;
  }
  // the highest bit where this row's candidate keys differ
  uint64_t umin = ~0ull, umax = 0ull;
  for (int j = 1 + lane; j < i; j += 32) {
    const uint64_t u = key_bits(j);
    umin = u < umin ? u : umin;
    umax = u > umax ? u : umax;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const uint64_t a = __shfl_xor_sync(0xffffffffu, umin, o);
    const uint64_t c = __shfl_xor_sync(0xffffffffu, umax, o);
    umin = a < umin ? a : umin;
    umax = c > umax ? c : umax;
  }
  uint64_t prefix, pmask;
  int rem = need;
  bool exact = false;
  if (umin == umax) {  // all candidates tie: lowest indices
    prefix = umin;
    pmask = ~0ull;
  } else {
    const int top = 63 - __clzll(static_cast<long long>(umin ^ umax));  // highest differing bit
    pmask = top >= 63 ? 0ull : (~0ull << (top + 1));
    prefix = umin & pmask;
    int shift = top - 7 < 0 ? 0 : top - 7;
    while (true) {
      for (int bin = lane; bin < 256; bin += 32) hist[bin] = 0;
      __syncwarp();
      for (int j = 1 + lane; j < i; j += 32) {
        const uint64_t u = key_bits(j);
        if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 0xff], 1);
      }
      __syncwarp();
      const DigitPick dp = pick_digit(hist, lane, rem);
      const int digit = dp.digit, above = dp.above, dcount = dp.dcount;
      rem -= above;
      prefix = (prefix & ~(0xffull << shift)) | (static_cast<uint64_t>(digit) << shift);
      pmask |= 0xffull << shift;
      if (dcount == rem) {
        exact = true;
        break;
      }
      if (shift == 0) break;
      shift = shift - 8 < 0 ? 0 : shift - 8;
    }
  }
  // ascending emission; threshold ties (full key equal) lowest-j first
  int written = 0, ties = 0;
  for (int j0 = 0; j0 <= i; j0 += 32) {
    const int j = j0 + lane;
    bool sel = false, tie = false;
    if (j <= i) {
      if (j == 0 || j == i) {
        sel = true;
      } else {
        const uint64_t um = key_bits(j) & pmask;
        if (um > prefix) {
          sel = true;
        } else if (um == prefix) {
          if (exact) sel = true;
          else tie = true;
        }
      }
    }
    const unsigned tb = __ballot_sync(0xffffffffu, tie);
    if (tie && ties + __popc(tb & lt_mask) < rem) sel = true;
    ties += __popc(tb);
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    const int pos = written + __popc(sb & lt_mask);
    if (sel && pos < kk)  // never past this row's slot
      for (int t = 0; t < ndst; ++t) dst[t * dstride + pos] = j;
    written += __popc(sb);
  }
}

struct SelSmem {
  float* s;       // [R][ldS] scaled logits
  float* qs;      // [R][D]
  float* ks;      // [kTileJ][D+4]
  double* lnn;    // [ldS] per-column term of the key: ln n_j, or beta * e_j (additive)
  int* hist;      // [kWarps][256]
};

template <int D, int R>
__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar,
    const float* __restrict__ vnorm, int BH, int Hq, int Hkv, int nb, int ldS, PlanDev plan,
    int64_t cap, SelMetric metric, int32_t* __restrict__ sel_idx, int32_t* __restrict__ sel_cnt,
    float* __restrict__ m_out) {
  constexpr int RPW = R / kWarps;  // rows per warp in phase 1
  constexpr int KLD = D + 4;       // padded kbar row (conflict-free 16-byte column reads)
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelSmem sm;
  sm.s = reinterpret_cast<float*>(smem_raw);
  sm.qs = sm.s + R * ldS;
  sm.ks = sm.qs + R * D;
  sm.lnn = reinterpret_cast<double*>(sm.ks + kTileJ * KLD);
  sm.hist = reinterpret_cast<int*>(sm.lnn + ldS);

  const int ntiles = (nb + R - 1) / R;
  const int tile = ntiles - 1 - static_cast<int>(blockIdx.x / BH);  // heaviest tiles first
  const int bh = static_cast<int>(blockIdx.x % BH);
  const int b = bh / Hq, h = bh % Hq;
  const int G = Hq / Hkv;
  const int64_t bg = static_cast<int64_t>(b) * Hkv + h / G;
  const int i0 = tile * R;
  const int rows = min(R, nb - i0);
  const int jend = i0 + rows;  // columns 0 .. jend-1
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;

  const float* qsrc = qbar + (static_cast<int64_t>(bh) * nb + i0) * D;
  const float* ksrc = kbar + bg * nb * D;
  const float* nsrc = vnorm + bg * nb;

  for (int idx = t; idx < R * D / 4; idx += kSelThreads) {
    const int r = idx / (D / 4), c4 = idx % (D / 4);
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rows) val = reinterpret_cast<const float4*>(qsrc + r * D)[c4];
    reinterpret_cast<float4*>(sm.qs + r * D)[c4] = val;
  }
  for (int j = t; j < jend; j += kSelThreads) {
    double c;
    if (!metric.additive) {
      c = log(static_cast<double>(nsrc[j]));
    } else if (metric.beta == 0.f) {
      c = 0.0;
    } else {
      double e = 2.0 * log(static_cast<double>(nsrc[j]));
      if (metric.clamp && e < 0.0) e = 0.0;
      c = static_cast<double>(metric.beta) * e;
    }
    sm.lnn[j] = c;
  }

  const float scale = rsqrtf(static_cast<float>(D));
  // ---- phase 1: s[r][j] for r < rows, j < jend
  for (int j0 = 0; j0 < jend; j0 += kTileJ) {
    __syncthreads();  // previous tile consumed (and qs / lnn visible on the first pass)
    for (int idx = t; idx < kTileJ * D / 4; idx += kSelThreads) {
      const int r = idx / (D / 4), c4 = idx % (D / 4);
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + r < jend) val = reinterpret_cast<const float4*>(ksrc + (j0 + r) * D)[c4];
      *reinterpret_cast<float4*>(sm.ks + r * KLD + c4 * 4) = val;
    }
    __syncthreads();
    float acc[RPW][2];
#pragma unroll
    for (int a = 0; a < RPW; ++a) acc[a][0] = acc[a][1] = 0.f;
    const float* k0 = sm.ks + lane * KLD;
    const float* k1 = sm.ks + (lane + 32) * KLD;
#pragma unroll 4
    for (int d = 0; d < D; d += 4) {
      const float4 x0 = *reinterpret_cast<const float4*>(k0 + d);
      const float4 x1 = *reinterpret_cast<const float4*>(k1 + d);
#pragma unroll
      for (int a = 0; a < RPW; ++a) {
        const float4 qv = *reinterpret_cast<const float4*>(sm.qs + (warp * RPW + a) * D + d);
        acc[a][0] = fmaf(qv.x, x0.x, acc[a][0]);
        acc[a][0] = fmaf(qv.y, x0.y, acc[a][0]);
        acc[a][0] = fmaf(qv.z, x0.z, acc[a][0]);
        acc[a][0] = fmaf(qv.w, x0.w, acc[a][0]);
        acc[a][1] = fmaf(qv.x, x1.x, acc[a][1]);
        acc[a][1] = fmaf(qv.y, x1.y, acc[a][1]);
        acc[a][1] = fmaf(qv.z, x1.z, acc[a][1]);
        acc[a][1] = fmaf(qv.w, x1.w, acc[a][1]);
      }
    }
#pragma unroll
    for (int a = 0; a < RPW; ++a) {
      const int r = warp * RPW + a;
      if (j0 + lane < jend) sm.s[r * ldS + j0 + lane] = acc[a][0] * scale;
      if (j0 + lane + 32 < jend) sm.s[r * ldS + j0 + lane + 32] = acc[a][1] * scale;
    }
  }
  __syncthreads();

  // ---- phase 2: one warp per row
  int* hist = sm.hist + warp * 256;
  for (int r = warp; r < rows; r += kWarps) {
    const int i = i0 + r;
    const float* srow = sm.s + r * ldS;
    const int kk = plan.k[i];
    int32_t* dst = sel_idx + static_cast<int64_t>(bh) * cap + plan.off[i];
    if (lane == 0) sel_cnt[static_cast<int64_t>(bh) * nb + i] = kk;

    if (m_out != nullptr && metric.additive) {  // diagnostic metric row: M_ij = s_ij + beta e_j
      float* mrow = m_out + static_cast<int64_t>(bh) * (static_cast<int64_t>(nb) * (nb + 1) / 2) +
                    static_cast<int64_t>(i) * (i + 1) / 2;
      for (int j = lane; j <= i; j += 32)
        mrow[j] = static_cast<float>(static_cast<double>(srow[j]) + sm.lnn[j]);
    } else if (m_out != nullptr) {  // diagnostic metric row, float32 softmax
      float mx = -INFINITY;
      for (int j = lane; j <= i; j += 32) mx = fmaxf(mx, srow[j]);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float z = 0.f;
      for (int j = lane; j <= i; j += 32) z += expf(srow[j] - mx);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      float* mrow = m_out + static_cast<int64_t>(bh) * (static_cast<int64_t>(nb) * (nb + 1) / 2) +
                    static_cast<int64_t>(i) * (i + 1) / 2;
      for (int j = lane; j <= i; j += 32) mrow[j] = expf(srow[j] - mx) / z * nsrc[j];
    }

    auto key_bits = [&](int j) -> uint64_t {
      return order_bits(static_cast<double>(srow[j]) + sm.lnn[j]);
    };
    select_row(i, kk, key_bits, hist, lane, dst, 0, 1);
  }
}

// 16-byte copy from global to shared memory; with full = false the destination is filled with 0
// (nothing is read from src).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool full) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(full ? 16 : 0)
               : "memory");
}

// ---- split design, step 1: pooled scores s_ij = qbar_i . kbar_j / sqrt(D) for j <= i of heads
// [h0, h0 + nh) of the B*Hq, into tri[(head - h0) * nb(nb+1)/2 + i(i+1)/2 + j]. One CTA per 64 x 64
// tile of (i, j) with the j tile at most the i tile; each thread holds the 4 x 4 scores of rows
// ty + 16a and columns tx + 16b (a, b < 4) of the tile, both tiles' pooled rows staged in shared
// memory (row stride D + 4 floats: the 16 columns a warp reads at one d fall in distinct banks).
constexpr int kScT = 64;

template <int D>
__global__ void __launch_bounds__(kSelThreads) score_tri_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, int Hq, int Hkv, int nb,
    int h0, int tiles_per_head, float* __restrict__ tri) {
  constexpr int LD = D + 4;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qs = reinterpret_cast<float*>(smem_raw);
  float* ks = qs + kScT * LD;
  const int hl = static_cast<int>(blockIdx.x) / tiles_per_head;
  const int t = static_cast<int>(blockIdx.x) % tiles_per_head;
  // t -> (ti, tj), tj <= ti, tiles of the lower triangle numbered row by row
  int ti = static_cast<int>((sqrtf(8.0f * static_cast<float>(t) + 1.0f) - 1.0f) * 0.5f);
  while (ti * (ti + 1) / 2 > t) --ti;
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  const int tj = t - ti * (ti + 1) / 2;
  const int64_t bh = static_cast<int64_t>(h0) + hl;
  const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
  const int G = Hq / Hkv;
  const float* qsrc = qbar + bh * nb * D;
  const float* ksrc = kbar + (static_cast<int64_t>(b) * Hkv + h / G) * nb * D;
  const int i0 = ti * kScT, j0 = tj * kScT;
  // Both tiles go straight from global to shared memory (cp.async, 16 bytes a copy; rows past
  // nb are filled with 0) in two halves of D, each its own group: the second half is in flight
  // while the first is multiplied.
  constexpr int kHalf = D / 2;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    for (int idx = threadIdx.x; idx < kScT * kHalf / 4; idx += kSelThreads) {
      const int r = idx / (kHalf / 4), c4 = hf * (kHalf / 4) + idx % (kHalf / 4);
      const bool qin = i0 + r < nb, kin = j0 + r < nb;
      cp_async16(qs + r * LD + 4 * c4, qsrc + static_cast<int64_t>(qin ? i0 + r : 0) * D + 4 * c4,
                 qin);
      cp_async16(ks + r * LD + 4 * c4, ksrc + static_cast<int64_t>(kin ? j0 + r : 0) * D + 4 * c4,
                 kin);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
  // d ascending, the same multiply-add chain per score as select_kernel
  auto madd = [&](int d) {
    float4 qv[4], kv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) qv[a] = *reinterpret_cast<const float4*>(qs + (ty + 16 * a) * LD + d);
#pragma unroll
    for (int c = 0; c < 4; ++c) kv[c] = *reinterpret_cast<const float4*>(ks + (tx + 16 * c) * LD + d);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[a][c] = fmaf(qv[a].x, kv[c].x, acc[a][c]);
        acc[a][c] = fmaf(qv[a].y, kv[c].y, acc[a][c]);
        acc[a][c] = fmaf(qv[a].z, kv[c].z, acc[a][c]);
        acc[a][c] = fmaf(qv[a].w, kv[c].w, acc[a][c]);
      }
  };
  asm volatile("cp.async.wait_group 1;" ::: "memory");  // first half landed (this thread's)
  __syncthreads();                                       // ... and every thread's
#pragma unroll 2
  for (int d = 0; d < kHalf; d += 4) madd(d);
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
#pragma unroll 2
  for (int d = kHalf; d < D; d += 4) madd(d);
  const float scale = rsqrtf(static_cast<float>(D));  // as in select_kernel
  float* dst = tri + static_cast<int64_t>(hl) * (static_cast<int64_t>(nb) * (nb + 1) / 2);
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
    if (i >= nb) continue;
    const int64_t rowoff = static_cast<int64_t>(i) * (i + 1) / 2;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + tx + 16 * c;
      if (j <= i) dst[rowoff + j] = acc[a][c] * scale;
    }
  }
}

// ---- split design, step 2: the selection of every row of heads [h0, h0 + nh) from their score
// rows in tri (written by score_tri_kernel). One CTA (8 warps) per (head, 8 consecutive query
// blocks), heaviest rows first, one row per warp; the per-column term of the key (ln n_j, or
// beta * e_j for the additive form) in shared memory. m_out as select_kernel writes it.
__global__ void __launch_bounds__(kSelThreads) select_s_kernel(
    const float* __restrict__ tri, const float* __restrict__ vnorm, int Hq, int Hkv, int nb,
    int h0, int nh, PlanDev plan, int64_t cap, SelMetric metric, int32_t* __restrict__ sel_idx,
    int32_t* __restrict__ sel_cnt, float* __restrict__ m_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int ldS = (nb + 3) & ~3;
  double* lnn = reinterpret_cast<double*>(smem_raw);                      // [ldS]
  int* hist_all = reinterpret_cast<int*>(lnn + ldS);                      // [kWarps][256]
  const int ntiles = (nb + kWarps - 1) / kWarps;
  const int tile = ntiles - 1 - static_cast<int>(blockIdx.x / nh);  // heaviest rows first
  const int sh = static_cast<int>(blockIdx.x % nh);
  const int64_t bh = static_cast<int64_t>(h0) + sh;
  const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
  const int G = Hq / Hkv;
  const int i0 = tile * kWarps;
  const int rows = min(kWarps, nb - i0);
  const int jend = i0 + rows;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const float* nsrc = vnorm + (static_cast<int64_t>(b) * Hkv + h / G) * nb;
  const int64_t trisz = static_cast<int64_t>(nb) * (nb + 1) / 2;
  for (int j = t; j < jend; j += kSelThreads) {
    double c;
    if (!metric.additive) {
      c = log(static_cast<double>(nsrc[j]));
    } else if (metric.beta == 0.f) {
      c = 0.0;
    } else {
      double e = 2.0 * log(static_cast<double>(nsrc[j]));
      if (metric.clamp && e < 0.0) e = 0.0;
      c = static_cast<double>(metric.beta) * e;
    }
    lnn[j] = c;
  }
  __syncthreads();
  if (warp >= rows) return;  // no __syncthreads below
  const int i = i0 + warp;
  const int kk = plan.k[i];
  const int64_t rowoff = static_cast<int64_t>(i) * (i + 1) / 2;
  const float* srow = tri + static_cast<int64_t>(sh) * trisz + rowoff;
  int* hist = hist_all + warp * 256;
  if (lane == 0) sel_cnt[bh * nb + i] = kk;
  if (m_out != nullptr && metric.additive) {  // diagnostic metric row: M_ij = s_ij + beta e_j
    for (int j = lane; j <= i; j += 32)
      m_out[bh * trisz + rowoff + j] = static_cast<float>(static_cast<double>(srow[j]) + lnn[j]);
  } else if (m_out != nullptr) {  // diagnostic metric row, float32 softmax
    float mx = -INFINITY;
    for (int j = lane; j <= i; j += 32) mx = fmaxf(mx, srow[j]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float z = 0.f;
    for (int j = lane; j <= i; j += 32) z += expf(srow[j] - mx);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    for (int j = lane; j <= i; j += 32)
      m_out[bh * trisz + rowoff + j] = expf(srow[j] - mx) / z * nsrc[j];
  }
  auto key_bits = [&](int j) -> uint64_t {
    return order_bits(static_cast<double>(__ldg(srow + j)) + lnn[j]);
  };
  select_row(i, kk, key_bits, hist, lane, sel_idx + bh * cap + plan.off[i], 0, 1);
}

// ---- GQA-group-shared selection: one kept list per (b, kv-head group, query block), chosen by
// the metric summed over the group's G query heads and written to each of them.
//   product:  sum_h m_hij = n_j * sum_h p_hij, ranked by ln n_j + logsumexp_h(s_hij - lse_hi),
//             lse_hi = logsumexp over j <= i of s_hij; the head terms are combined in double by
//             log-add-exp, so columns whose probabilities underflow float still rank;
//   additive: sum_h M_hij = sum_h s_hij + G * beta * e_j.
// One CTA (8 warps) per (b, g, 8 consecutive query blocks); the heads are visited in turn: the
// scores of one head's 8 rows are computed into shared memory, folded into a double key row per
// query block, and the next head reuses the space.
constexpr int kGR = 8;  // query blocks per CTA (one per warp)

template <int D>
__global__ void __launch_bounds__(kSelThreads) select_group_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar,
    const float* __restrict__ vnorm, int B, int Hq, int Hkv, int nb, int ldS, PlanDev plan,
    int64_t cap, SelMetric metric, int32_t* __restrict__ sel_idx, int32_t* __restrict__ sel_cnt,
    float* __restrict__ m_out) {
  constexpr int KLD = D + 4;
  static_assert(kGR == kWarps, "one query block per warp");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* acc = reinterpret_cast<double*>(smem_raw);  // [kGR][ldS] key under construction
  double* lnn = acc + kGR * ldS;                       // [ldS] per-column term
  float* srow_all = reinterpret_cast<float*>(lnn + ldS);  // [kGR][ldS] one head's scores
  float* qs = srow_all + kGR * ldS;                       // [kGR][D]
  float* ks = qs + kGR * D;                               // [kTileJ][KLD]
  int* hist_all = reinterpret_cast<int*>(ks + kTileJ * KLD);  // [kWarps][256]

  const int G = Hq / Hkv;
  const int BG = B * Hkv;
  const int ntiles = (nb + kGR - 1) / kGR;
  const int tile = ntiles - 1 - static_cast<int>(blockIdx.x / BG);  // heaviest tiles first
  const int bgi = static_cast<int>(blockIdx.x % BG);
  const int b = bgi / Hkv, g = bgi % Hkv;
  const int i0 = tile * kGR;
  const int rows = min(kGR, nb - i0);
  const int jend = i0 + rows;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t bg = static_cast<int64_t>(b) * Hkv + g;
  const float* ksrc = kbar + bg * nb * D;
  const float* nsrc = vnorm + bg * nb;
  const float scale = rsqrtf(static_cast<float>(D));

  for (int j = t; j < jend; j += kSelThreads) {
    double c;
    if (!metric.additive) {
      c = log(static_cast<double>(nsrc[j]));
    } else if (metric.beta == 0.f) {
      c = 0.0;
    } else {
      double e = 2.0 * log(static_cast<double>(nsrc[j]));
      if (metric.clamp && e < 0.0) e = 0.0;
      c = static_cast<double>(metric.beta) * e;
    }
    lnn[j] = c;
  }

  const int r = warp;  // this warp's query block in phases 1b and 2
  const int i = i0 + r;
  double* arow = acc + r * ldS;
  float* srow = srow_all + r * ldS;
  for (int h = 0; h < G; ++h) {
    const int64_t bh = static_cast<int64_t>(b) * Hq + g * G + h;
    const float* qsrc = qbar + (bh * nb + i0) * D;
    __syncthreads();  // the previous head's scores and qs are consumed
    for (int idx = t; idx < kGR * D / 4; idx += kSelThreads) {
      const int rr = idx / (D / 4), c4 = idx % (D / 4);
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (rr < rows) val = reinterpret_cast<const float4*>(qsrc + rr * D)[c4];
      reinterpret_cast<float4*>(qs + rr * D)[c4] = val;
    }
    // ---- phase 1: s[r][j] of head h for j < jend (warp w computes row w)
    for (int j0 = 0; j0 < jend; j0 += kTileJ) {
      __syncthreads();  // previous tile consumed (qs visible on the first pass)
      for (int idx = t; idx < kTileJ * D / 4; idx += kSelThreads) {
        const int rr = idx / (D / 4), c4 = idx % (D / 4);
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j0 + rr < jend) val = reinterpret_cast<const float4*>(ksrc + (j0 + rr) * D)[c4];
        *reinterpret_cast<float4*>(ks + rr * KLD + c4 * 4) = val;
      }
      __syncthreads();
      float a0 = 0.f, a1 = 0.f;
      const float* k0 = ks + lane * KLD;
      const float* k1 = ks + (lane + 32) * KLD;
      const float* qv = qs + r * D;
#pragma unroll 4
      for (int d = 0; d < D; d += 4) {
        const float4 x0 = *reinterpret_cast<const float4*>(k0 + d);
        const float4 x1 = *reinterpret_cast<const float4*>(k1 + d);
        const float4 q4 = *reinterpret_cast<const float4*>(qv + d);
        a0 = fmaf(q4.x, x0.x, a0);
        a0 = fmaf(q4.y, x0.y, a0);
        a0 = fmaf(q4.z, x0.z, a0);
        a0 = fmaf(q4.w, x0.w, a0);
        a1 = fmaf(q4.x, x1.x, a1);
        a1 = fmaf(q4.y, x1.y, a1);
        a1 = fmaf(q4.z, x1.z, a1);
        a1 = fmaf(q4.w, x1.w, a1);
      }
      if (j0 + lane < jend) srow[j0 + lane] = a0 * scale;
      if (j0 + lane + 32 < jend) srow[j0 + lane + 32] = a1 * scale;
    }
    __syncwarp();
    // ---- phase 1b: fold head h into the row's key (this warp's row only)
    if (r < rows) {
      if (!metric.additive) {
        float mx = -INFINITY;
        for (int j = lane; j <= i; j += 32) mx = fmaxf(mx, srow[j]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        double z = 0.0;
        for (int j = lane; j <= i; j += 32) z += exp(static_cast<double>(srow[j] - mx));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        const double lse = static_cast<double>(mx) + log(z);
        for (int j = lane; j <= i; j += 32) {
          const double x = static_cast<double>(srow[j]) - lse;  // log p_hij
          if (h == 0) {
            arow[j] = x;
          } else {  // log-add-exp
            const double a = arow[j];
            const double hi = fmax(a, x), lo = fmin(a, x);
            arow[j] = hi + log1p(exp(lo - hi));
          }
        }
      } else {
        for (int j = lane; j <= i; j += 32)
          arow[j] = (h == 0 ? 0.0 : arow[j]) + static_cast<double>(srow[j]);
      }
    }
  }
  __syncwarp();
  if (r >= rows) return;  // no __syncthreads below
  // ---- phase 2: the key, the diagnostic metric, the selection (this warp's row)
  const double gterm = metric.additive ? static_cast<double>(G) : 1.0;
  for (int j = lane; j <= i; j += 32) arow[j] += gterm * lnn[j];
  __syncwarp();
  const int kk = plan.k[i];
  const int64_t bh0 = static_cast<int64_t>(b) * Hq + g * G;
  for (int h = lane; h < G; h += 32) sel_cnt[(bh0 + h) * nb + i] = kk;
  if (m_out != nullptr) {
    // sum over the group's heads of the metric: n_j * sum_h p_hij (product) or the summed
    // additive score; the same row for every head of the group
    const int64_t tri = static_cast<int64_t>(nb) * (nb + 1) / 2;
    for (int j = lane; j <= i; j += 32) {
      const float mv = static_cast<float>(metric.additive ? arow[j] : exp(arow[j]));
      for (int h = 0; h < G; ++h)
        m_out[(bh0 + h) * tri + static_cast<int64_t>(i) * (i + 1) / 2 + j] = mv;
    }
  }
  auto key_bits = [&](int j) -> uint64_t { return order_bits(arow[j]); };
  select_row(i, kk, key_bits, hist_all + warp * 256, lane, sel_idx + bh0 * cap + plan.off[i], cap,
             G);
}

template <int D>
cudaError_t launch_group(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                         int Hkv, int nb, PlanDev plan, int64_t cap, SelMetric metric,
                         int32_t* sel_idx, int32_t* sel_cnt, float* m_out, cudaStream_t st) {
  const int ldS = (nb + 3) & ~3;
  const size_t smem = sizeof(double) * (static_cast<size_t>(kGR) * ldS + ldS) +
                      sizeof(float) * (static_cast<size_t>(kGR) * ldS + kGR * D +
                                       kTileJ * (D + 4)) +
                      sizeof(int) * kWarps * 256;
  auto kern = select_group_kernel<D>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t grid = static_cast<int64_t>(B) * Hkv * ((nb + kGR - 1) / kGR);
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), kSelThreads, smem, st>>>(qbar, kbar, vnorm, B, Hq, Hkv, nb,
                                                             ldS, plan, cap, metric, sel_idx,
                                                             sel_cnt, m_out);
  return cudaGetLastError();
}

template <int D, int R>
cudaError_t launch_rt(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                      int Hkv, int nb, PlanDev plan, int64_t cap, SelMetric metric,
                      int32_t* sel_idx, int32_t* sel_cnt, float* m_out, cudaStream_t st) {
  const int ldS = (nb + 3) & ~3;
  const size_t smem = sizeof(float) * (static_cast<size_t>(R) * ldS + R * D + kTileJ * (D + 4)) +
                      sizeof(double) * ldS + sizeof(int) * kWarps * 256;
  auto kern = select_kernel<D, R>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int BH = B * Hq;
  const int64_t grid = static_cast<int64_t>(BH) * ((nb + R - 1) / R);
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), kSelThreads, smem, st>>>(qbar, kbar, vnorm, BH, Hq, Hkv,
                                                             nb, ldS, plan, cap, metric,
                                                             sel_idx, sel_cnt, m_out);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                     int Hkv, int nb, PlanDev plan, int64_t cap, SelMetric metric,
                     int32_t* sel_idx, int32_t* sel_cnt, float* m_out, cudaStream_t st) {
  if (nb <= 1024)
    return launch_rt<D, 32>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx,
                            sel_cnt, m_out, st);
  if (nb <= 2048)
    return launch_rt<D, 16>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx,
                            sel_cnt, m_out, st);
  return launch_rt<D, 8>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx, sel_cnt,
                         m_out, st);
}

// ---- Selection from block probabilities p_ij (block scores by anti-diagonal sampling). ln p_ij
// takes the place of s_ij - lse_i: per head the key is ln p_ij + ln n_j (product) or
// ln p_ij + beta * e_j (additive); shared by a kv-head group it is ln n_j + logsumexp_h ln p_hij
// (product: the group's summed metric n_j * sum_h p_hij) or sum_h ln p_hij + G * beta * e_j.
// One CTA (8 warps) per (b, head or group, 8 consecutive query blocks), one row per warp; p rows
// are read from global memory (L1/L2), the group's combined row is built in shared memory.
template <bool kGroup>
__global__ void __launch_bounds__(kSelThreads) select_p_kernel(
    const float* __restrict__ p, const float* __restrict__ vnorm, int B, int Hq, int Hkv, int nb,
    int ldS, PlanDev plan, int64_t cap, SelMetric metric, int32_t* __restrict__ sel_idx,
    int32_t* __restrict__ sel_cnt, float* __restrict__ m_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* lnn = reinterpret_cast<double*>(smem_raw);                 // [ldS]
  double* acc = lnn + ldS;                                           // kGroup: [kWarps][ldS]
  int* hist_all = reinterpret_cast<int*>(acc + (kGroup ? kWarps * ldS : 0));  // [kWarps][256]
  const int G = Hq / Hkv;
  const int NH = kGroup ? B * Hkv : B * Hq;  // selection heads
  const int ntiles = (nb + kWarps - 1) / kWarps;
  const int tile = ntiles - 1 - static_cast<int>(blockIdx.x / NH);  // heaviest rows first
  const int sh = static_cast<int>(blockIdx.x % NH);
  const int b = kGroup ? sh / Hkv : sh / Hq;
  const int g = kGroup ? sh % Hkv : (sh % Hq) / G;  // kv head
  const int i0 = tile * kWarps;
  const int rows = min(kWarps, nb - i0);
  const int jend = i0 + rows;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t bg = static_cast<int64_t>(b) * Hkv + g;
  const float* nsrc = vnorm + bg * nb;
  const int64_t tri = static_cast<int64_t>(nb) * (nb + 1) / 2;
  for (int j = t; j < jend; j += kSelThreads) {
    double c;
    if (!metric.additive) {
      c = log(static_cast<double>(nsrc[j]));
    } else if (metric.beta == 0.f) {
      c = 0.0;
    } else {
      double e = 2.0 * log(static_cast<double>(nsrc[j]));
      if (metric.clamp && e < 0.0) e = 0.0;
      c = static_cast<double>(metric.beta) * e;
    }
    lnn[j] = c;
  }
  __syncthreads();
  if (warp >= rows) return;  // no __syncthreads below
  const int i = i0 + warp;
  const int kk = plan.k[i];
  const int64_t rowoff = static_cast<int64_t>(i) * (i + 1) / 2;
  int* hist = hist_all + warp * 256;
  if (!kGroup) {
    const int64_t bh = static_cast<int64_t>(b) * Hq + sh % Hq;
    const float* prow = p + bh * tri + rowoff;
    if (lane == 0) sel_cnt[bh * nb + i] = kk;
    if (m_out != nullptr)
      for (int j = lane; j <= i; j += 32)
        m_out[bh * tri + rowoff + j] =
            metric.additive ? static_cast<float>(log(static_cast<double>(prow[j])) + lnn[j])
                            : prow[j] * nsrc[j];
    auto key_bits = [&](int j) -> uint64_t {
      return order_bits(log(static_cast<double>(__ldg(prow + j))) + lnn[j]);
    };
    select_row(i, kk, key_bits, hist, lane, sel_idx + bh * cap + plan.off[i], 0, 1);
  } else {
    double* arow = acc + warp * ldS;
    const int64_t bh0 = static_cast<int64_t>(b) * Hq + g * G;
    for (int h = 0; h < G; ++h) {
      const float* prow = p + (bh0 + h) * tri + rowoff;
      for (int j = lane; j <= i; j += 32) {
        const double x = log(static_cast<double>(prow[j]));
        if (metric.additive) {
          arow[j] = (h == 0 ? 0.0 : arow[j]) + x;
        } else if (h == 0) {
          arow[j] = x;
        } else {  // log-add-exp; a zero probability adds nothing
          const double a = arow[j];
          const double hi = fmax(a, x), lo = fmin(a, x);
          arow[j] = lo == -INFINITY ? hi : hi + log1p(exp(lo - hi));
        }
      }
    }
    const double gterm = metric.additive ? static_cast<double>(G) : 1.0;
    for (int j = lane; j <= i; j += 32) arow[j] += gterm * lnn[j];
    __syncwarp();
    for (int h = lane; h < G; h += 32) sel_cnt[(bh0 + h) * nb + i] = kk;
    if (m_out != nullptr)
      for (int j = lane; j <= i; j += 32) {
        const float mv = static_cast<float>(metric.additive ? arow[j] : exp(arow[j]));
        for (int h = 0; h < G; ++h) m_out[(bh0 + h) * tri + rowoff + j] = mv;
      }
    auto key_bits = [&](int j) -> uint64_t { return order_bits(arow[j]); };
    select_row(i, kk, key_bits, hist, lane, sel_idx + bh0 * cap + plan.off[i], cap, G);
  }
}

template <bool kGroup>
cudaError_t launch_p(const float* p, const float* vnorm, int B, int Hq, int Hkv, int nb,
                     PlanDev plan, int64_t cap, SelMetric metric, int32_t* sel_idx,
                     int32_t* sel_cnt, float* m_out, cudaStream_t st) {
  const int ldS = (nb + 3) & ~3;
  const size_t smem = sizeof(double) * (static_cast<size_t>(ldS) * (kGroup ? 1 + kWarps : 1)) +
                      sizeof(int) * kWarps * 256;
  auto kern = select_p_kernel<kGroup>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t NH = kGroup ? static_cast<int64_t>(B) * Hkv : static_cast<int64_t>(B) * Hq;
  const int64_t grid = NH * ((nb + kWarps - 1) / kWarps);
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), kSelThreads, smem, st>>>(p, vnorm, B, Hq, Hkv, nb, ldS,
                                                             plan, cap, metric, sel_idx, sel_cnt,
                                                             m_out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_p(const float* p, const float* vnorm, int B, int Hq, int Hkv, int nb,
                            PlanDev plan, int64_t cap, SelMetric metric, int32_t* sel_idx,
                            int32_t* sel_cnt, float* m_out, cudaStream_t st) {
  if (B * Hq == 0 || nb == 0) return cudaSuccess;
  if (metric.group && Hq != Hkv)
    return launch_p<true>(p, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx, sel_cnt, m_out,
                          st);
  return launch_p<false>(p, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx, sel_cnt, m_out,
                         st);
}

// The split design over chunks of heads whose score triangles fit the scratch.
template <int D>
cudaError_t launch_split(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                         int Hkv, int nb, PlanDev plan, int64_t cap, SelMetric metric,
                         int32_t* sel_idx, int32_t* sel_cnt, float* m_out, float* scratch,
                         int chunk, cudaStream_t st) {
  const int nt = (nb + kScT - 1) / kScT;
  const int tiles = nt * (nt + 1) / 2;
  const size_t smem1 = sizeof(float) * 2 * kScT * (D + 4);
  const size_t smem2 = sizeof(double) * ((nb + 3) & ~3) + sizeof(int) * kWarps * 256;
  cudaError_t e = cudaFuncSetAttribute(score_tri_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem1));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(select_s_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem2));
  if (e != cudaSuccess) return e;
  const int heads = B * Hq;
  for (int h0 = 0; h0 < heads; h0 += chunk) {
    const int nh = std::min(chunk, heads - h0);
    const int64_t g1 = static_cast<int64_t>(nh) * tiles;
    const int64_t g2 = static_cast<int64_t>(nh) * ((nb + kWarps - 1) / kWarps);
    if (g1 > 0x7fffffff || g2 > 0x7fffffff) return cudaErrorInvalidConfiguration;
    score_tri_kernel<D><<<static_cast<unsigned>(g1), kSelThreads, smem1, st>>>(
        qbar, kbar, Hq, Hkv, nb, h0, tiles, scratch);
    select_s_kernel<<<static_cast<unsigned>(g2), kSelThreads, smem2, st>>>(
        scratch, vnorm, Hq, Hkv, nb, h0, nh, plan, cap, metric, sel_idx, sel_cnt, m_out);
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const float* qbar, const float* kbar, const float* vnorm, int B,
                          int Hq, int Hkv, int nb, int D, PlanDev plan, int64_t cap,
                          SelMetric metric, int32_t* sel_idx, int32_t* sel_cnt, float* m_out,
                          cudaStream_t st, float* scratch, size_t scratch_bytes) {
  if (B * Hq == 0 || nb == 0) return cudaSuccess;
  const size_t tri_bytes = sizeof(float) * (static_cast<size_t>(nb) * (nb + 1) / 2);
  const int64_t chunk = scratch ? static_cast<int64_t>(scratch_bytes / tri_bytes) : 0;
  if (!(metric.group && Hq != Hkv) && chunk >= 1) {
    const int c = static_cast<int>(std::min<int64_t>(chunk, static_cast<int64_t>(B) * Hq));
    if (D == 128)
      return launch_split<128>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx,
                               sel_cnt, m_out, scratch, c, st);
    if (D == 64)
      return launch_split<64>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx,
                              sel_cnt, m_out, scratch, c, st);
    return cudaErrorInvalidValue;
  }
  if (metric.group && Hq != Hkv) {
    if (D == 128)
      return launch_group<128>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx,
                               sel_cnt, m_out, st);
    if (D == 64)
      return launch_group<64>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx,
                              sel_cnt, m_out, st);
    return cudaErrorInvalidValue;
  }
  if (D == 128)
    return launch_d<128>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx, sel_cnt,
                         m_out, st);
  if (D == 64)
    return launch_d<64>(qbar, kbar, vnorm, B, Hq, Hkv, nb, plan, cap, metric, sel_idx, sel_cnt,
                        m_out, st);
  return cudaErrorInvalidValue;
}

}  // namespace stem
