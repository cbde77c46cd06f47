// Block pooling: "block downsampling" of Q, K and V, the first stage of Stem's prefill
// ("Stem: Rethinking Causal Information Flow in Sparse Attention", gist.science/es
// "Resumen tecnico" 2 "Implementacion" step 1; gist.science/it 2.C step 1; gist.science/nl
// "Implementatie" step 1). Mean pooling is the reading used:
//   qbar[b,h,i,:] = mean of Q rows i*block .. i*block+block-1,
//   kbar[b,g,i,:] = mean of K rows of block i,
//   vnorm[b,g,i]  = mean over the block's rows of the row's Euclidean norm, or (vmax) the
//                   largest row norm ("maximised magnitudes of V", gist.science/nl step 1).
// A partial last block (S % block != 0) is pooled over its S - i*block rows: rows past S are
// neither read nor counted.
//
// Design (HBM-bound: every input byte is read once, outputs are ~1/64 of the input):
//   - one CTA of 256 threads per (tensor, b, head, block) unit; a unit is one contiguous
//     block*D*sizeof(T) byte span (32 KB for bf16, block 128, D 128);
//   - each thread issues all of its 16-byte streaming loads before using any of them;
//   - float32 accumulation in a fixed pairwise order: within a thread across its rows, then a
//     shared-memory tree across row groups (depth log2(block) for the column sums); for V the
//     row's sum of squares is a register tree then a warp-shuffle tree. The result is
//     deterministic and its rounding error grows with log2(block), not with block.
#include <cuda_bf16.h>

#include "stem_internal.h"

namespace stem {
namespace {

constexpr int kPoolThreads = 256;

template <typename T>
struct Vec16;  // 16 bytes of T widened to float
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void widen(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void widen(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
};

// In-register pairwise sum of x[0..N), N a power of two.
template <int N>
__device__ __forceinline__ float pairwise(float* x) {
#pragma unroll
  for (int s = N / 2; s >= 1; s /= 2) {
#pragma unroll
    for (int i = 0; i < s; ++i) x[i] = x[i] + x[i + s];
  }
  return x[0];
}

template <typename T, int D, int BLOCK>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const T* __restrict__ q,
                                                            const T* __restrict__ k,
                                                            const T* __restrict__ v, int nq,
                                                            int nk, int nb, int S, int vmax,
                                                            float* __restrict__ qbar,
                                                            float* __restrict__ kbar,
                                                            float* __restrict__ vnorm) {
  constexpr int E = Vec16<T>::N;          // elements per 16-byte chunk
  constexpr int CPR = D / E;              // chunks per row (8, 16 or 32)
  constexpr int RPI = kPoolThreads / CPR; // rows per pass
  constexpr int ITERS = BLOCK / RPI;      // passes per block
  static_assert(ITERS >= 1 && (ITERS & (ITERS - 1)) == 0, "power-of-two passes");
  static_assert(CPR <= 32 && (CPR & (CPR - 1)) == 0, "row must fit in a warp");
  __shared__ float part[RPI][D];

  const int u = blockIdx.x;
  const int t = threadIdx.x;
  const int c = t % CPR;
  const int rg = t / CPR;

  int kind;  // 0 = Q, 1 = K, 2 = V
  int64_t unit;
  if (u < nq) {
    kind = 0;
    unit = u;
  } else if (u < nq + nk) {
    kind = 1;
    unit = u - nq;
  } else {
    kind = 2;
    unit = u - nq - nk;
  }
  const T* src = kind == 0 ? q : (kind == 1 ? k : v);
  const int64_t bh = unit / nb;
  const int64_t i = unit % nb;
  const uint4* base =
      reinterpret_cast<const uint4*>(src + (bh * S + i * BLOCK) * static_cast<int64_t>(D));
  const int n = static_cast<int>(min(static_cast<int64_t>(BLOCK), S - i * BLOCK));  // rows

  uint4 raw[ITERS];
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const int row = rg + it * RPI;
    raw[it] = row < n ? __ldcs(base + row * CPR + c) : make_uint4(0u, 0u, 0u, 0u);
  }

  if (kind < 2) {
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float col[ITERS];
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
        float f[E];
        Vec16<T>::widen(raw[it], f);
        col[it] = f[e];
      }
      acc[e] = pairwise<ITERS>(col);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) part[rg][c * E + e] = acc[e];
    __syncthreads();
#pragma unroll
    for (int s = RPI / 2; s >= 1; s /= 2) {
      for (int idx = t; idx < s * D; idx += kPoolThreads) {
        const int r = idx / D, d = idx % D;
        part[r][d] = part[r][d] + part[r + s][d];
      }
      __syncthreads();
    }
    float* dst = (kind == 0 ? qbar : kbar) + unit * D;
    for (int d = t; d < D; d += kPoolThreads) dst[d] = part[0][d] / static_cast<float>(n);
  } else {
    float norms[ITERS];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      float f[E];
      Vec16<T>::widen(raw[it], f);
#pragma unroll
      for (int e = 0; e < E; ++e) f[e] = f[e] * f[e];
      float sq = pairwise<E>(f);
#pragma unroll
      for (int o = CPR / 2; o >= 1; o /= 2) sq += __shfl_xor_sync(0xffffffffu, sq, o, CPR);
      norms[it] = sqrtf(sq);
    }
    float mine;
    if (vmax) {
      mine = norms[0];
#pragma unroll
      for (int it = 1; it < ITERS; ++it) mine = fmaxf(mine, norms[it]);
    } else {
      mine = pairwise<ITERS>(norms);
    }
    if (c == 0) part[rg][0] = mine;
    __syncthreads();
#pragma unroll
    for (int s = RPI / 2; s >= 1; s /= 2) {
      if (t < s) part[t][0] = vmax ? fmaxf(part[t][0], part[t + s][0]) : part[t][0] + part[t + s][0];
      __syncthreads();
    }
    if (t == 0) vnorm[unit] = vmax ? part[0][0] : part[0][0] / static_cast<float>(n);
  }
}

template <typename T, int D, int BLOCK>
cudaError_t launch_typed(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                         int S, bool vmax, float* qbar, float* kbar, float* vnorm,
                         cudaStream_t st) {
  const int nb = (S + BLOCK - 1) / BLOCK;
  const int64_t nq = static_cast<int64_t>(B) * Hq * nb;
  const int64_t nk = static_cast<int64_t>(B) * Hkv * nb;
  const int64_t units = nq + 2 * nk;
  if (units <= 0) return cudaSuccess;
  if (units > 0x7fffffff) return cudaErrorInvalidConfiguration;
  pool_kernel<T, D, BLOCK><<<static_cast<unsigned>(units), kPoolThreads, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<int>(nq), static_cast<int>(nk), nb, S, vmax ? 1 : 0, qbar, kbar, vnorm);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dispatch(const void* q, const void* k, const void* v, int B, int Hq,
                            int Hkv, int S, int D, int block, bool vmax, float* qbar, float* kbar,
                            float* vnorm, cudaStream_t st) {
  if (D == 128 && block == 128)
    return launch_typed<T, 128, 128>(q, k, v, B, Hq, Hkv, S, vmax, qbar, kbar, vnorm, st);
  if (D == 128 && block == 64)
    return launch_typed<T, 128, 64>(q, k, v, B, Hq, Hkv, S, vmax, qbar, kbar, vnorm, st);
  if (D == 64 && block == 128)
    return launch_typed<T, 64, 128>(q, k, v, B, Hq, Hkv, S, vmax, qbar, kbar, vnorm, st);
  if (D == 64 && block == 64)
    return launch_typed<T, 64, 64>(q, k, v, B, Hq, Hkv, S, vmax, qbar, kbar, vnorm, st);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_pool(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                        int Hkv, int S, int D, int block, bool vmax, float* qbar, float* kbar,
                        float* vnorm, cudaStream_t st) {
  if (dtype == 0)
    return launch_dispatch<__nv_bfloat16>(q, k, v, B, Hq, Hkv, S, D, block, vmax, qbar, kbar,
                                          vnorm, st);
  return launch_dispatch<float>(q, k, v, B, Hq, Hkv, S, D, block, vmax, qbar, kbar, vnorm, st);
}

}  // namespace stem
