// Block-sparse causal attention for float32 inputs, on the CUDA cores.
//
// Exact softmax attention of every query token of block i over every token of its kept blocks,
// token-causal inside block i ("Stem: Rethinking Causal Information Flow in Sparse Attention",
// gist.science/es "Resumen tecnico" 2 "Implementacion" step 3; gist.science/it 2.C step 3;
// gist.science/nl "Implementatie" step 3). float32 inputs have no tensor-core path of the same
// precision, so this kernel keeps everything in float32: four threads per query row, each
// owning D/4 output columns; the kept K/V blocks are staged one at a time in shared memory; an
// online softmax runs over chunks of 16 keys (one rescale per chunk).
#include <cuda_runtime.h>
#include <math.h>

#include "stem_internal.h"

namespace stem {
namespace {

constexpr int kTPR = 4;     // threads per query row
constexpr int kChunk = 16;  // keys per online-softmax step

template <int D, int BLOCK>
__global__ void __launch_bounds__(BLOCK* kTPR) attn_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    int Hq, int Hkv, int S, int nb, PlanDev plan, int64_t cap,
    const int32_t* __restrict__ sel_idx, float* __restrict__ out) {
  constexpr int DS = D / kTPR;  // columns per thread
  extern __shared__ __align__(16) float kv_smem[];
  float* ks = kv_smem;              // [BLOCK][D]
  float* vs = kv_smem + BLOCK * D;  // [BLOCK][D]

  const int G = Hq / Hkv;
  const int64_t item = blockIdx.x;
  const int64_t per_group = static_cast<int64_t>(G) * nb;
  const int64_t bg = item / per_group;
  const int rem = static_cast<int>(item % per_group);
  const int i = plan.order[rem / G];
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int h = g * G + rem % G;
  const int64_t bh = static_cast<int64_t>(b) * Hq + h;

  const int t = threadIdx.x;
  const int r = t / kTPR;   // query row within the block
  const int part = t % kTPR;
  const int64_t qtok = static_cast<int64_t>(i) * BLOCK + r;
  const bool qvalid = qtok < S;  // rows past S of a partial last block: computed on 0, not stored
  const int64_t qrow = bh * S + (qvalid ? qtok : S - 1);
  const float* kvk = k + (bg * S) * D;
  const float* kvv = v + (bg * S) * D;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));

  float qv[DS], o[DS];
#pragma unroll
  for (int d = 0; d < DS; ++d) {
    qv[d] = qvalid ? q[qrow * D + part * DS + d] * scale : 0.f;
    o[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  const int cnt = plan.k[i];
  const int32_t* list = sel_idx + bh * cap + plan.off[i];
  for (int e = 0; e < cnt; ++e) {
    const int j = min(max(list[e], 0), i);  // stay inside [0, i] whatever the list holds
    __syncthreads();
    const float4* srcK = reinterpret_cast<const float4*>(kvk + static_cast<int64_t>(j) * BLOCK * D);
    const float4* srcV = reinterpret_cast<const float4*>(kvv + static_cast<int64_t>(j) * BLOCK * D);
    const int nrows = static_cast<int>(min(static_cast<int64_t>(BLOCK),
                                           S - static_cast<int64_t>(j) * BLOCK));
    for (int idx = t; idx < BLOCK * D / 4; idx += BLOCK * kTPR) {
      const bool ok = idx / (D / 4) < nrows;  // rows past S: zeros (causally masked anyway)
      reinterpret_cast<float4*>(ks)[idx] = ok ? srcK[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
      reinterpret_cast<float4*>(vs)[idx] = ok ? srcV[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    const int last = (j == i) ? r : BLOCK - 1;  // token-causal on the diagonal block
    // trip count uniform across the warp (rows r|7 .. of one warp share it) for the shuffles;
    // c0 <= BLOCK-16 always, so every key read stays inside the staged block
    const int last_w = (j == i) ? (r | 7) : BLOCK - 1;
    for (int c0 = 0; c0 <= last_w; c0 += kChunk) {
      float sc[kChunk];
      float cmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < kChunk; ++c) {
        const float* kr = ks + (c0 + c) * D + part * DS;
        float acc = 0.f;
#pragma unroll
        for (int d = 0; d < DS; ++d) acc = fmaf(qv[d], kr[d], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        sc[c] = (c0 + c <= last) ? acc : -INFINITY;
        cmax = fmaxf(cmax, sc[c]);
      }
      const float mnew = fmaxf(m, cmax);
      const float alpha = expf(m - mnew);  // m == -inf on the first chunk: alpha = 0
      l *= alpha;
#pragma unroll
      for (int d = 0; d < DS; ++d) o[d] *= alpha;
#pragma unroll
      for (int c = 0; c < kChunk; ++c) {
        const float p = expf(sc[c] - mnew);
        l += p;
        const float* vr = vs + (c0 + c) * D + part * DS;
#pragma unroll
        for (int d = 0; d < DS; ++d) o[d] = fmaf(p, vr[d], o[d]);
      }
      m = mnew;
    }
  }
  const float inv = 1.0f / l;
  if (!qvalid) return;
#pragma unroll
  for (int d = 0; d < DS; ++d) out[qrow * D + part * DS + d] = o[d] * inv;
}

template <int D, int BLOCK>
cudaError_t launch_typed(const float* q, const float* k, const float* v, int B, int Hq, int Hkv,
                         int S, PlanDev plan, int64_t cap, const int32_t* sel_idx, float* out,
                         cudaStream_t st) {
  const int nb = (S + BLOCK - 1) / BLOCK;
  const int64_t items = static_cast<int64_t>(B) * Hq * nb;
  if (items == 0) return cudaSuccess;
  if (items > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const size_t smem = 2 * sizeof(float) * BLOCK * D;
  auto kern = attn_f32_kernel<D, BLOCK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(items), BLOCK * kTPR, smem, st>>>(q, k, v, Hq, Hkv, S, nb, plan,
                                                                cap, sel_idx, out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_f32(const float* q, const float* k, const float* v, int B, int Hq,
                            int Hkv, int S, int D, int block, PlanDev plan, int64_t cap,
                            const int32_t* sel_idx, const int32_t*, float* out,
                            cudaStream_t st) {
  if (D == 128 && block == 128)
    return launch_typed<128, 128>(q, k, v, B, Hq, Hkv, S, plan, cap, sel_idx, out, st);
  if (D == 128 && block == 64)
    return launch_typed<128, 64>(q, k, v, B, Hq, Hkv, S, plan, cap, sel_idx, out, st);
  if (D == 64 && block == 128)
    return launch_typed<64, 128>(q, k, v, B, Hq, Hkv, S, plan, cap, sel_idx, out, st);
  if (D == 64 && block == 64)
    return launch_typed<64, 64>(q, k, v, B, Hq, Hkv, S, plan, cap, sel_idx, out, st);
  return cudaErrorInvalidValue;
}

}  // namespace stem
