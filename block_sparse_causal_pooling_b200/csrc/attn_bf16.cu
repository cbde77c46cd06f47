// Block-sparse causal attention for bfloat16 inputs (tensor cores, float32 accumulation).
//
// Exact softmax attention of every query token of block i over every token of its kept blocks,
// token-causal inside block i ("Stem: Rethinking Causal Information Flow in Sparse Attention",
// gist.science/es "Resumen tecnico" 2 "Implementacion" step 3; gist.science/it 2.C step 3;
// gist.science/nl "Implementatie" step 3; gist.science/fr 2.C step 3).
//
// One CTA per work item (b, h, i): BLOCK query rows, BLOCK/16 warps of 16 rows each. The kept
// key blocks are streamed in sub-tiles of 64 keys through a two-stage cp.async pipeline
// (XOR-swizzled 16-byte chunks, conflict-free ldmatrix); S = Q K^T and O += P V run on
// mma.sync.m16n8k16 (bf16 in, f32 accumulate) with an online softmax in float32 (exp2 with the
// 1/sqrt(D) scale folded in). Work items are ordered kv-head-group-major so the CTAs in flight
// share one kv head's K/V in L2, heaviest query blocks first. In a partial last block (S not a
// multiple of BLOCK) rows past S are zero-filled on load and never stored.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "stem_internal.h"

namespace stem {
namespace {

constexpr int kKT = 64;  // keys per sub-tile

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
// 16 bytes, or 16 zero bytes (nothing read) when !valid; src must still point into the tensor.
__device__ __forceinline__ void cp_async16z(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float bf16r(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of the 16-byte chunk (row, chunk) in a [rows][D] bf16 tile, chunks XOR-swizzled
// by the row's low three bits.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * (D * 2) + ((chunk ^ (row & 7)) << 4));
}

template <int D, int BLOCK>
__global__ void __launch_bounds__(BLOCK * 2) attn_bf16_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, int Hq, int Hkv, int S, int nb, PlanDev plan,
    int64_t cap, const int32_t* __restrict__ sel_idx, __nv_bfloat16* __restrict__ out) {
  constexpr int NT = BLOCK * 2;        // threads: BLOCK/16 warps
  constexpr int CH = D / 8;            // 16-byte chunks per row
  constexpr int SUB = BLOCK / kKT;     // sub-tiles per key block
  constexpr int KC = D / 16;           // k16 chunks of the head dimension
  constexpr int NTD = D / 8;           // n8 tiles of the output
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* qs = smem;                                   // [BLOCK][D]
  unsigned char* ks = qs + BLOCK * D * 2;                     // [2][kKT][D]
  unsigned char* vs = ks + 2 * kKT * D * 2;                   // [2][kKT][D]

  const int G = Hq / Hkv;
  const int64_t item = blockIdx.x;
  const int64_t per_group = static_cast<int64_t>(G) * nb;
  const int64_t bg = item / per_group;
  const int rem = static_cast<int>(item % per_group);
  const int i = plan.order[rem / G];
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int h = g * G + rem % G;
  const int64_t bh = static_cast<int64_t>(b) * Hq + h;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const __nv_bfloat16* qsrc = q + (bh * S + static_cast<int64_t>(i) * BLOCK) * D;
  const __nv_bfloat16* ksrc = k + bg * S * D;
  const __nv_bfloat16* vsrc = v + bg * S * D;
  const int cnt = plan.k[i];
  const int32_t* list = sel_idx + bh * cap + plan.off[i];
  const int ntiles = cnt * SUB;

  auto tile_row0 = [&](int tt) -> int64_t {  // first key row of sub-tile tt
    const int j = min(max(list[tt / SUB], 0), i);
    return static_cast<int64_t>(j) * BLOCK + (tt % SUB) * kKT;
  };
  auto load_tile = [&](int tt, int stage) {
    const int64_t row0 = tile_row0(tt);
    const uint32_t kb = smem_u32(ks + stage * kKT * D * 2);
    const uint32_t vb = smem_u32(vs + stage * kKT * D * 2);
    for (int idx = t; idx < kKT * CH; idx += NT) {
      const int r = idx / CH, c = idx % CH;
      const bool ok = row0 + r < S;
      const int64_t rr = ok ? row0 + r : S - 1;
      cp_async16z(kb + swz<D>(r, c), ksrc + rr * D + c * 8, ok);
      cp_async16z(vb + swz<D>(r, c), vsrc + rr * D + c * 8, ok);
    }
  };

  // Q tile and the first K/V sub-tile
  {
    const uint32_t qb = smem_u32(qs);
    for (int idx = t; idx < BLOCK * CH; idx += NT) {
      const int r = idx / CH, c = idx % CH;
      const bool ok = static_cast<int64_t>(i) * BLOCK + r < S;
      cp_async16z(qb + swz<D>(r, c), qsrc + static_cast<int64_t>(ok ? r : 0) * D + c * 8, ok);
    }
  }
  load_tile(0, 0);
  cp_commit();

  const int wrow = warp * 16;  // first query row of this warp
  uint32_t qf[KC][4];
  float o[NTD][4];
#pragma unroll
  for (int n = 0; n < NTD; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));  // log2(e)/sqrt(D)
  const int gq = lane >> 2, tq = lane & 3;

  for (int tt = 0; tt < ntiles; ++tt) {
    const int stage = tt & 1;
    if (tt + 1 < ntiles) load_tile(tt + 1, stage ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    if (tt == 0) {
      const uint32_t qb = smem_u32(qs);
#pragma unroll
      for (int kc = 0; kc < KC; ++kc) {
        const int row = wrow + (lane & 15);
        const int chunk = kc * 2 + (lane >> 4);
        ldsm_x4(qb + swz<D>(row, chunk), qf[kc][0], qf[kc][1], qf[kc][2], qf[kc][3]);
      }
    }
    const uint32_t kb = smem_u32(ks + stage * kKT * D * 2);
    const uint32_t vb = smem_u32(vs + stage * kKT * D * 2);

    // S = Q K^T for 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {  // pairs of n8 tiles
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int chunk = kc * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz<D>(key, chunk), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[kc], b0, b1);
        mma_bf16(s[2 * np + 1], qf[kc], b2, b3);
      }
    }
    // causal mask on the diagonal block
    const int64_t row0 = tile_row0(tt);
    const int64_t qtok0 = static_cast<int64_t>(i) * BLOCK;
    if (row0 + kKT > qtok0) {
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t key = row0 + n * 8 + 2 * tq + (e & 1);
          const int64_t qt = qtok0 + wrow + gq + ((e >> 1) << 3);
          if (key > qt) s[n][e] = -INFINITY;
        }
      }
    }
    // online softmax (rows gq and gq+8 of this warp's 16)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float mx = -INFINITY;
#pragma unroll
      for (int n = 0; n < 8; ++n) mx = fmaxf(mx, fmaxf(s[n][2 * hr], s[n][2 * hr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(mrow[hr], mx * sl2);
      const float muse = (mnew == -INFINITY) ? 0.f : mnew;
      const float alpha = ex2(mrow[hr] - muse);
      mrow[hr] = mnew;
      float sum = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        // P rounded to bf16 here, so the row sum takes the same values that enter P V
        const float p0 = bf16r(ex2(s[n][2 * hr] * sl2 - muse));
        const float p1 = bf16r(ex2(s[n][2 * hr + 1] * sl2 - muse));
        s[n][2 * hr] = p0;
        s[n][2 * hr + 1] = p1;
        sum += p0 + p1;
      }
      lrow[hr] = lrow[hr] * alpha + sum;  // per-thread partial; quad-reduced at the end
#pragma unroll
      for (int n = 0; n < NTD; ++n) {
        o[n][2 * hr] *= alpha;
        o[n][2 * hr + 1] *= alpha;
      }
    }
    // O += P V
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {  // 16 keys per step
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kc][0], s[2 * kc][1]);
      pa[1] = pack_bf16(s[2 * kc][2], s[2 * kc][3]);
      pa[2] = pack_bf16(s[2 * kc + 1][0], s[2 * kc + 1][1]);
      pa[3] = pack_bf16(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
      for (int np = 0; np < NTD / 2; ++np) {  // pairs of n8 tiles of D
        const int key = kc * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int chunk = np * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz<D>(key, chunk), b0, b1, b2, b3);
        mma_bf16(o[2 * np], pa, b0, b1);
        mma_bf16(o[2 * np + 1], pa, b2, b3);
      }
    }
    __syncthreads();  // this stage is refilled two iterations from now
  }
  cp_wait<0>();

  // normalise and store
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    float l = lrow[hr];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = 1.0f / l;
    const int64_t tok = static_cast<int64_t>(i) * BLOCK + wrow + gq + hr * 8;
    if (tok >= S) continue;  // partial last block
    __nv_bfloat16* dst = out + (bh * S + tok) * D;
#pragma unroll
    for (int n = 0; n < NTD; ++n) {
      const uint32_t pk = pack_bf16(o[n][2 * hr] * inv, o[n][2 * hr + 1] * inv);
      *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * tq) = pk;
    }
  }
}

template <int D, int BLOCK>
cudaError_t launch_typed(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                         int S, PlanDev plan, int64_t cap, const int32_t* sel_idx, void* out,
                         cudaStream_t st) {
  const int nb = (S + BLOCK - 1) / BLOCK;
  const int64_t items = static_cast<int64_t>(B) * Hq * nb;
  if (items == 0) return cudaSuccess;
  if (items > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const size_t smem = static_cast<size_t>(BLOCK) * D * 2 + 4 * kKT * D * 2;
  auto kern = attn_bf16_mma_kernel<D, BLOCK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(items), BLOCK * 2, smem, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), Hq, Hkv, S, nb, plan, cap, sel_idx,
      static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace

// mma.sync path: block = 64 (the tcgen05 kernel in attn_sm100.cu covers block = 128).
cudaError_t launch_attn_bf16_mma(const void* q, const void* k, const void* v, int B, int Hq,
                                 int Hkv, int S, int D, int block, PlanDev plan, int64_t cap,
                                 const int32_t* sel_idx, void* out, cudaStream_t st) {
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
