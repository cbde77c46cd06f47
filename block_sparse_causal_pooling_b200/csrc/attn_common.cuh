// Shared device code of the tensor-core attention kernels (attn_sm100.cu for block 128,
// attn_sm100_b64.cu for block 64): the CTA's barrier block, the bounded waits, f32x2
// arithmetic, the product groups issued from one asm block, the shared-memory P store and the
// ring of claimed work items. Everything is in an anonymous namespace: each kernel file gets its
// own copy.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sm100.cuh"
#include "stem.h"

namespace stem {
namespace {

using namespace sm100;

constexpr int kN = 128;             // key columns of an S tile
constexpr int kMaxSlots = 4;        // K/V ring slots (at most)
constexpr int kThreads = 384;       // 12 warps: three warpgroups
constexpr int kGroupThreads = 128;  // softmax threads of one head
constexpr int kSoftmaxThreads = 2 * kGroupThreads;
constexpr uint32_t kTmemCols = 512;
constexpr int kItemRing = 8;                       // claimed work items in flight
constexpr int kItemReaders = 1 + kSoftmaxThreads;  // MMA thread and softmax threads
constexpr float kRescale = 8.0f;  // a row's reference max moves when exceeded by this (log2)

struct __align__(8) Bars {
  uint64_t q_full[2], q_empty[2];            // per tile (A, B)
  uint64_t kv_full[kMaxSlots], kv_empty[kMaxSlots];
  uint64_t s_full[2];   // S_T complete (commit)
  uint64_t s_free[2];   // S_T read into registers by the head's softmax threads
  uint64_t p_full[2];   // P_T written to shared memory
  uint64_t pv_done[2];  // P V_T complete (commit): P_T may be rewritten, O_T read
  uint64_t o_empty[2];  // the epilogue has read O_T
  uint64_t iq_full[kItemRing], iq_empty[kItemRing];  // claimed items, producer -> readers
  int64_t iq[kItemRing];                     // item index, or -1: none left
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
};


// ---------------------------------------------------------------- PTX helpers

// Bounded wait for the phase of parity `parity` of barrier b. Returns false (after recording
// the timeout) if it expired or another role already aborted. Inlined: a call inside the
// register-reallocated regions of the kernel would pin every warp to one register count.
__device__ __forceinline__ bool wait_bar_slow(uint64_t* b, uint32_t parity, Bars* bars,
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
// P V group: O += P V over the 128 keys, both operands in shared memory. A = P, K-major
// 128B-swizzled like a Q tile (keys 16kk.. of k-step kk at descriptor offset
// (kk / 4) * 1024 + (kk % 4) * 2); B = V MN-major (16 key rows of 128 bytes per k-step:
// descriptor offset kk * 128). acc0 = 0 starts O afresh.
// operands: %0 d, %1 a_lo, %2 b_lo, %3 hi, %4 idesc, %5 acc0
#define STEM_MMA_PV(AOFF, BOFF)                                                            \
  "add.u32 x, %1, " #AOFF ";\n\tadd.u32 y, %2, " #BOFF ";\n\t"                             \
  "mov.b64 a, {x, %3};\n\tmov.b64 b, {y, %3};\n\t"                                        \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, pt;\n\t"
__device__ __forceinline__ void mma_pv8(uint32_t d, uint32_t alo, uint32_t blo, uint32_t hi,
                                        uint32_t idesc, uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, pt;\n\t.reg .b32 x, y;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p0, %5, 0;\n\tsetp.eq.b32 pt, %4, %4;\n\t"
      "mov.b64 a, {%1, %3};\n\tmov.b64 b, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p0;\n\t"
      STEM_MMA_PV(2, 128) STEM_MMA_PV(4, 256) STEM_MMA_PV(6, 384) STEM_MMA_PV(1024, 512)
      STEM_MMA_PV(1026, 640) STEM_MMA_PV(1028, 768) STEM_MMA_PV(1030, 896)
      "}" ::"r"(d), "r"(alo), "r"(blo), "r"(hi), "r"(idesc), "r"(acc0)
      : "memory");
}
__device__ __forceinline__ void mma_pv4(uint32_t d, uint32_t alo, uint32_t blo, uint32_t hi,
                                        uint32_t idesc, uint32_t acc0) {  // 64 keys
  asm volatile(
      "{\n\t.reg .pred p0, pt;\n\t.reg .b32 x, y;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p0, %5, 0;\n\tsetp.eq.b32 pt, %4, %4;\n\t"
      "mov.b64 a, {%1, %3};\n\tmov.b64 b, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p0;\n\t"
      STEM_MMA_PV(2, 128) STEM_MMA_PV(4, 256) STEM_MMA_PV(6, 384)
      "}" ::"r"(d), "r"(alo), "r"(blo), "r"(hi), "r"(idesc), "r"(acc0)
      : "memory");
}
#undef STEM_MMA_PV

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void sched_step(uint32_t e, int i, int& ba, int& bb) {
  ba = min(static_cast<int>(e & 0xFFFFu), i);
  const uint32_t hb = e >> 16;
  bb = hb == 0xFFFFu ? -1 : min(static_cast<int>(hb), i);
}

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

}  // namespace
}  // namespace stem
