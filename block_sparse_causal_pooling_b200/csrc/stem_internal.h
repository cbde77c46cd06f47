// Internal declarations shared by the host API (api.cpp) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace stem {

// Device view of the budget plan (int32 arrays inside the workspace).
struct PlanDev {
  const int32_t* k;      // [nb]   k(i)
  const int32_t* off;    // [nb+1] prefix sums of k
  const int32_t* order;  // [nb]   query blocks sorted by k(i) descending (heaviest first)
};

// Block pooling (pool.cu). dtype: 0 bf16, 1 f32. vmax: vnorm is the largest V-row norm of the
// block instead of the mean.
cudaError_t launch_pool(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                        int Hkv, int S, int D, int block, bool vmax, float* qbar, float* kbar,
                        float* vnorm, cudaStream_t st);

// Block metric of the selection: product (rank by s + ln n) or additive (rank by
// s + beta * e, e = 2 ln n clamped at 0 when clamp).
struct SelMetric {
  bool additive = false;
  float beta = 0.f;
  bool clamp = true;
  bool group = false;  // one selection per kv-head group (metric summed over its query heads)
};

// Largest nb the group-shared selection supports (its per-CTA key rows live in shared memory).
constexpr int kGroupMaxNb = 1024;

// Metric + top-k selection (select.cu). With scratch (at least one head's score triangle,
// 4*nb*(nb+1)/2 bytes) and per-head selection it runs as two kernels, scores then selection,
// over chunks of heads; otherwise (scratch NULL, or group share) as one fused kernel. Both give
// the same selection.
cudaError_t launch_select(const float* qbar, const float* kbar, const float* vnorm, int B,
                          int Hq, int Hkv, int nb, int D, PlanDev plan, int64_t cap,
                          SelMetric metric, int32_t* sel_idx, int32_t* sel_cnt, float* m_out,
                          cudaStream_t st, float* scratch = nullptr, size_t scratch_bytes = 0);

// Block probabilities by anti-diagonal sampling (antidiag_sm100.cu), bf16 inputs, D 64 or 128,
// stride | block, stride | S, block/stride a power of two <= 32. p: [B*Hq][nb*(nb+1)/2] rows of
// p_ij (j <= i); scratch: antidiag_scratch_floats() floats; status as for the attention.
constexpr int kAdSlots = 148;  // most CTAs the kernel runs (one scratch slot each)
cudaError_t launch_antidiag(const void* q, const void* k, int B, int Hq, int Hkv, int S, int D,
                            int block, int stride, float* p, float* scratch, int32_t* status,
                            cudaStream_t st);
int64_t antidiag_units(int B, int Hq, int S, int stride);
size_t antidiag_scratch_floats(int B, int Hq, int S, int block, int stride);

// Top-k selection from block probabilities p (select.cu): ranks ln p_ij + ln n_j (product) or
// ln p_ij + beta * e_j (additive), per query head or summed over a kv-head group like
// launch_select.
cudaError_t launch_select_p(const float* p, const float* vnorm, int B, int Hq, int Hkv, int nb,
                            PlanDev plan, int64_t cap, SelMetric metric, int32_t* sel_idx,
                            int32_t* sel_cnt, float* m_out, cudaStream_t st);

// Block-sparse attention, bfloat16 inputs on the tensor cores (attn_sm100.cu for block 128,
// attn_sm100_b64.cu for block 64). `sched` is workspace of pairs_bytes() for the head-pair
// step schedule (pairs.cu).
cudaError_t launch_attn_bf16(const void* q, const void* k, const void* v, int B, int Hq,
                             int Hkv, int S, int D, int block, PlanDev plan, int64_t cap,
                             const int32_t* sel_idx, const int32_t* sel_cnt, uint32_t* sched,
                             void* out, int32_t* status, cudaStream_t st);

// Head-pair step schedules from the CSR lists (pairs.cu). `region` (pairs_bytes()) holds the
// attention kernel's work counter in its first kCounterBytes, which the pairing kernel sets to
// 0, then the schedule (pairs_schedule(region)).
constexpr size_t kCounterBytes = 256;
inline uint32_t* pairs_schedule(uint32_t* region) {
  return region + kCounterBytes / sizeof(uint32_t);
}
cudaError_t launch_pairs(const int32_t* sel_idx, int B, int Hq, int Hkv, int nb, PlanDev plan,
                         int64_t cap, uint32_t* region, cudaStream_t st);
// Workspace bytes of the counter and the schedule for any budget of this shape.
size_t pairs_bytes(int B, int Hq, int Hkv, int nb);

// Block-sparse attention, float32 inputs on the CUDA cores (attn_f32.cu).
cudaError_t launch_attn_f32(const float* q, const float* k, const float* v, int B, int Hq,
                            int Hkv, int S, int D, int block, PlanDev plan, int64_t cap,
                            const int32_t* sel_idx, const int32_t* sel_cnt, float* out,
                            cudaStream_t st);

// Number of SMs of the current device (cached per device).
int sm_count();

// Test switch of stem_test_withhold_q (attn_sm100.cu): read by the tensor-core kernels' launchers.
extern std::atomic<int> g_withhold_q;

}  // namespace stem
