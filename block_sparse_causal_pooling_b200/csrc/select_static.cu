// stem_select_static: the block selection of stem_select without any device allocation.
//
// Who needs it: some callers cannot give this library a workspace or let it call cudaMalloc,
// for example a host application that owns every device allocation through its own budgeted
// allocator, or a plugin that must not allocate behind that allocator's back. The selection
// kernel's only scratch is the budget plan it reads from global memory (k(i), the CSR offsets
// and the heavy-first row order, 3*nb+1 int32). Here that plan lives in a file-scope device
// array of fixed size, so the caller passes only inputs (pooled summaries) and outputs (CSR).
//
// The array: 64 KiB, 256-byte aligned, held by every GPU that loads the library until the
// process exits. It fits the plan for every nb this library accepts (nb <= STEM_MAX_NB = 4096
// needs 49,156 bytes); larger requests are rejected with STEM_ERR_UNSUPPORTED.
//
// The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
// that device current; that first call should come before any stream capture. Every call
// shares the array and rewrites the whole plan it uses (nothing needs to start at zero), so
// calls whose kernels overlap on the GPU race on it: issue them in stream order.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "stem.h"
#include "stem_internal.h"

namespace stem {
namespace {

constexpr size_t kStaticPlanBytes = 64 * 1024;
constexpr int kMaxDevices = 64;

__device__ __align__(256) int32_t g_static_plan[kStaticPlanBytes / sizeof(int32_t)];

std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {nullptr};
// host image of the plan, rebuilt under the mutex by every call
int32_t g_host_plan[kStaticPlanBytes / sizeof(int32_t)];

bool aligned_to(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

}  // namespace
}  // namespace stem

using namespace stem;

extern "C" int stem_select_static(const float* qbar, const float* kbar, const float* vnorm,
                                  int B, int Hq, int Hkv, int nb, int D, float rho_min,
                                  float tau, int k_min, int32_t* sel_idx, int32_t* sel_cnt,
                                  void* stream) {
  if (B < 0 || nb < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || (D != 64 && D != 128))
    return STEM_ERR_ARG;
  const size_t plan_bytes = sizeof(int32_t) * (3 * static_cast<size_t>(nb) + 1);
  if (nb > STEM_MAX_NB || plan_bytes > kStaticPlanBytes) return STEM_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * Hq * nb > 0x7fffffffLL / 4) return STEM_ERR_UNSUPPORTED;
  const int64_t cap = stem_sel_capacity(nb, rho_min, tau, k_min);
  if (cap < 0) return STEM_ERR_ARG;
  if (cap > 0x7fffffffLL) return STEM_ERR_UNSUPPORTED;
  if (B == 0 || nb == 0) return STEM_OK;
  if (!qbar || !kbar || !vnorm || !sel_idx || !sel_cnt) return STEM_ERR_ARG;
  if (!aligned_to(qbar, 16) || !aligned_to(kbar, 16) || !aligned_to(vnorm, 4) ||
      !aligned_to(sel_idx, 4) || !aligned_to(sel_cnt, 4))
    return STEM_ERR_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return STEM_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_addr[dev] == nullptr) {  // once per device, with that device current
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_plan) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return STEM_ERR_CUDA;
    }
    g_static_addr[dev] = p;
  }
  int32_t* k = g_host_plan;
  int32_t* off = k + nb;
  int32_t* order = off + nb + 1;
  if (stem_budget(nb, rho_min, tau, k_min, k, off) != STEM_OK) return STEM_ERR_ARG;
  for (int i = 0; i < nb; ++i) order[i] = i;
  // heaviest rows first; equal budgets: later rows first (a total order: no ties)
  std::sort(order, order + nb, [&](int a, int b) { return k[a] != k[b] ? k[a] > k[b] : a > b; });

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // pageable source: the call returns after the bytes are staged, so the host image is free
  // for the next call as soon as this one returns
  if (cudaMemcpyAsync(g_static_addr[dev], g_host_plan, plan_bytes, cudaMemcpyHostToDevice, st) !=
      cudaSuccess) {
    cudaGetLastError();
    return STEM_ERR_CUDA;
  }
  const int32_t* dk = static_cast<const int32_t*>(g_static_addr[dev]);
  PlanDev pd{dk, dk + nb, dk + 2 * nb + 1};
  const cudaError_t e = launch_select(qbar, kbar, vnorm, B, Hq, Hkv, nb, D, pd, cap, SelMetric{}, sel_idx,
                                      sel_cnt, nullptr, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return STEM_ERR_CUDA;
  }
  return STEM_OK;
}
