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
// that device current; that first call should come before any stream capture. The address is
// looked up again only when the device's context changes (after a cudaDeviceReset the module
// is loaded anew and the array has a new address). Every call shares the array and rewrites
// the whole plan it uses (nothing needs to start at zero), so calls whose kernels overlap on
// the GPU race on it: issue them in stream order.
//
// The plan reaches the array without a host-to-device copy: the host builds it and passes it
// by value as the parameters of a small kernel (at most two launches of 32,000 bytes), which
// writes it into the array. Launch parameters are copied when the launch is made, so nothing a
// later call does on the host can change what an earlier call's kernels read.
#include <cuda.h>
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

// One launch's share of the plan, passed by value (kernel parameters may take 32,764 bytes).
constexpr int kChunkInts = 8000;
struct PlanChunk {
  int32_t v[kChunkInts];
};
static_assert(sizeof(PlanChunk) + 2 * sizeof(int) <= 32764, "kernel parameter limit");

__global__ void write_plan_kernel(const PlanChunk c, int start, int n) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x)
    g_static_plan[start + t] = c.v[t];
}

std::mutex g_static_mu;
// per device: the array's address and the unique ID of the context it was looked up in
void* g_static_addr[kMaxDevices] = {nullptr};
unsigned long long g_static_ctx[kMaxDevices] = {0};
// host scratch of the plan (3 * STEM_MAX_NB + 1 int32 fit in two chunks), rebuilt under the
// mutex by every call; its bytes travel in the launch parameters
PlanChunk g_host_chunks[2];
static_assert(2 * kChunkInts >= 3 * STEM_MAX_NB + 1, "plan fits two chunks");

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique ID (for the life of the process) of the calling thread's current context; 0 if the
// driver cannot say.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    cudaGetLastError();
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

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
  const unsigned long long ctx = current_ctx_id();  // 0 before the runtime made one current
  if (g_static_addr[dev] == nullptr || ctx == 0 || ctx != g_static_ctx[dev]) {
    // once per device (and again after its context changed), with that device current
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_plan) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return STEM_ERR_CUDA;
    }
    g_static_addr[dev] = p;
    g_static_ctx[dev] = current_ctx_id();  // the lookup made the device's context current
  }
  // the plan in the two host chunks, as one array: k | off | order
  int32_t plan[2 * kChunkInts];
  int32_t* k = plan;
  int32_t* off = k + nb;
  int32_t* order = off + nb + 1;
  if (stem_budget(nb, rho_min, tau, k_min, k, off) != STEM_OK) return STEM_ERR_ARG;
  for (int i = 0; i < nb; ++i) order[i] = i;
  // heaviest rows first; equal budgets: later rows first (a total order: no ties)
  std::sort(order, order + nb, [&](int a, int b) { return k[a] != k[b] ? k[a] > k[b] : a > b; });
  const int n_ints = 3 * nb + 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int start = 0, c = 0; start < n_ints; start += kChunkInts, ++c) {
    const int n = std::min(kChunkInts, n_ints - start);
    std::copy(plan + start, plan + start + n, g_host_chunks[c].v);
    write_plan_kernel<<<(n + 255) / 256, 256, 0, st>>>(g_host_chunks[c], start, n);
    if (cudaGetLastError() != cudaSuccess) return STEM_ERR_CUDA;
  }
  const int32_t* dk = static_cast<const int32_t*>(g_static_addr[dev]);
  PlanDev pd{dk, dk + nb, dk + 2 * nb + 1};
  const cudaError_t e = launch_select(qbar, kbar, vnorm, B, Hq, Hkv, nb, D, pd, cap,
                                      SelMetric{}, sel_idx, sel_cnt, nullptr, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return STEM_ERR_CUDA;
  }
  return STEM_OK;
}
