// C ABI of the Stem block-sparse causal prefill library (declared in include/stem.h).
//
// Host responsibilities: argument validation (before anything is enqueued), the Token
// Position-Decay budget in double precision ("Stem: Rethinking Causal Information Flow in
// Sparse Attention", gist.science/es "Resumen tecnico" 2.A; gist.science/it 2.A: linear
// interpolation from k_start to mu * k_start; exponential decay per the shd-paper.top "key
// design" paragraph), a per-parameter plan cache, the workspace carve-up, and the launch
// sequence pool -> select -> sparse attention.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "stem.h"
#include "stem_internal.h"

namespace stem {
namespace {

constexpr size_t kAlign = 256;
constexpr size_t kScoreCap = 128ull << 20;  // most bytes of score triangles in the workspace
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ------------------------------------------------------------------ budget

stem_method_t default_method(float rho_min, float tau, int k_min) {
  stem_method_t m;
  std::memset(&m, 0, sizeof m);
  m.schedule = STEM_SCHED_EXP;
  m.rho_min = rho_min;
  m.tau = tau;
  m.mu = 1.0f;
  m.k_min = k_min;
  m.metric = STEM_METRIC_PRODUCT;
  m.clamp = 1;
  m.vsum = STEM_VSUM_MEAN;
  m.share = STEM_SHARE_HEAD;
  return m;
}

bool method_ok(int nb, const stem_method_t& m) {
  if (nb < 0 || m.k_min < 1) return false;
  if (m.schedule == STEM_SCHED_EXP) {
    if (!(std::isfinite(m.rho_min) && m.rho_min > 0.0f && m.rho_min <= 1.0f &&
          std::isfinite(m.tau) && m.tau > 0.0f))
      return false;
  } else if (m.schedule == STEM_SCHED_LINEAR) {
    if (!(std::isfinite(m.k_start) && m.k_start > 0.0f && std::isfinite(m.mu) && m.mu > 0.0f &&
          m.mu <= 1.0f))
      return false;
  } else {
    return false;
  }
  if (m.metric == STEM_METRIC_ADDITIVE) {
    if (!(std::isfinite(m.beta) && m.beta >= 0.0f) || (m.clamp != 0 && m.clamp != 1))
      return false;
  } else if (m.metric != STEM_METRIC_PRODUCT) {
    return false;
  }
  if (m.share != STEM_SHARE_HEAD && m.share != STEM_SHARE_GROUP) return false;
  if (m.score != STEM_SCORE_POOLED && m.score != STEM_SCORE_ANTIDIAG) return false;
  return m.vsum == STEM_VSUM_MEAN || m.vsum == STEM_VSUM_MAX;
}

bool antidiag(const stem_method_t& m) { return m.score == STEM_SCORE_ANTIDIAG; }

// The anti-diagonal estimator's shape rules: a power-of-two stride dividing the block (at most
// 32 groups per block) and the sequence; bfloat16 inputs.
int check_antidiag(int S, int block, int dtype, int stride) {
  if (stride < 1 || (stride & (stride - 1)) || block % stride || block / stride > 32 ||
      S % stride)
    return STEM_ERR_ARG;
  if (dtype != STEM_BF16) return STEM_ERR_UNSUPPORTED;
  return STEM_OK;
}

// Exponential: k(i) = min(i+1, max(k_min, ceil(rho(i) (i+1)))), rho(i) = rho_min + (1-rho_min)
// e^{-i/tau}. Linear: k(i) = min(i+1, max(k_min, ceil(k_start (1 - (1-mu) i/(nb-1))))), the
// interpolation from k_start at the first query block to mu * k_start at the last. Block 0
// alone at i = 0, at least the sink and the diagonal for i >= 1.
int budget_k(int i, int nb, const stem_method_t& m) {
  if (i == 0) return 1;
  double want;
  if (m.schedule == STEM_SCHED_LINEAR) {
    const double t = nb > 1 ? static_cast<double>(i) / static_cast<double>(nb - 1) : 0.0;
    const double k_lin =
        static_cast<double>(m.k_start) * (1.0 - (1.0 - static_cast<double>(m.mu)) * t);
    want = std::ceil(k_lin);
  } else {
    const double rho_min = m.rho_min;
    const double rho =
        rho_min + (1.0 - rho_min) * std::exp(-static_cast<double>(i) / static_cast<double>(m.tau));
    want = std::ceil(rho * static_cast<double>(i + 1));
  }
  double kk = std::max(want, static_cast<double>(m.k_min));
  kk = std::min(kk, static_cast<double>(i + 1));
  return std::max(2, static_cast<int>(kk));
}

struct Plan {
  int nb = 0;
  int64_t cap = 0;
  int32_t* host = nullptr;  // pinned: k[nb] | off[nb+1] | order[nb]
  size_t bytes = 0;
};

using PlanKey = std::tuple<int, int, uint32_t, uint32_t, int>;
std::mutex g_plan_mu;
std::map<PlanKey, Plan> g_plans;

uint32_t fbits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

size_t plan_bytes(int nb) { return align_up(sizeof(int32_t) * (3 * static_cast<size_t>(nb) + 1)); }

// Returns the cached plan (building it on first use), or nullptr on a pinned-allocation failure.
const Plan* get_plan(int nb, const stem_method_t& m) {
  std::lock_guard<std::mutex> lock(g_plan_mu);
  const bool lin = m.schedule == STEM_SCHED_LINEAR;
  const PlanKey key{nb, m.schedule, fbits(lin ? m.k_start : m.rho_min), fbits(lin ? m.mu : m.tau),
                    m.k_min};
  auto it = g_plans.find(key);
  if (it != g_plans.end()) return &it->second;
  Plan p;
  p.nb = nb;
  p.bytes = plan_bytes(nb);
  if (cudaMallocHost(reinterpret_cast<void**>(&p.host), p.bytes) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  std::memset(p.host, 0, p.bytes);
  int32_t* k = p.host;
  int32_t* off = k + nb;
  int32_t* order = off + nb + 1;
  int64_t tot = 0;
  for (int i = 0; i < nb; ++i) {
    k[i] = budget_k(i, nb, m);
    off[i] = static_cast<int32_t>(tot);
    tot += k[i];
  }
  off[nb] = static_cast<int32_t>(tot);
  p.cap = tot;
  for (int i = 0; i < nb; ++i) order[i] = i;
  // heaviest query blocks first; equal budgets: later blocks first
  std::stable_sort(order, order + nb, [&](int a, int b) {
    return k[a] != k[b] ? k[a] > k[b] : a > b;
  });
  return &g_plans.emplace(key, p).first->second;
}

// ------------------------------------------------------------------ workspace layout

struct Layout {
  size_t status = 0, plan = 0, sched = 0, sched_end = 0, qbar = 0, kbar = 0, vnorm = 0,
         adp = 0, ads = 0, total = 0;
};

// m (with S and block) adds the anti-diagonal estimator's regions when it asks for them.
Layout layout(int B, int Hq, int Hkv, int nb, int D, const stem_method_t* m = nullptr, int S = 0,
              int block = 0) {
  Layout L;
  size_t o = 0;
  L.status = o;
  o += kAlign;
  L.plan = o;
  o += plan_bytes(nb);
  // The head-pair schedule (attention stage) and the selection's score triangles (selection
  // stage, before it) share one region: every head's triangle up to 128 MB, at least the
  // schedule's size (the selection then runs over chunks of heads).
  L.sched = o;
  const size_t tri = sizeof(float) * static_cast<size_t>(nb) * (nb + 1) / 2;
  const size_t scores = std::min(tri * static_cast<size_t>(B) * Hq, kScoreCap);
  o += align_up(std::max(pairs_bytes(B, Hq, Hkv, nb), scores));
  L.sched_end = o;
  L.qbar = o;
  o += align_up(sizeof(float) * static_cast<size_t>(B) * Hq * nb * D);
  L.kbar = o;
  o += align_up(sizeof(float) * static_cast<size_t>(B) * Hkv * nb * D);
  L.vnorm = o;
  o += align_up(sizeof(float) * static_cast<size_t>(B) * Hkv * nb);
  if (m != nullptr && antidiag(*m)) {
    L.adp = o;  // p [B*Hq][nb*(nb+1)/2]
    o += align_up(sizeof(float) * static_cast<size_t>(B) * Hq * nb * (nb + 1) / 2);
    L.ads = o;  // estimator scratch
    o += align_up(sizeof(float) * antidiag_scratch_floats(B, Hq, S, block, m->stride));
  }
  L.total = o;
  return L;
}

// ------------------------------------------------------------------ validation

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int nblocks(int S, int block) { return (S + block - 1) / block; }

int check_shape(int B, int Hq, int Hkv, int S, int D, int block, int dtype) {
  if (B < 0 || S < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return STEM_ERR_ARG;
  if (D != 64 && D != 128) return STEM_ERR_ARG;
  if (block != 64 && block != 128) return STEM_ERR_ARG;
  if (dtype != STEM_BF16 && dtype != STEM_F32) return STEM_ERR_ARG;
  // element counts must fit comfortably in int64 and grid sizes in int32; a partial last block
  // (S % block != 0) is a block of its own
  const int64_t nb = nblocks(S, block);
  if (static_cast<int64_t>(B) * Hq * nb > 0x7fffffffLL / 4) return STEM_ERR_UNSUPPORTED;
  if (nb > STEM_MAX_NB) return STEM_ERR_UNSUPPORTED;
  return STEM_OK;
}

bool is_empty(int B, int S) { return B == 0 || S == 0; }

int64_t capacity(int nb, const stem_method_t& m) {
  int64_t tot = 0;
  for (int i = 0; i < nb; ++i) tot += budget_k(i, nb, m);
  return tot;
}

int check_params(int nb, const stem_method_t& m) {
  if (!method_ok(nb, m)) return STEM_ERR_ARG;
  // off[] is int32: the capacity must fit
  const int64_t cap = capacity(nb, m);
  if (cap > 0x7fffffffLL) return STEM_ERR_UNSUPPORTED;
  if (m.share == STEM_SHARE_GROUP && nb > kGroupMaxNb) return STEM_ERR_UNSUPPORTED;
  return STEM_OK;
}

SelMetric sel_metric(const stem_method_t& m) {
  SelMetric s;
  s.additive = m.metric == STEM_METRIC_ADDITIVE;
  s.beta = m.beta;
  s.clamp = m.clamp != 0;
  s.group = m.share == STEM_SHARE_GROUP;
  return s;
}

int cuda_err(cudaError_t e) {
  if (e == cudaSuccess) return STEM_OK;
  cudaGetLastError();  // clear a sticky launch error in this thread's runtime state
  return STEM_ERR_CUDA;
}

int upload_plan(const Plan* p, void* ws, const Layout& L, cudaStream_t st, PlanDev* dev) {
  auto* base = static_cast<unsigned char*>(ws) + L.plan;
  const cudaError_t e = cudaMemcpyAsync(base, p->host, p->bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_err(e);
  const auto* k = reinterpret_cast<const int32_t*>(base);
  dev->k = k;
  dev->off = k + p->nb;
  dev->order = k + 2 * p->nb + 1;
  return STEM_OK;
}

int elem_size(int dtype) { return dtype == STEM_BF16 ? 2 : 4; }

// ------------------------------------------------------------------ the path

stem_method_t args_method(const stem_args_t* a) {
  return a->method ? *a->method : default_method(a->rho_min, a->tau, a->k_min);
}

int enqueue_kernels(const stem_args_t* a, const stem_method_t& m, int nb, int64_t cap,
                    PlanDev pd, cudaStream_t st);

int run_prefill(const stem_args_t* a, cudaStream_t st) {
  if (a == nullptr) return STEM_ERR_ARG;
  int rc = check_shape(a->B, a->Hq, a->Hkv, a->S, a->D, a->block, a->dtype);
  if (rc != STEM_OK) return rc;
  const int nb = nblocks(a->S, a->block);
  const stem_method_t m = args_method(a);
  rc = check_params(nb, m);
  if (rc != STEM_OK) return rc;
  if (antidiag(m) && (rc = check_antidiag(a->S, a->block, a->dtype, m.stride)) != STEM_OK)
    return rc;
  if (is_empty(a->B, a->S)) return STEM_OK;
  if (!a->q || !a->k || !a->v || !a->out || !a->sel_idx || !a->sel_cnt) return STEM_ERR_ARG;
  if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->out, 16) ||
      !aligned(a->sel_idx, 4) || !aligned(a->sel_cnt, 4) || !aligned(a->status, 4))
    return STEM_ERR_ARG;
  const Layout L = layout(a->B, a->Hq, a->Hkv, nb, a->D, &m, a->S, a->block);
  if (a->workspace == nullptr || !aligned(a->workspace, kAlign) || a->workspace_bytes < L.total)
    return STEM_ERR_WORKSPACE;
  const Plan* plan = get_plan(nb, m);
  if (plan == nullptr) return STEM_ERR_CUDA;

  auto* ws = static_cast<unsigned char*>(a->workspace);
  if (a->status) {
    rc = cuda_err(cudaMemsetAsync(a->status, 0, sizeof(int32_t), st));
    if (rc != STEM_OK) return rc;
  }
  PlanDev pd;
  rc = upload_plan(plan, ws, L, st, &pd);
  if (rc != STEM_OK) return rc;
  return enqueue_kernels(a, m, nb, plan->cap, pd, st);
}

// The three stages of a validated call whose plan is already on the device (pd) and whose status
// word, if any, is already cleared: kernels (and the optional timing events) only, no copies.
int enqueue_kernels(const stem_args_t* a, const stem_method_t& m, int nb, int64_t cap,
                    PlanDev pd, cudaStream_t st) {
  int rc = STEM_OK;
  const Layout L = layout(a->B, a->Hq, a->Hkv, nb, a->D, &m, a->S, a->block);
  auto* ws = static_cast<unsigned char*>(a->workspace);
  float* qbar = reinterpret_cast<float*>(ws + L.qbar);
  float* kbar = reinterpret_cast<float*>(ws + L.kbar);
  float* vnorm = reinterpret_cast<float*>(ws + L.vnorm);
  auto mark = [&](int n) -> int {
    if (a->events == nullptr || a->events[n] == nullptr) return STEM_OK;
    return cuda_err(cudaEventRecord(static_cast<cudaEvent_t>(a->events[n]), st));
  };
  if ((rc = mark(0)) != STEM_OK) return rc;
  rc = cuda_err(launch_pool(a->q, a->k, a->v, a->dtype, a->B, a->Hq, a->Hkv, a->S, a->D,
                            a->block, m.vsum == STEM_VSUM_MAX, qbar, kbar, vnorm, st));
  if (rc != STEM_OK) return rc;
  if ((rc = mark(1)) != STEM_OK) return rc;
  if (antidiag(m)) {
    float* p = reinterpret_cast<float*>(ws + L.adp);
    rc = cuda_err(launch_antidiag(a->q, a->k, a->B, a->Hq, a->Hkv, a->S, a->D, a->block,
                                  m.stride, p, reinterpret_cast<float*>(ws + L.ads), a->status,
                                  st));
    if (rc != STEM_OK) return rc;
    rc = cuda_err(launch_select_p(p, vnorm, a->B, a->Hq, a->Hkv, nb, pd, cap, sel_metric(m),
                                  a->sel_idx, a->sel_cnt, nullptr, st));
  } else {
    // the score triangles go to the schedule region, which the attention stage fills later
    rc = cuda_err(launch_select(qbar, kbar, vnorm, a->B, a->Hq, a->Hkv, nb, a->D, pd, cap,
                                sel_metric(m), a->sel_idx, a->sel_cnt, nullptr, st,
                                reinterpret_cast<float*>(ws + L.sched), L.sched_end - L.sched));
  }
  if (rc != STEM_OK) return rc;
  if ((rc = mark(2)) != STEM_OK) return rc;
  if (a->dtype == STEM_BF16) {
    rc = cuda_err(launch_attn_bf16(a->q, a->k, a->v, a->B, a->Hq, a->Hkv, a->S, a->D, a->block,
                                   pd, cap, a->sel_idx, a->sel_cnt,
                                   reinterpret_cast<uint32_t*>(ws + L.sched), a->out, a->status,
                                   st));
  } else {
    rc = cuda_err(launch_attn_f32(static_cast<const float*>(a->q),
                                  static_cast<const float*>(a->k),
                                  static_cast<const float*>(a->v), a->B, a->Hq, a->Hkv, a->S,
                                  a->D, a->block, pd, cap, a->sel_idx, a->sel_cnt,
                                  static_cast<float*>(a->out), st));
  }
  if (rc != STEM_OK) return rc;
  return mark(3);
}

// Internal grow-only device buffers, one per (device, user): slot 0 is stem_prefill's
// workspace, slot 1 the arena of stem_prefill_host.
struct DeviceScratch {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_scratch_mu;
std::map<std::pair<int, int>, DeviceScratch> g_scratch;

int get_scratch(size_t need, void** out, int slot) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  DeviceScratch& s = g_scratch[{dev, slot}];
  if (s.bytes < need) {
    if (s.ptr) {
      // the previous buffer may still be read by queued work
      e = cudaDeviceSynchronize();
      if (e != cudaSuccess) return cuda_err(e);
      cudaFree(s.ptr);
      s.ptr = nullptr;
      s.bytes = 0;
    }
    e = cudaMalloc(&s.ptr, need);
    if (e != cudaSuccess) return cuda_err(e);
    s.bytes = need;
  }
  *out = s.ptr;
  return STEM_OK;
}

}  // namespace

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace stem

using namespace stem;

extern "C" {

int stem_budget_m(int nb, const stem_method_t* m, int32_t* k_out, int32_t* off_out) {
  if (m == nullptr || !method_ok(nb, *m)) return STEM_ERR_ARG;
  int64_t tot = 0;
  for (int i = 0; i < nb; ++i) {
    const int k = budget_k(i, nb, *m);
    if (off_out) off_out[i] = static_cast<int32_t>(tot);
    if (k_out) k_out[i] = k;
    tot += k;
    if (tot > 0x7fffffffLL) return STEM_ERR_ARG;
  }
  if (off_out) off_out[nb] = static_cast<int32_t>(tot);
  return STEM_OK;
}

int stem_budget(int nb, float rho_min, float tau, int k_min, int32_t* k_out, int32_t* off_out) {
  const stem_method_t m = default_method(rho_min, tau, k_min);
  return stem_budget_m(nb, &m, k_out, off_out);
}

int64_t stem_sel_capacity_m(int nb, const stem_method_t* m) {
  if (m == nullptr || !method_ok(nb, *m)) return STEM_ERR_ARG;
  return capacity(nb, *m);
}

int64_t stem_sel_capacity(int nb, float rho_min, float tau, int k_min) {
  const stem_method_t m = default_method(rho_min, tau, k_min);
  return stem_sel_capacity_m(nb, &m);
}

size_t stem_workspace_size(int B, int Hq, int Hkv, int S, int D, int block) {
  if (check_shape(B, Hq, Hkv, S, D, block, STEM_BF16) != STEM_OK) return 0;
  if (is_empty(B, S)) return 0;
  return layout(B, Hq, Hkv, nblocks(S, block), D).total;
}

size_t stem_workspace_size_m(int B, int Hq, int Hkv, int S, int D, int block,
                             const stem_method_t* m) {
  if (m == nullptr) return 0;
  if (check_shape(B, Hq, Hkv, S, D, block, STEM_BF16) != STEM_OK) return 0;
  const int nb = nblocks(S, block);
  if (!method_ok(nb, *m)) return 0;
  if (antidiag(*m) && check_antidiag(S, block, STEM_BF16, m->stride) != STEM_OK) return 0;
  if (is_empty(B, S)) return 0;
  return layout(B, Hq, Hkv, nb, D, m, S, block).total;
}

const char* stem_strerror(int code) {
  switch (code) {
    case STEM_OK: return "success";
    case STEM_ERR_ARG: return "invalid argument (pointer, shape or budget parameter)";
    case STEM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case STEM_ERR_CUDA: return "CUDA error (launch failure, no device or no sm_100a support)";
    case STEM_ERR_TIMEOUT: return "a device-side wait exceeded its bound";
    case STEM_ERR_UNSUPPORTED: return "request exceeds this build's limits";
    default: return "unknown error code";
  }
}

int stem_prefill_ex(const stem_args_t* a, void* stream) {
  return run_prefill(a, static_cast<cudaStream_t>(stream));
}

int stem_prefill(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int S,
                 int D, int block, float rho_min, float tau, int k_min, void* out,
                 int32_t* sel_idx, int32_t* sel_cnt) {
  stem_args_t a;
  std::memset(&a, 0, sizeof a);
  a.q = q;
  a.k = k;
  a.v = v;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.S = S;
  a.D = D;
  a.block = block;
  a.rho_min = rho_min;
  a.tau = tau;
  a.k_min = k_min;
  a.dtype = STEM_BF16;
  a.out = out;
  a.sel_idx = sel_idx;
  a.sel_cnt = sel_cnt;
  int rc = check_shape(B, Hq, Hkv, S, D, block, STEM_BF16);
  if (rc != STEM_OK) return rc;
  if (is_empty(B, S)) return run_prefill(&a, nullptr);
  rc = check_params(nblocks(S, block), default_method(rho_min, tau, k_min));
  if (rc != STEM_OK) return rc;
  a.workspace_bytes = stem_workspace_size(B, Hq, Hkv, S, D, block);
  rc = get_scratch(a.workspace_bytes, &a.workspace, 0);
  if (rc != STEM_OK) return rc;
  return run_prefill(&a, nullptr);
}

// Host buffers: the problem splits into independent pieces, each a pair of query heads of one
// (batch b, kv-head group g) with the group's K and V (the whole group when the selection is
// shared by the group). Piece c's inputs go up on one stream (K and V with the group's first
// piece), its kernels run on a second once they have arrived, and its results come down on a
// third once its kernels are done, so the copies of one piece overlap the kernels of the others
// and the two PCIe directions overlap each other; small pieces keep the pipeline's fill (the
// first piece's upload) and drain (the last piece's kernels and download) short. Each head's
// results are those of the device-buffer path: selection and attention are per head, and the
// pieces keep the attention kernel's head pairs.
int stem_prefill_host(const stem_args_t* h) {
  if (h == nullptr) return STEM_ERR_ARG;
  int rc = check_shape(h->B, h->Hq, h->Hkv, h->S, h->D, h->block, h->dtype);
  if (rc != STEM_OK) return rc;
  const int nb = nblocks(h->S, h->block);
  const stem_method_t m = args_method(h);
  rc = check_params(nb, m);
  if (rc != STEM_OK) return rc;
  if (antidiag(m) && (rc = check_antidiag(h->S, h->block, h->dtype, m.stride)) != STEM_OK)
    return rc;
  if (is_empty(h->B, h->S)) return STEM_OK;
  if (!h->q || !h->k || !h->v || !h->out || !h->sel_idx || !h->sel_cnt) return STEM_ERR_ARG;
  const int G = h->Hq / h->Hkv;
  const int hp = (m.share == STEM_SHARE_GROUP || G < 2) ? G : 2;  // query heads per piece
  const int per_group = (G + hp - 1) / hp;
  const int np = h->B * h->Hkv * per_group;  // pieces
  const size_t es = elem_size(h->dtype);
  const int64_t cap = capacity(nb, m);
  const size_t hb = es * static_cast<size_t>(h->S) * h->D;  // one head of q, k, v or out
  const size_t sih = sizeof(int32_t) * static_cast<size_t>(cap);  // one head's CSR
  const size_t sch = sizeof(int32_t) * static_cast<size_t>(nb);   // one head's counts
  const size_t nq = static_cast<size_t>(h->B) * h->Hq, nkv = static_cast<size_t>(h->B) * h->Hkv;
  const Layout Lc = layout(1, hp, 1, nb, h->D, &m, h->S, h->block);  // one piece's workspace
  const Plan* plan = get_plan(nb, m);
  if (plan == nullptr) return STEM_ERR_CUDA;
  // device arena: piece status words | the plan | piece workspaces | q | k | v | out | sel_idx |
  // sel_cnt (the tensors in their host layout). The plan and the cleared status words go up
  // first on the input stream: a copy issued on the compute stream would wait in the copy
  // engine behind every piece's inputs.
  const size_t o_plan = align_up(sizeof(int32_t) * np);
  const size_t o_ws = o_plan + plan_bytes(nb);
  const size_t wsb = align_up(Lc.total);
  const size_t o_q = o_ws + wsb * np, o_k = o_q + align_up(hb * nq),
               o_v = o_k + align_up(hb * nkv), o_out = o_v + align_up(hb * nkv),
               o_si = o_out + align_up(hb * nq), o_sc = o_si + align_up(sih * nq),
               total = o_sc + align_up(sch * nq);
  static std::mutex host_mu;  // host-buffer calls share one arena: one at a time
  std::lock_guard<std::mutex> lock(host_mu);
  void* arena = nullptr;
  rc = get_scratch(total, &arena, 1);
  if (rc != STEM_OK) return rc;
  auto* base = static_cast<unsigned char*>(arena);
  cudaStream_t sin = nullptr, srun = nullptr, sout = nullptr;
  std::vector<cudaEvent_t> ev(2 * static_cast<size_t>(np), nullptr);
  cudaError_t e = cudaSuccess;
  auto cleanup = [&]() {
    for (cudaStream_t s : {sin, srun, sout})
      if (s) cudaStreamSynchronize(s);
    for (cudaEvent_t x : ev)
      if (x) cudaEventDestroy(x);
    for (cudaStream_t s : {sin, srun, sout})
      if (s) cudaStreamDestroy(s);
  };
  auto up = [&](size_t off, const void* src, size_t bytes) {
    return cudaMemcpyAsync(base + off, src, bytes, cudaMemcpyHostToDevice, sin);
  };
  auto down = [&](void* dst, size_t off, size_t bytes) {
    return cudaMemcpyAsync(dst, base + off, bytes, cudaMemcpyDeviceToHost, sout);
  };
  do {
    if ((e = cudaStreamCreateWithFlags(&sin, cudaStreamNonBlocking))) break;
    if ((e = cudaStreamCreateWithFlags(&srun, cudaStreamNonBlocking))) break;
    if ((e = cudaStreamCreateWithFlags(&sout, cudaStreamNonBlocking))) break;
    for (auto& x : ev)
      if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming))) break;
    if (e) break;
    if ((e = cudaMemsetAsync(base, 0, sizeof(int32_t) * np, sin))) break;
    if ((e = cudaMemcpyAsync(base + o_plan, plan->host, plan->bytes, cudaMemcpyHostToDevice, sin)))
      break;
    PlanDev pd;
    pd.k = reinterpret_cast<const int32_t*>(base + o_plan);
    pd.off = pd.k + nb;
    pd.order = pd.k + 2 * nb + 1;
    for (int c = 0; c < np && rc == STEM_OK && e == cudaSuccess; ++c) {
      const int bg = c / per_group, pi = c % per_group;
      const int nh = std::min(hp, G - pi * hp);
      const size_t qh0 = static_cast<size_t>(bg) * G + static_cast<size_t>(pi) * hp;  // 1st head
      if (pi == 0) {  // the group's K and V go up with its first piece
        if ((e = up(o_k + hb * bg, static_cast<const unsigned char*>(h->k) + hb * bg, hb))) break;
        if ((e = up(o_v + hb * bg, static_cast<const unsigned char*>(h->v) + hb * bg, hb))) break;
      }
      if ((e = up(o_q + hb * qh0, static_cast<const unsigned char*>(h->q) + hb * qh0, hb * nh)))
        break;
      stem_args_t d = *h;
      d.B = 1;
      d.Hq = nh;
      d.Hkv = 1;
      d.q = base + o_q + hb * qh0;
      d.k = base + o_k + hb * bg;
      d.v = base + o_v + hb * bg;
      d.out = base + o_out + hb * qh0;
      d.sel_idx = reinterpret_cast<int32_t*>(base + o_si + sih * qh0);
      d.sel_cnt = reinterpret_cast<int32_t*>(base + o_sc + sch * qh0);
      d.workspace = base + o_ws + wsb * c;
      d.workspace_bytes = Lc.total;
      d.status = reinterpret_cast<int32_t*>(base) + c;
      d.events = nullptr;
      if ((e = cudaEventRecord(ev[2 * c], sin))) break;
      if ((e = cudaStreamWaitEvent(srun, ev[2 * c], 0))) break;
      if ((rc = enqueue_kernels(&d, m, nb, plan->cap, pd, srun)) != STEM_OK) break;
      if ((e = cudaEventRecord(ev[2 * c + 1], srun))) break;
      if ((e = cudaStreamWaitEvent(sout, ev[2 * c + 1], 0))) break;
      if ((e = down(static_cast<unsigned char*>(h->out) + hb * qh0, o_out + hb * qh0, hb * nh)))
        break;
      if ((e = down(reinterpret_cast<unsigned char*>(h->sel_idx) + sih * qh0, o_si + sih * qh0,
                    sih * nh)))
        break;
      if ((e = down(reinterpret_cast<unsigned char*>(h->sel_cnt) + sch * qh0, o_sc + sch * qh0,
                    sch * nh)))
        break;
    }
  } while (false);
  cleanup();
  if (rc != STEM_OK) return rc;
  if (e != cudaSuccess) return cuda_err(e);
  std::vector<int32_t> status(np, 0);
  e = cudaMemcpy(status.data(), base, sizeof(int32_t) * np, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_err(e);
  for (int32_t x : status)
    if (x < 0) return x;
  return STEM_OK;
}

int stem_pool_m(const void* q, const void* k, const void* v, int dtype, int B, int Hq, int Hkv,
                int S, int D, int block, const stem_method_t* m, float* qbar, float* kbar,
                float* vnorm, void* stream) {
  if (m == nullptr || (m->vsum != STEM_VSUM_MEAN && m->vsum != STEM_VSUM_MAX)) return STEM_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, S, D, block, dtype);
  if (rc != STEM_OK) return rc;
  if (is_empty(B, S)) return STEM_OK;
  if (!q || !k || !v || !qbar || !kbar || !vnorm) return STEM_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(qbar, 16) ||
      !aligned(kbar, 16) || !aligned(vnorm, 4))
    return STEM_ERR_ARG;
  return cuda_err(launch_pool(q, k, v, dtype, B, Hq, Hkv, S, D, block, m->vsum == STEM_VSUM_MAX,
                              qbar, kbar, vnorm, static_cast<cudaStream_t>(stream)));
}

int stem_pool(const void* q, const void* k, const void* v, int dtype, int B, int Hq, int Hkv,
              int S, int D, int block, float* qbar, float* kbar, float* vnorm, void* stream) {
  const stem_method_t m = default_method(1.0f, 1.0f, 1);
  return stem_pool_m(q, k, v, dtype, B, Hq, Hkv, S, D, block, &m, qbar, kbar, vnorm, stream);
}

int stem_select_m(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                  int Hkv, int nb, int D, const stem_method_t* m, int32_t* sel_idx,
                  int32_t* sel_cnt, float* m_out, void* workspace, size_t workspace_bytes,
                  void* stream) {
  if (nb < 0 || m == nullptr) return STEM_ERR_ARG;
  if (nb > STEM_MAX_NB) return STEM_ERR_UNSUPPORTED;
  // the selection sees blocks only: validate as a shape with block 64
  int rc = check_shape(B, Hq, Hkv, nb * 64, D, 64, STEM_F32);
  if (rc != STEM_OK) return rc;
  rc = check_params(nb, *m);
  if (rc != STEM_OK) return rc;
  if (is_empty(B, nb)) return STEM_OK;
  if (!qbar || !kbar || !vnorm || !sel_idx || !sel_cnt) return STEM_ERR_ARG;
  if (!aligned(qbar, 16) || !aligned(kbar, 16) || !aligned(vnorm, 4) || !aligned(sel_idx, 4) ||
      !aligned(sel_cnt, 4) || !aligned(m_out, 4))
    return STEM_ERR_ARG;
  const Layout L = layout(B, Hq, Hkv, nb, D);
  if (workspace == nullptr || !aligned(workspace, kAlign) || workspace_bytes < L.plan + plan_bytes(nb))
    return STEM_ERR_WORKSPACE;
  const Plan* plan = get_plan(nb, *m);
  if (plan == nullptr) return STEM_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  PlanDev pd;
  rc = upload_plan(plan, workspace, L, st, &pd);
  if (rc != STEM_OK) return rc;
  // a workspace of stem_workspace_size has room for score triangles after the plan; a smaller
  // one (the plan only) runs the fused kernel, with the same selection
  float* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (workspace_bytes >= L.sched_end) {
    scratch = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + L.sched);
    scratch_bytes = L.sched_end - L.sched;
  }
  return cuda_err(launch_select(qbar, kbar, vnorm, B, Hq, Hkv, nb, D, pd, plan->cap,
                                sel_metric(*m), sel_idx, sel_cnt, m_out, st, scratch,
                                scratch_bytes));
}

int stem_antidiag_m(const void* q, const void* k, int dtype, int B, int Hq, int Hkv, int S, int D,
                    int block, const stem_method_t* m, float* p, void* workspace,
                    size_t workspace_bytes, int32_t* status, void* stream) {
  if (m == nullptr) return STEM_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, S, D, block, dtype);
  if (rc != STEM_OK) return rc;
  rc = check_antidiag(S, block, dtype, m->stride);
  if (rc != STEM_OK) return rc;
  if (is_empty(B, S)) return STEM_OK;
  if (!q || !k || !p) return STEM_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(p, 4) || !aligned(status, 4))
    return STEM_ERR_ARG;
  stem_method_t ma = *m;
  ma.score = STEM_SCORE_ANTIDIAG;
  const int nb = nblocks(S, block);
  const Layout L = layout(B, Hq, Hkv, nb, D, &ma, S, block);
  if (workspace == nullptr || !aligned(workspace, kAlign) || workspace_bytes < L.total)
    return STEM_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (status) {
    rc = cuda_err(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    if (rc != STEM_OK) return rc;
  }
  return cuda_err(launch_antidiag(q, k, B, Hq, Hkv, S, D, block, m->stride, p,
                                  reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) +
                                                           L.ads),
                                  status, st));
}

int stem_select_p_m(const float* p, const float* vnorm, int B, int Hq, int Hkv, int nb,
                    const stem_method_t* m, int32_t* sel_idx, int32_t* sel_cnt, float* m_out,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (nb < 0 || m == nullptr) return STEM_ERR_ARG;
  if (nb > STEM_MAX_NB) return STEM_ERR_UNSUPPORTED;
  int rc = check_shape(B, Hq, Hkv, nb * 64, 64, 64, STEM_F32);  // the selection sees blocks only
  if (rc != STEM_OK) return rc;
  rc = check_params(nb, *m);
  if (rc != STEM_OK) return rc;
  if (is_empty(B, nb)) return STEM_OK;
  if (!p || !vnorm || !sel_idx || !sel_cnt) return STEM_ERR_ARG;
  if (!aligned(p, 4) || !aligned(vnorm, 4) || !aligned(sel_idx, 4) || !aligned(sel_cnt, 4) ||
      !aligned(m_out, 4))
    return STEM_ERR_ARG;
  const Layout L = layout(B, Hq, Hkv, nb, 64);
  if (workspace == nullptr || !aligned(workspace, kAlign) || workspace_bytes < L.plan + plan_bytes(nb))
    return STEM_ERR_WORKSPACE;
  const Plan* plan = get_plan(nb, *m);
  if (plan == nullptr) return STEM_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  PlanDev pd;
  rc = upload_plan(plan, workspace, L, st, &pd);
  if (rc != STEM_OK) return rc;
  return cuda_err(launch_select_p(p, vnorm, B, Hq, Hkv, nb, pd, plan->cap, sel_metric(*m), sel_idx,
                                  sel_cnt, m_out, st));
}

int stem_select(const float* qbar, const float* kbar, const float* vnorm, int B, int Hq,
                int Hkv, int nb, int D, float rho_min, float tau, int k_min, int32_t* sel_idx,
                int32_t* sel_cnt, float* m_out, void* workspace, size_t workspace_bytes,
                void* stream) {
  const stem_method_t m = default_method(rho_min, tau, k_min);
  return stem_select_m(qbar, kbar, vnorm, B, Hq, Hkv, nb, D, &m, sel_idx, sel_cnt, m_out,
                       workspace, workspace_bytes, stream);
}

int stem_sparse_attn_m(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                       int Hkv, int S, int D, int block, const stem_method_t* m,
                       const int32_t* sel_idx, const int32_t* sel_cnt, void* out,
                       void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  if (m == nullptr) return STEM_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, S, D, block, dtype);
  if (rc != STEM_OK) return rc;
  const int nb = nblocks(S, block);
  rc = check_params(nb, *m);
  if (rc != STEM_OK) return rc;
  if (is_empty(B, S)) return STEM_OK;
  if (!q || !k || !v || !out || !sel_idx || !sel_cnt) return STEM_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(sel_idx, 4) || !aligned(sel_cnt, 4) || !aligned(status, 4))
    return STEM_ERR_ARG;
  const Layout L = layout(B, Hq, Hkv, nb, D);
  if (workspace == nullptr || !aligned(workspace, kAlign) || workspace_bytes < L.sched_end)
    return STEM_ERR_WORKSPACE;
  const Plan* plan = get_plan(nb, *m);
  if (plan == nullptr) return STEM_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (status) {
    rc = cuda_err(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    if (rc != STEM_OK) return rc;
  }
  PlanDev pd;
  rc = upload_plan(plan, workspace, L, st, &pd);
  if (rc != STEM_OK) return rc;
  if (dtype == STEM_BF16)
    return cuda_err(launch_attn_bf16(q, k, v, B, Hq, Hkv, S, D, block, pd, plan->cap, sel_idx,
                                     sel_cnt,
                                     reinterpret_cast<uint32_t*>(
                                         static_cast<unsigned char*>(workspace) + L.sched),
                                     out, status, st));
  return cuda_err(launch_attn_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                  static_cast<const float*>(v), B, Hq, Hkv, S, D, block, pd,
                                  plan->cap, sel_idx, sel_cnt, static_cast<float*>(out), st));
}

int stem_sparse_attn(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                     int Hkv, int S, int D, int block, float rho_min, float tau, int k_min,
                     const int32_t* sel_idx, const int32_t* sel_cnt, void* out, void* workspace,
                     size_t workspace_bytes, int32_t* status, void* stream) {
  const stem_method_t m = default_method(rho_min, tau, k_min);
  return stem_sparse_attn_m(q, k, v, dtype, B, Hq, Hkv, S, D, block, &m, sel_idx, sel_cnt, out,
                            workspace, workspace_bytes, status, stream);
}

// ------------------------------------------------------------------ variable-length batches

static int check_cu(int nseq, const int32_t* cu) {
  if (nseq < 0 || cu == nullptr || cu[0] != 0) return STEM_ERR_ARG;
  for (int s = 0; s < nseq; ++s)
    if (cu[s + 1] < cu[s]) return STEM_ERR_ARG;
  return STEM_OK;
}

int64_t stem_varlen_sel_capacity(int nseq, const int32_t* cu, int block, const stem_method_t* m) {
  if (m == nullptr || (block != 64 && block != 128)) return STEM_ERR_ARG;
  if (check_cu(nseq, cu) != STEM_OK) return STEM_ERR_ARG;
  int64_t total = 0;
  for (int s = 0; s < nseq; ++s) {
    const int nb = nblocks(cu[s + 1] - cu[s], block);
    if (!method_ok(nb, *m)) return STEM_ERR_ARG;
    total += capacity(nb, *m);
  }
  return total;
}

size_t stem_varlen_workspace_size_m(int nseq, const int32_t* cu, int Hq, int Hkv, int D,
                                    int block, const stem_method_t* m) {
  if (check_cu(nseq, cu) != STEM_OK) return 0;
  size_t most = 0;
  for (int s = 0; s < nseq; ++s) {
    const int S = cu[s + 1] - cu[s];
    if (S == 0) continue;
    const size_t n = m ? stem_workspace_size_m(1, Hq, Hkv, S, D, block, m)
                       : stem_workspace_size(1, Hq, Hkv, S, D, block);
    if (n == 0) return 0;
    most = std::max(most, n);
  }
  return most;
}

size_t stem_varlen_workspace_size(int nseq, const int32_t* cu, int Hq, int Hkv, int D,
                                  int block) {
  return stem_varlen_workspace_size_m(nseq, cu, Hq, Hkv, D, block, nullptr);
}

int stem_prefill_varlen(const stem_varlen_args_t* a, void* stream) {
  if (a == nullptr || a->method == nullptr) return STEM_ERR_ARG;
  int rc = check_cu(a->nseq, a->cu_seqlens);
  if (rc != STEM_OK) return rc;
  const stem_method_t& m = *a->method;
  const int32_t* cu = a->cu_seqlens;
  // validate every sequence before anything is enqueued
  size_t need = 0;
  for (int s = 0; s < a->nseq; ++s) {
    const int S = cu[s + 1] - cu[s];
    rc = check_shape(1, a->Hq, a->Hkv, S, a->D, a->block, a->dtype);
    if (rc != STEM_OK) return rc;
    rc = check_params(nblocks(S, a->block), m);
    if (rc != STEM_OK) return rc;
    if (antidiag(m) && (rc = check_antidiag(S, a->block, a->dtype, m.stride)) != STEM_OK)
      return rc;
    if (S > 0)
      need = std::max(need,
                      layout(1, a->Hq, a->Hkv, nblocks(S, a->block), a->D, &m, S, a->block).total);
  }
  if (need == 0) return STEM_OK;  // no tokens
  if (!a->q || !a->k || !a->v || !a->out || !a->sel_idx || !a->sel_cnt) return STEM_ERR_ARG;
  if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->out, 16) ||
      !aligned(a->sel_idx, 4) || !aligned(a->sel_cnt, 4) || !aligned(a->status, 4))
    return STEM_ERR_ARG;
  if (a->workspace == nullptr || !aligned(a->workspace, kAlign) || a->workspace_bytes < need)
    return STEM_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a->status) {
    rc = cuda_err(cudaMemsetAsync(a->status, 0, sizeof(int32_t), st));
    if (rc != STEM_OK) return rc;
  }
  const size_t es = elem_size(a->dtype);
  int64_t capo = 0, nbo = 0;  // CSR and count offsets of the sequences before s
  for (int s = 0; s < a->nseq; ++s) {
    const int S = cu[s + 1] - cu[s];
    if (S == 0) continue;
    const int nb = nblocks(S, a->block);
    const Plan* plan = get_plan(nb, m);
    if (plan == nullptr) return STEM_ERR_CUDA;
    const int64_t tok = cu[s];
    stem_args_t d;
    std::memset(&d, 0, sizeof d);
    d.q = static_cast<const unsigned char*>(a->q) + es * a->Hq * a->D * tok;
    d.k = static_cast<const unsigned char*>(a->k) + es * a->Hkv * a->D * tok;
    d.v = static_cast<const unsigned char*>(a->v) + es * a->Hkv * a->D * tok;
    d.out = static_cast<unsigned char*>(a->out) + es * a->Hq * a->D * tok;
    d.sel_idx = a->sel_idx + static_cast<int64_t>(a->Hq) * capo;
    d.sel_cnt = a->sel_cnt + static_cast<int64_t>(a->Hq) * nbo;
    d.B = 1;
    d.Hq = a->Hq;
    d.Hkv = a->Hkv;
    d.S = S;
    d.D = a->D;
    d.block = a->block;
    d.dtype = a->dtype;
    d.workspace = a->workspace;
    d.workspace_bytes = a->workspace_bytes;
    d.status = a->status;
    d.method = a->method;
    // the plan goes into the shared workspace in stream order, after the previous sequence's
    // kernels have read theirs
    PlanDev pd;
    rc = upload_plan(plan, a->workspace, layout(1, a->Hq, a->Hkv, nb, a->D, &m, S, a->block), st,
                     &pd);
    if (rc != STEM_OK) return rc;
    rc = enqueue_kernels(&d, m, nb, plan->cap, pd, st);
    if (rc != STEM_OK) return rc;
    capo += plan->cap;
    nbo += nb;
  }
  return STEM_OK;
}

}  // extern "C"
