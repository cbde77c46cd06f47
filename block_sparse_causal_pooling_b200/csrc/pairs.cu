// Step schedule of a head pair for the tensor-core attention kernel.
//
// Two query heads of one kv-head group at the same query block i keep exactly k(i) key blocks
// each ("Stem: Rethinking Causal Information Flow in Sparse Attention": the position-dependent
// budget of gist.science/es "Resumen tecnico" 2.A depends only on i). Their kept lists pair up
// completely: every block both keep is one step served by one K/V tile, and the blocks only A
// keeps zip with the blocks only B keeps (as many of each). The attention kernel walks these
// k(i) steps for the two heads together, so a shared block is fetched from L2 once.
//
// Output, per item (b, g, p, i) with heads A = g*G + 2p and B = A + 1:
//   sched[((b*Hkv + g)*P + p)*cap + off(i) + t] = blockA | blockB << 16,  t < k(i),
// shared blocks first (ascending), then the lone pairs (ascending in each head). blockB is
// 0xFFFF when G is odd and the pair has no head B (then blockA = list A in order).
//
// One warp per item: a lane takes one entry of a list, tests membership in the other list by
// binary search, and ballots give every entry its output position.
//
// The region also holds, in its first kCounterBytes, the attention kernel's work counter, which
// this kernel sets to 0 (the attention kernel runs next on the same stream and claims its work
// items from it).
#include <cuda_runtime.h>

#include "stem_internal.h"

namespace stem {
namespace {

constexpr int kPairWarps = 8;

__device__ __forceinline__ int clampb(int x, int i) { return min(max(x, 0), i); }

// Is x in the ascending list l[0..k)?
__device__ __forceinline__ bool member(const int32_t* l, int k, int x, int i) {
  int lo = 0, hi = k - 1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    const int v = clampb(l[mid], i);
    if (v == x) return true;
    if (v < x) lo = mid + 1; else hi = mid - 1;
  }
  return false;
}

__global__ void __launch_bounds__(kPairWarps * 32) pairs_kernel(
    const int32_t* __restrict__ sel_idx, int Hq, int Hkv, int nb, int64_t items, PlanDev plan,
    int64_t cap, uint16_t* __restrict__ sched, unsigned long long* __restrict__ counter) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *counter = 0ull;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * kPairWarps + (threadIdx.x >> 5);
  if (item >= items) return;
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const int G = Hq / Hkv;
  const int P = (G + 1) >> 1;
  const int i = static_cast<int>(item % nb);
  const int64_t gp = item / nb;  // (b*Hkv + g)*P + p
  const int p = static_cast<int>(gp % P);
  const int64_t bg = gp / P;
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int hA = g * G + 2 * p;
  const bool hasB = 2 * p + 1 < G;
  const int k = plan.k[i];
  const int64_t off = plan.off[i];
  const int32_t* la = sel_idx + (static_cast<int64_t>(b) * Hq + hA) * cap + off;
  const int32_t* lb = la + cap;  // head hA + 1 (valid only when hasB)
  uint16_t* out = sched + 2 * (gp * cap + off);

  if (!hasB) {
    for (int t = lane; t < k; t += 32) {
      out[2 * t] = static_cast<uint16_t>(clampb(la[t], i));
      out[2 * t + 1] = 0xFFFF;
    }
    return;
  }
  // pass 1: number of shared blocks
  int shared = 0;
  for (int t0 = 0; t0 < k; t0 += 32) {
    const int t = t0 + lane;
    const bool in = t < k && member(lb, k, clampb(la[t], i), i);
    shared += __popc(__ballot_sync(0xffffffffu, in));
  }
  // pass 2: entries of A -> shared slots (both halves) or lone slots (low half)
  int ns = 0, nla = 0;
  for (int t0 = 0; t0 < k; t0 += 32) {
    const int t = t0 + lane;
    const int a = t < k ? clampb(la[t], i) : 0;
    const bool in = t < k && member(lb, k, a, i);
    const unsigned bs = __ballot_sync(0xffffffffu, in);
    const unsigned bl = __ballot_sync(0xffffffffu, t < k && !in);
    if (t < k) {
      if (in) {
        const int pos = ns + __popc(bs & lt);
        out[2 * pos] = static_cast<uint16_t>(a);
        out[2 * pos + 1] = static_cast<uint16_t>(a);
      } else {
        const int pos = shared + nla + __popc(bl & lt);
        if (pos < k) out[2 * pos] = static_cast<uint16_t>(a);
      }
    }
    ns += __popc(bs);
    nla += __popc(bl);
  }
  // pass 3: entries only B keeps -> lone slots (high half)
  int nlb = 0;
  for (int t0 = 0; t0 < k; t0 += 32) {
    const int t = t0 + lane;
    const int bv = t < k ? clampb(lb[t], i) : 0;
    const bool lone = t < k && !member(la, k, bv, i);
    const unsigned bl = __ballot_sync(0xffffffffu, lone);
    if (lone) {
      const int pos = shared + nlb + __popc(bl & lt);
      if (pos < k) out[2 * pos + 1] = static_cast<uint16_t>(bv);
    }
    nlb += __popc(bl);
  }
}

}  // namespace

cudaError_t launch_pairs(const int32_t* sel_idx, int B, int Hq, int Hkv, int nb, PlanDev plan,
                         int64_t cap, uint32_t* region, cudaStream_t st) {
  auto* counter = reinterpret_cast<unsigned long long*>(region);
  uint32_t* sched = pairs_schedule(region);
  const int G = Hq / Hkv;
  const int64_t items = static_cast<int64_t>(B) * Hkv * ((G + 1) / 2) * nb;
  if (items == 0) return cudaSuccess;
  const int64_t grid = (items + kPairWarps - 1) / kPairWarps;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  pairs_kernel<<<static_cast<unsigned>(grid), kPairWarps * 32, 0, st>>>(
      sel_idx, Hq, Hkv, nb, items, plan, cap, reinterpret_cast<uint16_t*>(sched), counter);
  return cudaGetLastError();
}

size_t pairs_bytes(int B, int Hq, int Hkv, int nb) {
  const int G = Hq / Hkv;
  // the work counter, then the schedule (upper bound: cap <= nb (nb + 1) / 2 for any budget)
  return kCounterBytes + sizeof(uint32_t) * static_cast<size_t>(B) * Hkv * ((G + 1) / 2) *
                             (static_cast<size_t>(nb) * (nb + 1) / 2);
}

}  // namespace stem
