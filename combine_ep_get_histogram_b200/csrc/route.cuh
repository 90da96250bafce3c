// Group-limited top-k routing: router scores [T, E] -> topk_idx [T, k] and
// topk_weights [T, k], the input of the layout step.
//
// The pages describe group-limited gating in words: experts are split into
// groups, a token first picks its best groups and then its top-k experts
// inside them ("top-4 groups, top-8 experts":
// "deepep-expert-parallel-communication-library", sections 一
// and 三).  Reading taken where they are silent: a group's score is the
// largest score of its experts; groups and experts are chosen by descending
// score with ties to the lower index; topk_idx lists the experts by
// descending score; the weights are the softmax of the chosen scores.
//
// One warp per token.  Lane l holds the scores of the contiguous experts
// [l*NQ, (l+1)*NQ), so lane order is expert order.  Scores become
// order-preserving 32-bit keys (-0 folded into +0, so equal scores stay
// equal).  Every arg-max over the warp is a max-reduction (redux.sync) of the
// lanes' best keys plus a ballot: the lowest lane holding the maximum holds
// the lowest expert index.  The selections compare input scores only, so
// they are exact; the softmax uses fp32 expf.  Scores must be finite.
//
// Three kernels.  route_aligned_kernel serves shapes whose groups fall on
// lane boundaries (E and the group size multiples of NQ, and a power-of-two
// number of lanes per group; 256 experts in 8 groups is one): a group's
// maximum is the lanes' maxima combined by xor shuffles inside the group's
// lane segment, a group's rank is counted from one shuffle per group, each
// lane sorts its candidates once (a bitonic network over 64-bit (key,
// expert) composites), and a pick takes the largest first key over the
// warp, the winning lane dropping its first entry.
// route_compact_kernel is the same with the chosen groups' experts first
// moved onto all 32 lanes, NC < NQ to a lane, in expert order: each lane
// then sorts NC composites instead of NQ (top-4 of 8 groups of 32: 4 instead
// of 8), which measured 18 % faster at 32768 tokens x 256 experts.
// route_group_limited_kernel serves every other shape: one warp
// max-reduction per group over per-expert group ids.
#pragma once

#include "common.cuh"

namespace ep {

constexpr int kRouteMaxPerLane = kMaxE / kWarp;  // 32
constexpr int kRouteMaxGroups = 32;
constexpr int kRouteThreads = 256;

struct RouteParams {
  const float* scores;
  int T, E, k, n_groups, topk_groups;
  int64_t* topk_idx;
  float* topk_weights;
};

// Order-preserving key of a finite float: a > b  <=>  key(a) > key(b), and
// key(-0) == key(+0).
__device__ __forceinline__ int32_t route_key(float f) {
  const int32_t i = __float_as_int(f + 0.0f);  // -0 + 0 = +0
  return i >= 0 ? i : i ^ 0x7fffffff;
}

constexpr int32_t kRouteNoKey = INT32_MIN;  // below every finite score's key

// NQ = experts per lane (E <= 32*NQ); the caller picks the smallest of
// 1, 2, 4, 8, 16, 32 that holds E.
// Programmatic-launch prologue of the router kernels (common.cuh): let the
// next kernel be scheduled, bring the warp's first score row into L2, then
// wait for the previous kernel's writes.
__device__ __forceinline__ void route_prologue(const RouteParams& p) {
  pdl_allow_next();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * (kRouteThreads / kWarp) + threadIdx.x / kWarp;
  if (t0 < p.T) prefetch_l2(p.scores + t0 * p.E, 4 * static_cast<int64_t>(p.E), threadIdx.x & (kWarp - 1), kWarp);
  pdl_wait_prev();
}

template <int NQ>
__global__ void __launch_bounds__(kRouteThreads) route_group_limited_kernel(RouteParams p) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int per = p.E / p.n_groups;
  const int e0 = lane * NQ;
  route_prologue(p);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kRouteThreads / kWarp) + threadIdx.x / kWarp; t < p.T;
       t += static_cast<int64_t>(gridDim.x) * (kRouteThreads / kWarp)) {
    const float* s = p.scores + t * p.E;
    float v[NQ];
    int32_t key[NQ];
    int gq[NQ];  // group of expert e0+q, -1 past E
    if (NQ % 4 == 0 && e0 + NQ <= p.E && (reinterpret_cast<uintptr_t>(s + e0) & 15) == 0) {
#pragma unroll
      for (int q = 0; q < NQ; q += 4) {
        const float4 f = *reinterpret_cast<const float4*>(s + e0 + q);
        v[q] = f.x;
        v[q + 1] = f.y;
        v[q + 2] = f.z;
        v[q + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < NQ; ++q) v[q] = e0 + q < p.E ? s[e0 + q] : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = e0 + q;
      const bool ok = e < p.E;
      key[q] = ok ? route_key(v[q]) : kRouteNoKey;
      gq[q] = ok ? e / per : -1;
    }
    // group scores: lane g keeps group g's key (one max-reduction per group)
    int32_t my_gkey = kRouteNoKey;
    for (int g = 0; g < p.n_groups; ++g) {
      int32_t m = kRouteNoKey;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (gq[q] == g) m = max(m, key[q]);
      m = __reduce_max_sync(0xffffffffu, m);
      if (lane == g) my_gkey = m;
    }
    // the chosen groups: per pick, the largest key, lowest group among equals
    uint32_t chosen = 0;
    for (int n = 0; n < p.topk_groups; ++n) {
      const bool cand = lane < p.n_groups && !((chosen >> lane) & 1u);
      const int32_t gk = cand ? my_gkey : kRouteNoKey;
      const int32_t top = __reduce_max_sync(0xffffffffu, gk);
      const uint32_t holders = __ballot_sync(0xffffffffu, cand && gk == top);
      chosen |= 1u << (__ffs(holders) - 1);
    }
    uint32_t open = 0;  // bit q: expert e0+q is still a candidate
#pragma unroll
    for (int q = 0; q < NQ; ++q)
      if (gq[q] >= 0 && ((chosen >> gq[q]) & 1u)) open |= 1u << q;
    // the best experts, in order: per round, each lane offers its best open
    // expert (lowest index among equal keys), the warp takes the maximum key
    // and, among lanes that hold it, the lowest lane
    float my_score = 0.0f;
    int my_expert = -1;
    for (int j = 0; j < p.k; ++j) {
      int32_t bk = kRouteNoKey;
      int bq = -1;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (((open >> q) & 1u) && key[q] > bk) {
          bk = key[q];
          bq = q;
        }
      const int32_t top = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t holders = __ballot_sync(0xffffffffu, bq >= 0 && bk == top);
      const int win = __ffs(holders) - 1;
      float sv = 0.0f;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q == bq) sv = v[q];
      const int wq = __shfl_sync(0xffffffffu, bq, win);
      const float ws = __shfl_sync(0xffffffffu, sv, win);
      if (lane == win) open &= ~(1u << wq);
      if (lane == j) {
        my_score = ws;
        my_expert = win * NQ + wq;
      }
    }
    // softmax of the chosen scores (the first one is the largest)
    const float top = __shfl_sync(0xffffffffu, my_score, 0);
    const float ex = lane < p.k ? expf(my_score - top) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < p.k) {
      p.topk_idx[t * p.k + lane] = my_expert;
      p.topk_weights[t * p.k + lane] = __fdiv_rn(ex, sum);
    }
  }
}

// Order of a candidate within a lane: larger composite = earlier (larger
// key, then lower local index q).  0 is below every candidate.
__device__ __forceinline__ uint64_t route_composite(int32_t key, int q) {
  return (static_cast<uint64_t>(static_cast<uint32_t>(key) ^ 0x80000000u) << 32) |
         static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(q));
}

// The score whose key is `key` (-0 comes back as +0, which changes no
// difference taken from it).
__device__ __forceinline__ float route_score(int32_t key) {
  return __int_as_float(key >= 0 ? key : key ^ 0x7fffffff);
}

__device__ __forceinline__ void route_cas(uint64_t& a, uint64_t& b) {  // a >= b afterwards
  const bool swap = b > a;
  const uint64_t hi = swap ? b : a;
  b = swap ? a : b;
  a = hi;
}

// Descending bitonic sort of N (a power of two) composites.
template <int N>
__device__ __forceinline__ void route_sort_desc(uint64_t (&a)[N]) {
#pragma unroll
  for (int k = 2; k <= N; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) {
          if ((i & k) == 0)
            route_cas(a[i], a[l]);
          else
            route_cas(a[l], a[i]);
        }
      }
}

// Groups on lane boundaries: E % NQ == 0, (E / n_groups) % NQ == 0 and
// lpg = E / n_groups / NQ a power of two, so group g is lanes
// [g*lpg, (g+1)*lpg) and lanes from E/NQ on hold no expert.  Each lane sorts
// its candidates once; a pick is a max-reduction of the lanes' first keys, a
// ballot (the lowest lane among equal keys holds the lowest expert), and the
// winning lane drops its first entry.
template <int NQ>
__global__ void __launch_bounds__(kRouteThreads) route_aligned_kernel(RouteParams p) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int lpg = p.E / p.n_groups / NQ;
  const int e0 = lane * NQ;
  const bool has = e0 < p.E;
  const int my_g = lane / lpg;
  route_prologue(p);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kRouteThreads / kWarp) + threadIdx.x / kWarp; t < p.T;
       t += static_cast<int64_t>(gridDim.x) * (kRouteThreads / kWarp)) {
    const float* s = p.scores + t * p.E;
    float v[NQ];
    if (NQ % 4 == 0 && has && (reinterpret_cast<uintptr_t>(s + e0) & 15) == 0) {
#pragma unroll
      for (int q = 0; q < NQ; q += 4) {
        const float4 f = *reinterpret_cast<const float4*>(s + e0 + q);
        v[q] = f.x;
        v[q + 1] = f.y;
        v[q + 2] = f.z;
        v[q + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < NQ; ++q) v[q] = has ? s[e0 + q] : 0.0f;
    }
    int32_t gk = kRouteNoKey;
    uint64_t c[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int32_t key = has ? route_key(v[q]) : kRouteNoKey;
      gk = max(gk, key);
      c[q] = has ? route_composite(key, q) : 0;
    }
    // group maximum over the group's lane segment
    for (int o = 1; o < lpg; o <<= 1) gk = max(gk, __shfl_xor_sync(0xffffffffu, gk, o));
    // rank of this lane's group: groups with a larger maximum, or an equal
    // one and a lower index
    int rank = 0;
    for (int g = 0; g < p.n_groups; ++g) {
      const int32_t other = __shfl_sync(0xffffffffu, gk, g * lpg);
      rank += (other > gk || (other == gk && g < my_g)) ? 1 : 0;
    }
    if (!(has && rank < p.topk_groups)) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) c[q] = 0;
    }
    route_sort_desc<NQ>(c);
    int32_t my_key = 0;
    int my_expert = -1;
    for (int j = 0; j < p.k; ++j) {
      const uint32_t head = static_cast<uint32_t>(c[0] >> 32);
      const uint32_t top = __reduce_max_sync(0xffffffffu, head);
      const int win = __ffs(__ballot_sync(0xffffffffu, head == top)) - 1;
      const uint32_t lo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(c[0]), win);
      if (lane == j) {
        my_key = static_cast<int32_t>(top ^ 0x80000000u);
        my_expert = win * NQ + static_cast<int>(0xFFFFFFFFu - lo);
      }
      if (lane == win) {
#pragma unroll
        for (int q = 0; q + 1 < NQ; ++q) c[q] = c[q + 1];
        c[NQ - 1] = 0;
      }
    }
    // softmax of the chosen scores (the first one is the largest)
    const float my_score = lane < p.k ? route_score(my_key) : 0.0f;
    const float top = __shfl_sync(0xffffffffu, my_score, 0);
    const float ex = lane < p.k ? expf(my_score - top) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < p.k) {
      p.topk_idx[t * p.k + lane] = my_expert;
      p.topk_weights[t * p.k + lane] = __fdiv_rn(ex, sum);
    }
  }
}

// Groups on lane boundaries as in route_aligned_kernel, and the chosen
// groups' topk_groups * (E / n_groups) experts moved onto the lanes, NC to a
// lane (NC a power of two below NQ, at least the candidates over 32), in
// expert order: lane L takes candidates [L*NC, (L+1)*NC) of the chosen groups
// listed in ascending group order, which lie in one group and one source
// lane (NC divides NQ and the group size).  The lowest lane among equal keys
// still holds the lowest expert, so picks and ties are those of
// route_aligned_kernel.
template <int NQ, int NC>
__global__ void __launch_bounds__(kRouteThreads) route_compact_kernel(RouteParams p) {
  static_assert(NC < NQ && NQ % NC == 0, "compaction takes fewer candidates per lane");
  const int lane = threadIdx.x & (kWarp - 1);
  const int per = p.E / p.n_groups;
  const int lpg = per / NQ;
  const int e0 = lane * NQ;
  const bool has = e0 < p.E;
  const int my_g = lane / lpg;
  const int f0 = lane * NC;  // this lane's first place in the list of candidates
  const bool holds = f0 < p.topk_groups * per;
  const int cg = f0 / per, x = f0 - cg * per;  // chosen group (by rank in group order) and place in it
  route_prologue(p);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kRouteThreads / kWarp) + threadIdx.x / kWarp; t < p.T;
       t += static_cast<int64_t>(gridDim.x) * (kRouteThreads / kWarp)) {
    const float* s = p.scores + t * p.E;
    float v[NQ];
    if (NQ % 4 == 0 && has && (reinterpret_cast<uintptr_t>(s + e0) & 15) == 0) {
#pragma unroll
      for (int q = 0; q < NQ; q += 4) {
        const float4 f = *reinterpret_cast<const float4*>(s + e0 + q);
        v[q] = f.x;
        v[q + 1] = f.y;
        v[q + 2] = f.z;
        v[q + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < NQ; ++q) v[q] = has ? s[e0 + q] : 0.0f;
    }
    int32_t gk = kRouteNoKey;
#pragma unroll
    for (int q = 0; q < NQ; ++q) gk = max(gk, has ? route_key(v[q]) : kRouteNoKey);
    // group maximum over the group's lane segment, and the group's rank
    for (int o = 1; o < lpg; o <<= 1) gk = max(gk, __shfl_xor_sync(0xffffffffu, gk, o));
    int rank = 0;
    for (int g = 0; g < p.n_groups; ++g) {
      const int32_t other = __shfl_sync(0xffffffffu, gk, g * lpg);
      rank += (other > gk || (other == gk && g < my_g)) ? 1 : 0;
    }
    // the chosen groups' first lanes, and this lane's group among them
    const unsigned lead = __ballot_sync(0xffffffffu, has && (lane & (lpg - 1)) == 0 && rank < p.topk_groups);
    unsigned m = lead;
    for (int i = 0; i < cg; ++i) m &= m - 1;  // drop the cg lower chosen groups
    const int g = holds ? (__ffs(m) - 1) / lpg : 0;
    const int ef = g * per + x;  // this lane's first candidate expert
    const int src = ef / NQ, pos = ef - src * NQ;
    // fetch scores [pos, pos + NC) of lane src: in round r every lane offers
    // its scores [r*NC, (r+1)*NC)
    float nv[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) nv[j] = 0.0f;
#pragma unroll
    for (int r = 0; r < NQ / NC; ++r)
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        const float val = __shfl_sync(0xffffffffu, v[r * NC + j], src);
        if (pos == r * NC) nv[j] = val;
      }
    uint64_t c[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) c[j] = holds ? route_composite(route_key(nv[j]), ef + j) : 0;
    route_sort_desc<NC>(c);
    int32_t my_key = 0;
    int my_expert = -1;
    for (int j = 0; j < p.k; ++j) {
      const uint32_t head = static_cast<uint32_t>(c[0] >> 32);
      const uint32_t top = __reduce_max_sync(0xffffffffu, head);
      const int win = __ffs(__ballot_sync(0xffffffffu, head == top)) - 1;
      const uint32_t lo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(c[0]), win);
      if (lane == j) {
        my_key = static_cast<int32_t>(top ^ 0x80000000u);
        my_expert = static_cast<int>(0xFFFFFFFFu - lo);  // the composite carries the expert itself
      }
      if (lane == win) {
#pragma unroll
        for (int q = 0; q + 1 < NC; ++q) c[q] = c[q + 1];
        c[NC - 1] = 0;
      }
    }
    // softmax of the chosen scores (the first one is the largest)
    const float my_score = lane < p.k ? route_score(my_key) : 0.0f;
    const float top = __shfl_sync(0xffffffffu, my_score, 0);
    const float ex = lane < p.k ? expf(my_score - top) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < p.k) {
      p.topk_idx[t * p.k + lane] = my_expert;
      p.topk_weights[t * p.k + lane] = __fdiv_rn(ex, sum);
    }
  }
}

}  // namespace ep
