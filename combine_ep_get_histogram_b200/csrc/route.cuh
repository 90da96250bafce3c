// Group-limited top-k routing: router scores [T, E] -> topk_idx [T, k] and
// topk_weights [T, k], the input of the layout step.
//
// The pages describe group-limited gating in words: experts are split into
// groups, a token first picks its best groups and then its top-k experts
// inside them ("top-4 groups, top-8 experts": blog.hotdry.top, sections 一
// and 三).  Reading taken where they are silent: a group's score is the
// largest score of its experts; groups and experts are chosen by descending
// score with ties to the lower index; topk_idx lists the experts by
// descending score; the weights are the softmax of the chosen scores.
//
// One warp per token.  Lane l holds the scores of the contiguous experts
// [l*NQ, (l+1)*NQ), so lane order is expert order.  Scores become
// order-preserving 32-bit keys (-0 folded into +0, so equal scores stay
// equal); each group's maximum is one warp max-reduction (redux.sync), and
// every arg-max over the warp is a max-reduction of the lanes' best keys plus
// a ballot: the lowest lane holding the maximum holds the lowest expert index.
// The selections compare input scores only, so they are exact; the softmax
// uses fp32 expf.  Scores must be finite.
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
template <int NQ>
__global__ void __launch_bounds__(kRouteThreads) route_group_limited_kernel(RouteParams p) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int per = p.E / p.n_groups;
  const int e0 = lane * NQ;
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

}  // namespace ep
