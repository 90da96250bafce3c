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
// One warp per token.  Lane l holds the scores of experts l + 32q (coalesced
// 128-byte loads).  Group maxima are warp reductions; groups, then experts,
// are picked by repeated warp arg-max over (score, lower index first).  The
// selections compare input scores only, so they are exact; the softmax uses
// fp32 expf.  Scores must be finite.
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

// (v, i) beats (w, j): higher score, then lower index
__device__ __forceinline__ bool route_better(float v, int i, float w, int j) {
  return v > w || (v == w && i < j);
}

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    const int j = __shfl_xor_sync(0xffffffffu, i, o);
    if (route_better(w, j, v, i)) {
      v = w;
      i = j;
    }
  }
}

// NQ = values per lane (E <= 32*NQ); the caller picks the smallest of
// 1, 2, 4, 8, 16, 32 that holds E.
template <int NQ>
__global__ void __launch_bounds__(kRouteThreads) route_group_limited_kernel(RouteParams p) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int per = p.E / p.n_groups;
  const float kNone = -__int_as_float(0x7f800000);  // -inf: below every finite score
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kRouteThreads / kWarp) + threadIdx.x / kWarp; t < p.T;
       t += static_cast<int64_t>(gridDim.x) * (kRouteThreads / kWarp)) {
    const float* s = p.scores + t * p.E;
    float v[NQ];
    int gq[NQ];  // group of this lane's q-th expert, -1 past E
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = q * kWarp + lane;
      const bool ok = e < p.E;
      v[q] = ok ? s[e] : kNone;
      gq[q] = ok ? e / per : -1;
    }
    // group scores: lane g ends up holding the score of group g
    float my_group = kNone;
    for (int g = 0; g < p.n_groups; ++g) {
      float m = kNone;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (gq[q] == g) m = fmaxf(m, v[q]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == g) my_group = m;
    }
    // the best groups, one arg-max per pick
    uint32_t chosen = 0;
    for (int n = 0; n < p.topk_groups; ++n) {
      const bool cand = lane < p.n_groups && !((chosen >> lane) & 1u);
      float gv = cand ? my_group : kNone;
      int gi = cand ? lane : kWarp;
      warp_argmax(gv, gi);
      if (gi < kWarp) chosen |= 1u << gi;
    }
    // candidates: this lane's experts in the chosen groups
    uint32_t open = 0;  // bit q: expert q*32+lane is still a candidate
#pragma unroll
    for (int q = 0; q < NQ; ++q)
      if (gq[q] >= 0 && ((chosen >> gq[q]) & 1u)) open |= 1u << q;
    // the best experts, in order
    float my_score = 0.0f;
    int my_expert = -1;
    for (int j = 0; j < p.k; ++j) {
      float bv = kNone;
      int bi = p.E;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int e = q * kWarp + lane;
        if (((open >> q) & 1u) && route_better(v[q], e, bv, bi)) {
          bv = v[q];
          bi = e;
        }
      }
      warp_argmax(bv, bi);
      if (bi < p.E && (bi & (kWarp - 1)) == lane) open &= ~(1u << (bi / kWarp));
      if (lane == j) {
        my_score = bv;
        my_expert = bi;
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
