// Routing layout: per-expert / per-rank histograms, offsets,
// is_token_in_rank and the stable slot of every (token, expert) pair.
//
// The pages name the quantities (per-expert token counts as the skew check:
// "DeepEP：专为MoE模型打造的All-to-All通信库", section 5.2; the handle that
// dispatch returns and combine reuses: "DeepEP：MoE 专家并行 EP 通信 kernel
// 编译与使用指南", section 五).  The slot order is (token, top-k position)
// inside each expert's block of rows.
//
// Design: a counting sort in three launches, no atomics whose order can
// change a result and no inter-CTA waiting.
//   1. layout_count_kernel: one CTA per tile of whole tokens inside one
//      source rank.  Shared-memory histogram of the tile's pairs by expert
//      (warp-aggregated with __match_any_sync) and by destination rank
//      (tokens with >= 1 pair there); writes is_token_in_rank rows and the
//      tile's column of the [E+R, tiles] count matrix.
//   2. layout_scan_kernel: one CTA per column: exclusive scan over tiles in
//      place, column total on the side.
//   3. layout_assign_kernel: one CTA per tile: exclusive scan of the expert
//      totals (expert_offset), then the tile's pairs are ranked in (t, j)
//      order: each warp owns a contiguous run of pairs, counts it per
//      expert, the eight warp counts are scanned per expert from the tile's
//      base, and each warp walks its run again giving lane l of a 32-pair
//      chunk the rank popc(same_expert_mask & lanemask_lt).  CTA 0 also
//      writes the per-rank and per-(rank, expert) summaries.
#pragma once

#include "common.cuh"

namespace ep {

struct LayoutParams {
  const int64_t* topk_idx;
  int T, k, E, R, Tr, Er;
  int tile_t;          // tokens per tile
  int tiles_per_rank;  // ceil(Tr / tile_t)
  int nt;              // tiles = R * tiles_per_rank
  int ncol;            // E + R columns
  int32_t* colhist;    // [ncol * nt]: counts, then exclusive prefixes over tiles
  int32_t* coltotal;   // [ncol]
  int32_t* num_tokens_per_expert;
  int32_t* expert_offset;
  int32_t* num_tokens_per_rank;
  int32_t* count_src_rank_expert;
  int32_t* src_rank_expert_offset;
  uint8_t* is_token_in_rank;
  int32_t* slot_of_pair;
  int32_t* src_of_slot;
  int32_t* error_word;
};

__device__ __forceinline__ void tile_range(const LayoutParams& p, int tile, int& t0, int& t1) {
  const int r = tile / p.tiles_per_rank;
  const int b = tile - r * p.tiles_per_rank;
  t0 = r * p.Tr + b * p.tile_t;
  t1 = min(t0 + p.tile_t, (r + 1) * p.Tr);
}

// Expert id of a pair, or -1 for masked / out-of-range ids.
__device__ __forceinline__ int pair_expert(const LayoutParams& p, int64_t e, bool& bad) {
  if (e == -1) return -1;
  if (e < -1 || e >= p.E) { bad = true; return -1; }
  return static_cast<int>(e);
}

__global__ void __launch_bounds__(kLayoutThreads) layout_count_kernel(LayoutParams p) {
  extern __shared__ int32_t smem[];
  int32_t* hist = smem;                                          // [E + R]
  uint8_t* flags = reinterpret_cast<uint8_t*>(smem + p.ncol);    // [tile_t * R]
  const int tile = blockIdx.x;
  int t0, t1;
  tile_range(p, tile, t0, t1);
  const int ntok = t1 - t0;
  const int npairs = ntok * p.k;
  for (int i = threadIdx.x; i < p.ncol; i += blockDim.x) hist[i] = 0;
  for (int i = threadIdx.x; i < ntok * p.R; i += blockDim.x) flags[i] = 0;
  __syncthreads();

  bool bad = false;
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t* idx = p.topk_idx + static_cast<int64_t>(t0) * p.k;
  for (int base = 0; base < npairs; base += blockDim.x) {  // uniform trip count
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < npairs) e = pair_expert(p, idx[i], bad);
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      if (lane == __ffs(same) - 1) atomicAdd(&hist[e], __popc(same));
      flags[(i / p.k) * p.R + e / p.Er] = 1;
    }
  }
  __syncthreads();

  uint8_t* itr = p.is_token_in_rank + static_cast<int64_t>(t0) * p.R;
  for (int i = threadIdx.x; i < ntok * p.R; i += blockDim.x) {
    const uint8_t f = flags[i];
    itr[i] = f;
    if (f) atomicAdd(&hist[p.E + i % p.R], 1);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < p.ncol; c += blockDim.x)
    p.colhist[static_cast<int64_t>(c) * p.nt + tile] = hist[c];
  if (bad) atomicOr(p.error_word, 1);
}

// Exclusive scan of `n` values in place by one CTA (each thread takes a
// contiguous segment); returns the total to every thread.
__device__ int32_t block_exclusive_scan(int32_t* data, int n, int32_t* scratch /*[kWarp]*/) {
  const int nthr = blockDim.x;
  const int per = (n + nthr - 1) / nthr;
  const int lo = min(n, static_cast<int>(threadIdx.x) * per);
  const int hi = min(n, lo + per);
  int32_t s = 0;
  for (int i = lo; i < hi; ++i) s += data[i];
  // inclusive scan of the per-thread sums
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
  int32_t inc = s;
  for (int d = 1; d < kWarp; d <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += v;
  }
  if (lane == kWarp - 1) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int nw = (nthr + kWarp - 1) / kWarp;
    int32_t w = lane < nw ? scratch[lane] : 0;
    for (int d = 1; d < kWarp; d <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += v;
    }
    scratch[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  int32_t run = inc - s + (warp > 0 ? scratch[warp - 1] : 0);
  const int32_t total = scratch[(nthr + kWarp - 1) / kWarp - 1];
  for (int i = lo; i < hi; ++i) {
    const int32_t v = data[i];
    data[i] = run;
    run += v;
  }
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kLayoutThreads) layout_scan_kernel(LayoutParams p) {
  __shared__ int32_t scratch[kWarp];
  const int c = blockIdx.x;
  int32_t* col = p.colhist + static_cast<int64_t>(c) * p.nt;
  const int32_t total = block_exclusive_scan(col, p.nt, scratch);
  if (threadIdx.x == 0) p.coltotal[c] = total;
}

__global__ void __launch_bounds__(kLayoutThreads) layout_assign_kernel(LayoutParams p) {
  extern __shared__ int32_t smem[];
  int32_t* eoff = smem;                       // [E + 1]
  int32_t* whist = smem + p.E + 1;            // [kLayoutWarps * E]
  __shared__ int32_t scratch[kWarp];
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;

  // expert_offset = exclusive scan of the expert totals (every CTA)
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) eoff[e] = p.coltotal[e];
  __syncthreads();
  const int32_t p_eff = block_exclusive_scan(eoff, p.E, scratch);
  if (threadIdx.x == 0) eoff[p.E] = p_eff;
  __syncthreads();

  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
      p.expert_offset[e] = eoff[e];
      if (e < p.E) p.num_tokens_per_expert[e] = p.coltotal[e];
    }
    for (int r = threadIdx.x; r < p.R; r += blockDim.x) p.num_tokens_per_rank[r] = p.coltotal[p.E + r];
    for (int i = threadIdx.x; i < p.R * p.E; i += blockDim.x) {
      const int r = i / p.E, e = i - r * p.E;
      const int32_t* col = p.colhist + static_cast<int64_t>(e) * p.nt;
      const int32_t pre = p.tiles_per_rank > 0 ? col[r * p.tiles_per_rank] : 0;
      const int32_t nxt = (r + 1 < p.R && p.tiles_per_rank > 0) ? col[(r + 1) * p.tiles_per_rank]
                                                                : p.coltotal[e];
      p.src_rank_expert_offset[i] = eoff[e] + pre;
      p.count_src_rank_expert[i] = nxt - pre;
    }
  }
  // rows past the last valid pair have no source
  const int64_t P = static_cast<int64_t>(p.T) * p.k;
  for (int64_t i = p_eff + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < P;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p.src_of_slot[i] = -1;

  const int tile = blockIdx.x;
  if (tile >= p.nt) return;
  int t0, t1;
  tile_range(p, tile, t0, t1);
  const int npairs = (t1 - t0) * p.k;
  const int64_t pair0 = static_cast<int64_t>(t0) * p.k;

  for (int i = threadIdx.x; i < kLayoutWarps * p.E; i += blockDim.x) whist[i] = 0;
  __syncthreads();

  // each warp owns pairs [w*S, min((w+1)*S, npairs)), S a multiple of 32
  const int S = ((npairs + kLayoutWarps - 1) / kLayoutWarps + kWarp - 1) / kWarp * kWarp;
  const int my_lo = warp * S, my_hi = min(my_lo + S, npairs);
  int32_t* wh = whist + warp * p.E;
  int ereg[kMaxChunksPerWarp];
  bool bad = false;
#pragma unroll
  for (int c = 0; c < kMaxChunksPerWarp; ++c) {
    const int i = my_lo + c * kWarp + lane;
    int e = -1;
    if (i < my_hi) e = pair_expert(p, p.topk_idx[pair0 + i], bad);
    ereg[c] = e;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(same) - 1) wh[e] += __popc(same);
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    int32_t run = eoff[e] + p.colhist[static_cast<int64_t>(e) * p.nt + tile];
    for (int w = 0; w < kLayoutWarps; ++w) {
      const int32_t c = whist[w * p.E + e];
      whist[w * p.E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int c = 0; c < kMaxChunksPerWarp; ++c) {
    const int i = my_lo + c * kWarp + lane;
    const int e = ereg[c];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int32_t s = wh[e] + __popc(same & lt);
      p.slot_of_pair[pair0 + i] = s;
      p.src_of_slot[s] = static_cast<int32_t>(pair0 + i);
    } else if (i < my_hi) {
      p.slot_of_pair[pair0 + i] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(same) - 1) wh[e] += __popc(same);
    __syncwarp();
  }
}

}  // namespace ep
