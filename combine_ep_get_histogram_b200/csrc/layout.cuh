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
//      place; the column's total and summaries (num_tokens_per_expert,
//      num_tokens_per_rank, count_src_rank_expert, and the per-rank offsets
//      relative to the expert's first row).
//   3. layout_assign_kernel: one CTA per tile: exclusive scan of the expert
//      totals (expert_offset), then the tile's pairs are ranked in (t, j)
//      order: each warp owns a contiguous run of pairs, counts it per
//      expert, the eight warp counts are scanned per expert from the tile's
//      base, and each warp walks its run again giving lane l of a 32-pair
//      chunk the rank popc(same_expert_mask & lanemask_lt).  The CTAs also
//      add expert_offset to the per-(rank, expert) offsets, a slice each.
#pragma once

#include <cooperative_groups.h>

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
  // 0: the kernel lets the next one on the stream be scheduled at its start.
  // 1: only after its own programmatic-launch wait, so that the next kernel
  // is scheduled only once every kernel before this one has completed (set on
  // the last layout kernel of the fused layout + dispatch call, whose
  // dispatch reads x before its own wait).
  int late_trigger;
};

// The programmatic-launch prologue of every layout kernel: trigger, an
// optional L2 prefetch of what the kernel reads first, wait (and the late
// trigger described above).
__device__ __forceinline__ void layout_trigger_early(const LayoutParams& p) {
  if (!p.late_trigger) pdl_allow_next();
}
__device__ __forceinline__ void layout_wait(const LayoutParams& p) {
  pdl_wait_prev();
  if (p.late_trigger) pdl_allow_next();
}

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
  bool bad = false;
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t* idx = p.topk_idx + static_cast<int64_t>(t0) * p.k;
  layout_trigger_early(p);
  prefetch_l2(idx, static_cast<int64_t>(npairs) * 8, threadIdx.x, blockDim.x);
  layout_wait(p);
  // a tile holds at most kTilePairs pairs: every thread loads its (up to)
  // kPairsPerThread expert ids first, then counts them
  int e[kPairsPerThread];
#pragma unroll
  for (int c = 0; c < kPairsPerThread; ++c) {
    const int i = c * kLayoutThreads + threadIdx.x;
    e[c] = i < npairs ? pair_expert(p, idx[i], bad) : -1;
  }
  for (int i = threadIdx.x; i < p.ncol; i += blockDim.x) hist[i] = 0;
  for (int i = threadIdx.x; i < ntok * p.R; i += blockDim.x) flags[i] = 0;
  __syncthreads();
#pragma unroll
  for (int c = 0; c < kPairsPerThread; ++c) {
    const int i = c * kLayoutThreads + threadIdx.x;
    const unsigned same = __match_any_sync(0xffffffffu, e[c]);
    if (e[c] >= 0) {
      if (lane == __ffs(same) - 1) atomicAdd(&hist[e[c]], __popc(same));
      flags[(i / p.k) * p.R + e[c] / p.Er] = 1;
    }
  }
  __syncthreads();

  uint8_t* itr = p.is_token_in_rank + static_cast<int64_t>(t0) * p.R;
  for (int base = 0; base < ntok * p.R; base += blockDim.x) {  // uniform trip count
    const int i = base + threadIdx.x;
    const uint8_t f = i < ntok * p.R ? flags[i] : 0;
    if (i < ntok * p.R) itr[i] = f;
    const int key = f ? i % p.R : -1;
    const unsigned same = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && lane == __ffs(same) - 1) atomicAdd(&hist[p.E + key], __popc(same));
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
  layout_trigger_early(p);
  layout_wait(p);
  const int32_t total = block_exclusive_scan(col, p.nt, scratch);
  if (threadIdx.x == 0) p.coltotal[c] = total;
  if (c < p.E) {
    // expert column: totals, and per source rank the pairs before the rank's
    // first tile (offsets relative to expert_offset[c]; the assign kernel adds it)
    if (threadIdx.x == 0) p.num_tokens_per_expert[c] = total;
    for (int r = threadIdx.x; r < p.R; r += blockDim.x) {
      const int32_t pre = p.tiles_per_rank > 0 ? col[r * p.tiles_per_rank] : 0;
      const int32_t nxt = (r + 1 < p.R && p.tiles_per_rank > 0) ? col[(r + 1) * p.tiles_per_rank] : total;
      p.src_rank_expert_offset[r * p.E + c] = pre;
      p.count_src_rank_expert[r * p.E + c] = nxt - pre;
    }
  } else if (threadIdx.x == 0) {
    p.num_tokens_per_rank[c - p.E] = total;
  }
}

__global__ void __launch_bounds__(kLayoutThreads) layout_assign_kernel(LayoutParams p) {
  extern __shared__ int32_t smem[];
  int32_t* eoff = smem;                       // [E + 1]
  int32_t* whist = smem + p.E + 1;            // [kLayoutWarps * E]
  __shared__ int32_t scratch[kWarp];
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
  const int tile = blockIdx.x;
  const bool has_tile = tile < p.nt;

  // issue the tile's loads first: its pairs' expert ids (each warp owns the
  // contiguous run [w*S, min((w+1)*S, npairs)), S a multiple of 32) and its
  // per-expert base within each expert block
  int t0 = 0, t1 = 0;
  if (has_tile) tile_range(p, tile, t0, t1);
  const int npairs = (t1 - t0) * p.k;
  const int64_t pair0 = static_cast<int64_t>(t0) * p.k;
  const int S = ((npairs + kLayoutWarps - 1) / kLayoutWarps + kWarp - 1) / kWarp * kWarp;
  const int my_lo = warp * S, my_hi = min(my_lo + S, npairs);
  int ereg[kMaxChunksPerWarp];
  bool bad = false;  // already reported by layout_count_kernel
  layout_trigger_early(p);
  layout_wait(p);
#pragma unroll
  for (int c = 0; c < kMaxChunksPerWarp; ++c) {
    const int i = my_lo + c * kWarp + lane;
    ereg[c] = i < my_hi ? pair_expert(p, p.topk_idx[pair0 + i], bad) : -1;
  }
  int32_t tile_base[kMaxE / kLayoutThreads];
#pragma unroll
  for (int c = 0; c < kMaxE / kLayoutThreads; ++c) {
    const int e = c * kLayoutThreads + threadIdx.x;
    tile_base[c] = (has_tile && e < p.E) ? p.colhist[static_cast<int64_t>(e) * p.nt + tile] : 0;
  }

  // expert_offset = exclusive scan of the expert totals (every CTA)
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) eoff[e] = p.coltotal[e];
  for (int i = threadIdx.x; i < kLayoutWarps * p.E; i += blockDim.x) whist[i] = 0;
  __syncthreads();
  const int32_t p_eff = block_exclusive_scan(eoff, p.E, scratch);
  if (threadIdx.x == 0) eoff[p.E] = p_eff;
  __syncthreads();

  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) p.expert_offset[e] = eoff[e];
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.R * p.E; i += gridDim.x * blockDim.x)
    p.src_rank_expert_offset[i] += eoff[i % p.E];
  // rows past the last valid pair have no source
  const int64_t P = static_cast<int64_t>(p.T) * p.k;
  for (int64_t i = p_eff + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < P;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p.src_of_slot[i] = -1;
  if (!has_tile) return;

  int32_t* wh = whist + warp * p.E;
#pragma unroll
  for (int c = 0; c < kMaxChunksPerWarp; ++c) {
    const int e = ereg[c];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(same) - 1) wh[e] += __popc(same);
    __syncwarp();
  }
  __syncthreads();
#pragma unroll
  for (int c = 0; c < kMaxE / kLayoutThreads; ++c) {
    const int e = c * kLayoutThreads + threadIdx.x;
    if (e < p.E) {
      int32_t run = eoff[e] + tile_base[c];
      for (int w = 0; w < kLayoutWarps; ++w) {
        const int32_t n = whist[w * p.E + e];
        whist[w * p.E + e] = run;
        run += n;
      }
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

// ----------------------------------------- small problems, one CTA cluster
//
// Up to kSmallMaxPairs pairs (the decode shape, 8 ranks x 128 tokens x
// top-8, is 8192) are handled by one cluster of C CTAs, in one launch: 16
// (a non-portable cluster size) where the device can hold such a cluster,
// else the portable 8.  CTA c takes the tile of whole tokens
// [c*T/C, (c+1)*T/C).  Phase 1, per CTA: per-warp expert histograms of the
// tile's pairs (each warp owns a contiguous run of pairs), per-(source rank,
// expert) counts and per-rank token counts (warp-aggregated shared-memory
// atomics, whose sums do not depend on order), is_token_in_rank.  Cluster
// barrier.  Phase 2: every CTA reads the other tiles' histograms through
// distributed shared memory, so it knows the expert totals (expert_offset)
// and how many pairs of each expert come from earlier tiles; it scans its
// warp histograms from there and ranks its pairs with
// popc(same_expert_mask & lanemask_lt).  CTA 0 writes the summaries.  A
// final cluster barrier keeps every CTA's shared memory alive until the
// others have read it.

constexpr int kClusterCtas = 8;      // portable cluster size
constexpr int kClusterCtasWide = 16; // non-portable: halves each CTA's pairs (decode layout 14.7 -> 14.4 us per call)
constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / kWarp;
constexpr int kSmallMaxPairs = 16384;
constexpr int kSmallMaxE = 256;
constexpr int kSmallMaxR = 64;
constexpr int kSmallMaxRE = 2048;
constexpr int kSmallMaxTileFlags = 8192;  // tile tokens x R flag bytes
// pair chunks per warp: pairs per CTA <= (T/C + 1) * k <= kSmallMaxPairs / C + kMaxK
__host__ __device__ constexpr int small_chunks(int C) {
  return ((kSmallMaxPairs / C + kMaxK) / kSmallWarps + kWarp - 1) / kWarp + 1;
}

__host__ __device__ inline int small_tile_tokens(int T, int C) { return (T + C - 1) / C; }

// The limits are those of the 8-CTA cluster, whose tiles are the larger.
__host__ __device__ inline bool layout_small_fits(int T, int k, int E, int R) {
  return static_cast<int64_t>(T) * k <= kSmallMaxPairs && E <= kSmallMaxE && R <= kSmallMaxR &&
         R * E <= kSmallMaxRE && static_cast<int64_t>(small_tile_tokens(T, kClusterCtas)) * R <= kSmallMaxTileFlags;
}

// shared memory, int32 words then flag bytes:
//   hist[E] base[E] whist[W][E] eoff[E+1] cnt[R*E] rank_cnt[R] flags[tile tokens * R]
__host__ __device__ inline int layout_small_smem(int T, int E, int R, int C) {
  return (2 * E + kSmallWarps * E + (E + 1) + R * E + R) * 4 + small_tile_tokens(T, C) * R;
}
// the largest of the above over every shape layout_small_fits admits (36 KB)
constexpr int kSmallMaxSmem =
    (2 * kSmallMaxE + kSmallWarps * kSmallMaxE + (kSmallMaxE + 1) + kSmallMaxRE + kSmallMaxR) * 4 + kSmallMaxTileFlags;

template <int C>
__global__ void __cluster_dims__(C, 1, 1) __launch_bounds__(kSmallThreads)
layout_small_kernel(LayoutParams p) {
  constexpr int kSmallChunks = small_chunks(C);
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ int32_t smem[];
  int32_t* hist = smem;                              // [E]   this tile's pairs per expert (read by all CTAs)
  int32_t* base = hist + p.E;                        // [E]   pairs of each expert in earlier tiles
  int32_t* whist = base + p.E;                       // [W][E]
  int32_t* eoff = whist + kSmallWarps * p.E;         // [E + 1]
  int32_t* cnt = eoff + p.E + 1;                     // [R][E] this tile's pairs by (source rank, expert)
  int32_t* rank_cnt = cnt + p.R * p.E;               // [R]   this tile's tokens per destination rank
  uint8_t* flags = reinterpret_cast<uint8_t*>(rank_cnt + p.R);  // [tile tokens][R]
  __shared__ int32_t scratch[kWarp];
  const int c = static_cast<int>(cluster.block_rank());
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
  const int t0 = static_cast<int>(static_cast<int64_t>(c) * p.T / C);
  const int t1 = static_cast<int>(static_cast<int64_t>(c + 1) * p.T / C);
  const int ntok = t1 - t0;
  const int npairs = ntok * p.k;
  const int64_t pair0 = static_cast<int64_t>(t0) * p.k;
  const int S = ((npairs + kSmallWarps - 1) / kSmallWarps + kWarp - 1) / kWarp * kWarp;
  const int my_lo = warp * S, my_hi = min(my_lo + S, npairs);
  const int my_chunks = my_hi > my_lo ? (my_hi - my_lo + kWarp - 1) / kWarp : 0;  // chunks holding pairs (warp-uniform)

  bool bad = false;
  int ereg[kSmallChunks];
  layout_trigger_early(p);
  prefetch_l2(p.topk_idx + pair0, static_cast<int64_t>(npairs) * 8, threadIdx.x, blockDim.x);
  layout_wait(p);
#pragma unroll
  for (int q = 0; q < kSmallChunks; ++q) {
    const int i = my_lo + q * kWarp + lane;
    ereg[q] = i < my_hi ? pair_expert(p, p.topk_idx[pair0 + i], bad) : -1;
  }
  for (int i = threadIdx.x; i < (2 + kSmallWarps) * p.E; i += blockDim.x) hist[i] = 0;  // hist, base, whist
  for (int i = threadIdx.x; i < p.R * p.E + p.R; i += blockDim.x) cnt[i] = 0;         // cnt, rank_cnt
  for (int i = threadIdx.x; i < ntok * p.R; i += blockDim.x) flags[i] = 0;
  __syncthreads();

  // ---- phase 1: count this tile.  When the tile's tokens all belong to one
  // source rank (the decode shape: one rank per CTA), its (rank, expert)
  // counts are the tile's expert histogram and need no counting of their own.
  const int r_first = ntok > 0 ? t0 / p.Tr : 0;
  const bool one_rank = ntok > 0 && (t1 - 1) / p.Tr == r_first;
  int32_t* wh = whist + warp * p.E;
#pragma unroll
  for (int q = 0; q < kSmallChunks; ++q) {
    if (q >= my_chunks) break;
    const int i = my_lo + q * kWarp + lane;
    const int e = ereg[q];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(same) - 1) wh[e] += __popc(same);
    const int tl = e >= 0 ? i / p.k : 0;  // token within the tile
    if (!one_rank) {
      const int key = e >= 0 ? ((t0 + tl) / p.Tr) * p.E + e : -1;
      const unsigned same_key = __match_any_sync(0xffffffffu, key);
      if (key >= 0 && lane == __ffs(same_key) - 1) atomicAdd(&cnt[key], __popc(same_key));
    }
    if (e >= 0) flags[tl * p.R + e / p.Er] = 1;
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    int32_t tot = 0;
    for (int w = 0; w < kSmallWarps; ++w) tot += whist[w * p.E + e];
    hist[e] = tot;
    if (one_rank) cnt[r_first * p.E + e] = tot;
  }
  for (int b0 = 0; b0 < ntok * p.R; b0 += blockDim.x) {  // uniform trip count
    const int i = b0 + threadIdx.x;
    const uint8_t f = i < ntok * p.R ? flags[i] : 0;
    if (i < ntok * p.R) p.is_token_in_rank[static_cast<int64_t>(t0) * p.R + i] = f;
    const int key = f ? i % p.R : -1;
    const unsigned same = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && lane == __ffs(same) - 1) atomicAdd(&rank_cnt[key], __popc(same));
  }
  cluster.sync();  // every tile's hist, cnt and rank_cnt are final

  // ---- phase 2: totals and this tile's bases from every tile's histogram
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    int32_t tot = 0, before = 0;
#pragma unroll
    for (int r = 0; r < C; ++r) {
      const int32_t n = cluster.map_shared_rank(hist, r)[e];
      before += r < c ? n : 0;
      tot += n;
    }
    eoff[e] = tot;
    base[e] = before;
  }
  __syncthreads();
  const int32_t p_eff = block_exclusive_scan(eoff, p.E, scratch);
  if (threadIdx.x == 0) eoff[p.E] = p_eff;
  __syncthreads();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    int32_t run = eoff[e] + base[e];
    for (int w = 0; w < kSmallWarps; ++w) {
      const int32_t n = whist[w * p.E + e];
      whist[w * p.E + e] = run;
      run += n;
    }
  }
  __syncthreads();
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int q = 0; q < kSmallChunks; ++q) {
    if (q >= my_chunks) break;
    const int i = my_lo + q * kWarp + lane;
    const int e = ereg[q];
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

  // summaries, spread over the cluster: CTA c owns experts [e_lo, e_hi) and
  // writes their offsets and counts (CTA C-1 also the end offset), and the
  // token counts of destination ranks c, c + C, ...  One thread per (rank,
  // owned expert) and one per owned destination rank gather the cluster's
  // counts in a single round of distributed-shared-memory loads; then one
  // thread per owned expert walks the ranks for the offsets.  whist is free
  // again after the ranking loop.
  const int e_lo = c * p.E / C, e_hi = (c + 1) * p.E / C, ne = e_hi - e_lo;
  for (int e = e_lo + threadIdx.x; e < e_hi; e += blockDim.x) {
    p.expert_offset[e] = eoff[e];
    p.num_tokens_per_expert[e] = eoff[e + 1] - eoff[e];
  }
  if (c == C - 1 && threadIdx.x == 0) p.expert_offset[p.E] = eoff[p.E];
  __syncthreads();
  int32_t* tot_re = whist;  // [R][e_hi - e_lo]
  const int nre = p.R * ne, nr = (p.R - c + C - 1) / C;
  for (int i = threadIdx.x; i < nre + nr; i += blockDim.x) {
    const bool re = i < nre;
    const int r = re ? i / ne : c + C * (i - nre);
    const int e = re ? e_lo + (i - r * ne) : 0;
    int32_t* word = re ? cnt + r * p.E + e : rank_cnt + r;  // this CTA's copy; the others' at the same offset
    int32_t m = 0;
#pragma unroll
    for (int q = 0; q < C; ++q) m += *cluster.map_shared_rank(word, q);
    if (re) {
      tot_re[i] = m;
      p.count_src_rank_expert[r * p.E + e] = m;
    } else {
      p.num_tokens_per_rank[r] = m;
    }
  }
  __syncthreads();
  for (int el = threadIdx.x; el < ne; el += blockDim.x) {
    int32_t run = eoff[e_lo + el];
    for (int r = 0; r < p.R; ++r) {
      p.src_rank_expert_offset[r * p.E + e_lo + el] = run;
      run += tot_re[r * ne + el];
    }
  }
  const int P = p.T * p.k;
  for (int i = p_eff + c * blockDim.x + threadIdx.x; i < P; i += C * blockDim.x) p.src_of_slot[i] = -1;
  if (bad) atomicOr(p.error_word, 1);
  cluster.sync();  // keep this CTA's shared memory until the others are done reading it
}

// ------------------------------------------------ padded low-latency layout
//
// Receive rows [E][R][M]: the pairs of (source rank r, expert e) fill block
// (e*R + r) from its first row in (t, j) order.  No block depends on another
// source rank, so one CTA per source rank does the whole layout in one
// launch: per-warp expert histograms of the rank's pairs (contiguous runs),
// an exclusive scan over warps per expert from 0, ranking with
// popc(same_expert_mask & lanemask_lt).  Totals over ranks
// (num_tokens_per_expert, num_tokens_per_rank): with R <= kPadClusterMax the
// R CTAs are one thread-block cluster, and after a cluster barrier CTA c sums
// its slice of the experts and ranks over every CTA's counts through
// distributed shared memory (no atomics, nothing to zero first); with more
// ranks they are integer atomics into arrays zeroed just before the launch.
// Either way the values do not depend on order.  Rows a block does not fill
// are marked -1 in src_of_slot.

constexpr int kPadThreads = 512;
constexpr int kPadWarps = kPadThreads / kWarp;
constexpr int kPadMaxPairs = 8192;   // pairs of one source rank
constexpr int kPadMaxFlags = 32768;  // (T/R) x R token-rank flag bytes
constexpr int kPadChunks = (kPadMaxPairs / kPadWarps + kWarp - 1) / kWarp;  // 16
constexpr int kPadClusterMax = 8;    // portable cluster size

__host__ __device__ inline int layout_padded_smem(int Tr, int E, int R) {
  return (kPadWarps * E + E + R) * 4 + Tr * R;  // whist[W][E] cnt[E] rank_cnt[R] flags[Tr][R]
}
constexpr int kPadMaxSmem = (kPadWarps * kMaxE + kMaxE + kMaxR) * 4 + kPadMaxFlags;

template <bool CLUSTER>
__global__ void __launch_bounds__(kPadThreads) layout_padded_kernel(LayoutParams p, int M) {
  extern __shared__ int32_t smem[];
  int32_t* whist = smem;                         // [W][E]
  int32_t* cnt = whist + kPadWarps * p.E;        // [E] this rank's pairs per expert
  int32_t* rank_cnt = cnt + p.E;                 // [R] this rank's tokens per destination rank
  uint8_t* flags = reinterpret_cast<uint8_t*>(rank_cnt + p.R);  // [Tr][R]
  const int r = blockIdx.x;
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
  const int npairs = p.Tr * p.k;
  const int64_t pair0 = static_cast<int64_t>(r) * p.Tr * p.k;
  const int S = ((npairs + kPadWarps - 1) / kPadWarps + kWarp - 1) / kWarp * kWarp;
  const int my_lo = warp * S, my_hi = min(my_lo + S, npairs);
  const int my_chunks = my_hi > my_lo ? (my_hi - my_lo + kWarp - 1) / kWarp : 0;  // chunks holding pairs (warp-uniform)

  bool bad = false, over = false;
  int ereg[kPadChunks];
  layout_trigger_early(p);
  prefetch_l2(p.topk_idx + pair0, static_cast<int64_t>(npairs) * 8, threadIdx.x, blockDim.x);
  layout_wait(p);
#pragma unroll
  for (int q = 0; q < kPadChunks; ++q) {
    const int i = my_lo + q * kWarp + lane;
    ereg[q] = i < my_hi ? pair_expert(p, p.topk_idx[pair0 + i], bad) : -1;
  }
  for (int i = threadIdx.x; i < (kPadWarps + 1) * p.E + p.R; i += blockDim.x) whist[i] = 0;  // whist, cnt, rank_cnt
  for (int i = threadIdx.x; i < p.Tr * p.R; i += blockDim.x) flags[i] = 0;
  __syncthreads();

  int32_t* wh = whist + warp * p.E;
#pragma unroll
  for (int q = 0; q < kPadChunks; ++q) {
    if (q >= my_chunks) break;
    const int i = my_lo + q * kWarp + lane;
    const int e = ereg[q];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(same) - 1) wh[e] += __popc(same);
    if (e >= 0) flags[(i / p.k) * p.R + e / p.Er] = 1;
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    int32_t run = 0;
    for (int w = 0; w < kPadWarps; ++w) {
      const int32_t n = whist[w * p.E + e];
      whist[w * p.E + e] = run;
      run += n;
    }
    cnt[e] = run;
    p.count_src_rank_expert[r * p.E + e] = run;
    p.src_rank_expert_offset[r * p.E + e] = (e * p.R + r) * M;
    if (!CLUSTER && run > 0) atomicAdd(&p.num_tokens_per_expert[e], run);
  }
  if (r == 0)
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) p.expert_offset[e] = e * p.R * M;
  __syncthreads();

  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int q = 0; q < kPadChunks; ++q) {
    if (q >= my_chunks) break;
    const int i = my_lo + q * kWarp + lane;
    const int e = ereg[q];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int32_t pos = wh[e] + __popc(same & lt);
      if (pos < M) {
        const int32_t row = (e * p.R + r) * M + pos;
        p.slot_of_pair[pair0 + i] = row;
        p.src_of_slot[row] = static_cast<int32_t>(pair0 + i);
      } else {
        p.slot_of_pair[pair0 + i] = -1;
        over = true;
      }
    } else if (i < my_hi) {
      p.slot_of_pair[pair0 + i] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(same) - 1) wh[e] += __popc(same);
    __syncwarp();
  }
  // rows of this rank's blocks that no pair filled: one warp per expert block
  for (int e = warp; e < p.E; e += kPadWarps) {
    int32_t* blk = p.src_of_slot + static_cast<int64_t>(e * p.R + r) * M;
    for (int i = min(cnt[e], M) + lane; i < M; i += kWarp) blk[i] = -1;
  }
  // is_token_in_rank and token counts per destination rank
  uint8_t* itr = p.is_token_in_rank + static_cast<int64_t>(r) * p.Tr * p.R;
  for (int b0 = 0; b0 < p.Tr * p.R; b0 += blockDim.x) {  // uniform trip count
    const int i = b0 + threadIdx.x;
    const uint8_t f = i < p.Tr * p.R ? flags[i] : 0;
    if (i < p.Tr * p.R) itr[i] = f;
    const int key = f ? i % p.R : -1;
    const unsigned same = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && lane == __ffs(same) - 1) atomicAdd(&rank_cnt[key], __popc(same));
  }
  __syncthreads();
  if constexpr (CLUSTER) {
    // every CTA's cnt and rank_cnt are final; CTA r sums its slice of the
    // experts and of the destination ranks over the cluster
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int e_lo = r * p.E / p.R, e_hi = (r + 1) * p.E / p.R;
    for (int e = e_lo + threadIdx.x; e < e_hi; e += blockDim.x) {
      int32_t n = 0;
      for (int q = 0; q < p.R; ++q) n += cluster.map_shared_rank(cnt, q)[e];
      p.num_tokens_per_expert[e] = n;
    }
    if (threadIdx.x == 0) {
      int32_t n = 0;
      for (int q = 0; q < p.R; ++q) n += cluster.map_shared_rank(rank_cnt, q)[r];
      p.num_tokens_per_rank[r] = n;
    }
    cluster.sync();  // keep this CTA's shared memory until the others have read it
  } else {
    for (int d = threadIdx.x; d < p.R; d += blockDim.x)
      if (rank_cnt[d] > 0) atomicAdd(&p.num_tokens_per_rank[d], rank_cnt[d]);
  }
  if (bad) atomicOr(p.error_word, 1);
  if (over) atomicOr(p.error_word, 2);
}

}  // namespace ep
