// Multi-GPU expert parallelism: the data-movement kernels of one rank, with
// every receive-side row in its owner rank's buffer.
//
// One process per GPU.  Rank r holds tokens [r*T/R, (r+1)*T/R) and experts
// [r*E/R, (r+1)*E/R).  Every rank has all ranks' expert ids and has run the
// same layout over them, so slots are global: the pair (t, j) to expert e
// takes slot s in e's block, exactly as on one GPU.  The owner o = e / (E/R)
// keeps the rows [expert_offset[o*E/R], expert_offset[(o+1)*E/R]) of the
// global receive buffer, and slot s is its local row s - expert_offset[o*E/R].
// The kernels fuse the exchange with the arithmetic (the pages' dispatch and
// combine are all-to-alls between ranks: "DeepEP：MoE 专家并行 EP 通信 kernel
// 编译与使用指南", section 五; the normal kernels move tokens over NVLink:
// "deepep-expert-parallel-communication-library", section 一).
// Dispatch quantises this rank's tokens and stores each row straight into
// its owner's buffer.  Combine and dispatch backward load the owners' rows
// and reduce them.  Combine backward loads y from, and stores grad_y into,
// the owners' buffers.  An owner's buffer may be another GPU's memory
// (NVLink peer addresses).  The kernels use plain loads and stores, and
// dispatch TMA bulk stores; nothing loads with TMA or multicasts.  On one
// GPU, the owners' buffers are R local allocations, and their concatenation
// equals the single-GPU receive buffer row for row.
//
// The kernels follow the single-GPU ones.  Dispatch builds each row once in
// shared memory and writes it to its owners with TMA bulk copies for 4 to 16
// chunks (a warp per (token, 512-channel chunk) storing 16-byte pieces for
// other widths).  The gathers take a warp per (token, chunk), their k row
// loads in flight in batches of 8; combine backward a warp per pair, four
// chunks at a time with one partial sum each.  Bounds are checked per piece
// only when H is not a multiple of 512.  Peer links (about 0.8 TB/s per
// direction) rather than HBM bound them.
#pragma once

#include "movement.cuh"

namespace ep {

constexpr int kMaxPeers = 64;

// Per owner rank: the base of its buffer (row 0 = its first global slot).
struct PeerRows {
  void* base[kMaxPeers];
};

struct PeerParams {
  int T, H, k, G, chunks;          // T: this rank's tokens
  int t_begin;                     // global index of this rank's first token
  int Er, R;                       // experts per rank, ranks
  const int32_t* slot_of_pair;     // [T_all * k], the global layout
  const int64_t* topk_idx;         // [T_all * k], every rank's expert ids
  const int32_t* expert_offset;    // [E + 1], global
  const float* topk_weights;       // [T * k], this rank's tokens
};

// Every owner's first global row, staged in shared memory once per CTA so
// that a pair's local row needs no dependent global load.
__device__ __forceinline__ void load_owner_rows(const PeerParams& p, int32_t* row0) {
  for (int o = threadIdx.x; o < p.R; o += blockDim.x) row0[o] = p.expert_offset[o * p.Er];
  __syncthreads();
}

// Slot, owner rank and the owner's local row of this rank's pair (t, j);
// slot -1 (masked pair): owner 0, row -1.
__device__ __forceinline__ int peer_pair(const PeerParams& p, const int32_t* row0, int t, int j, int& owner,
                                         int& row) {
  const int64_t ug = (static_cast<int64_t>(p.t_begin) + t) * p.k + j;
  const int s = p.slot_of_pair[ug];
  const int64_t e = p.topk_idx[ug];
  owner = 0;
  row = -1;
  if (s >= 0) {  // a slot means a valid expert id, below E <= 1024: a 32-bit division
    owner = static_cast<int>(e) / p.Er;
    row = s - row0[owner];
  }
  return s;
}

// Per expert, the address global slot 0 would have in its owner's buffer of
// rows of row_bytes (the owner's base minus its first row times row_bytes, in
// 64-bit integer arithmetic; only rows inside the buffer are ever formed from
// it).  Staged in shared memory once per CTA, it puts a pair's row one add
// from its slot: no division and no second lookup between the id and slot
// loads and the row loads of the gathers, which resolve the k pairs of a
// token once per chunk (the peer combine over all prefill tokens as one
// launch: 741-751 us with the division and the owner's first row per pair,
// 661-664 us with the table).  The caller synchronises.
__device__ __forceinline__ void load_expert_bases(const PeerParams& p, const PeerRows& rows, int row_bytes,
                                                  unsigned long long* base_of) {
  const int E = p.Er * p.R;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int o = e / p.Er;
    base_of[e] = reinterpret_cast<unsigned long long>(rows.base[o]) -
                 static_cast<unsigned long long>(p.expert_offset[o * p.Er]) * static_cast<unsigned>(row_bytes);
  }
}

// Address of the owner's row of this rank's pair (t, j); 0 for a masked pair.
__device__ __forceinline__ unsigned long long peer_row_addr(const PeerParams& p, const unsigned long long* base_of,
                                                            int t, int j, int row_bytes) {
  const int64_t ug = (static_cast<int64_t>(p.t_begin) + t) * p.k + j;
  const int s = p.slot_of_pair[ug];
  if (s < 0) return 0ull;  // masked (or an id the layout rejected): no table entry is read
  const int e = static_cast<int>(p.topk_idx[ug]);
  return base_of[e] + static_cast<unsigned long long>(s) * static_cast<unsigned>(row_bytes);
}

template <bool FP8>
__global__ void __launch_bounds__(kMoveThreads)
dispatch_peers_kernel(PeerParams p, const uint16_t* __restrict__ x, PeerRows rx, PeerRows rscale, PeerRows rweight) {
  __shared__ int32_t row0[kMaxPeers];
  pdl_allow_next();
  pdl_wait_prev();
  load_owner_rows(p, row0);
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t nunits = static_cast<int64_t>(p.T) * p.chunks;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp; u < nunits;
       u += static_cast<int64_t>(gridDim.x) * kMoveWarps) {
    const int t = static_cast<int>(u / p.chunks);
    const int c = static_cast<int>(u - static_cast<int64_t>(t) * p.chunks);
    const int h0 = piece_channel(c, lane), h1 = h0 + kHalfChunk;
    const bool a0 = h0 < p.H, a1 = h1 < p.H;
    const uint16_t* xr = x + static_cast<int64_t>(t) * p.H;
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    if (a0) v0 = ld_ro_v4(xr + h0);
    if (a1) v1 = ld_ro_v4(xr + h1);
    int my_slot = -1, my_owner = 0, my_row = -1;
    if (lane < p.k) my_slot = peer_pair(p, row0, t, lane, my_owner, my_row);
    uint2 q0 = make_uint2(0, 0), q1 = q0;
    float sc0 = 1.0f, sc1 = 1.0f;
    if constexpr (FP8) {
      q0 = quantize_piece(v0, sc0);
      q1 = quantize_piece(v1, sc1);
    }
    const bool scale_lane = (lane & (kLanesPerGroup - 1)) == 0;
    for (int j = 0; j < p.k; ++j) {
      const int s = __shfl_sync(0xffffffffu, my_slot, j);
      const int o = __shfl_sync(0xffffffffu, my_owner, j);
      const int row = __shfl_sync(0xffffffffu, my_row, j);
      if (s < 0) continue;
      if constexpr (FP8) {
        uint8_t* dst = static_cast<uint8_t*>(rx.base[o]) + static_cast<int64_t>(row) * p.H;
        float* srow = static_cast<float*>(rscale.base[o]) + static_cast<int64_t>(row) * p.G;
        if (a0) {
          *reinterpret_cast<uint2*>(dst + h0) = q0;
          if (scale_lane) srow[h0 / kGroup] = sc0;
        }
        if (a1) {
          *reinterpret_cast<uint2*>(dst + h1) = q1;
          if (scale_lane) srow[h1 / kGroup] = sc1;
        }
      } else {
        uint16_t* dst = static_cast<uint16_t*>(rx.base[o]) + static_cast<int64_t>(row) * p.H;
        if (a0) st_v4(dst + h0, v0);
        if (a1) st_v4(dst + h1, v1);
      }
    }
    if (c == 0 && lane < p.k && my_slot >= 0 && rweight.base[my_owner] != nullptr)
      static_cast<float*>(rweight.base[my_owner])[my_row] = p.topk_weights[static_cast<int64_t>(t) * p.k + lane];
  }
}

// Dispatch in the single-GPU kernel's form (dispatch_tma_kernel): a CTA per
// token and a warp per 512-channel chunk; the E4M3 (or BF16) row is built
// once in shared memory and leaves as one TMA bulk copy per pair
// (cp.async.bulk.global.shared::cta, a plain store: no multicast) into its
// owner's buffer, local or a peer's.  Scales and weights leave by plain
// stores.  The host launches it for 4 to 16 chunks (1536 < H <= 8192), as on
// one GPU; the shared-memory stage holds each pair's owner next to its row.
template <bool FP8>
__global__ void __launch_bounds__(kTmaMaxChunks * kWarp, 3)
dispatch_tma_peers_kernel(PeerParams p, const uint16_t* __restrict__ x, PeerRows rx, PeerRows rscale,
                          PeerRows rweight) {
  extern __shared__ __align__(128) uint8_t tma_smem[];
  __shared__ int32_t row0[kMaxPeers];
  __shared__ int32_t owner_stage[2 * kMaxK];
  pdl_allow_next();
  pdl_wait_prev();
  load_owner_rows(p, row0);
  const TmaSmemLayout L = tma_smem_layout(p.H, FP8);
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
  const int h0 = piece_channel(warp, lane), h1 = h0 + kHalfChunk;  // one chunk per warp
  const bool a0 = h0 < p.H, a1 = h1 < p.H;
  const int row_bytes = FP8 ? p.H : 2 * p.H;

  uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
  int t = blockIdx.x;
  if (t < p.T) {
    const uint16_t* xr = x + static_cast<int64_t>(t) * p.H;
    if (a0) v0 = ld_ro_v4(xr + h0);
    if (a1) v1 = ld_ro_v4(xr + h1);
  }
  for (int it = 0; t < p.T; ++it, t += gridDim.x) {
    const int stage = it & 1;
    uint8_t* row = tma_smem + (it % L.stages) * L.row_bytes;
    int32_t* srow = reinterpret_cast<int32_t*>(tma_smem + L.off_slot) + stage * kMaxK;  // owner's local row
    int32_t* sowner = owner_stage + stage * kMaxK;
    float* sw = reinterpret_cast<float*>(tma_smem + L.off_w) + stage * kMaxK;
    float* sscale = reinterpret_cast<float*>(tma_smem + L.off_scale) + stage * p.G;

    // prefetch the next token of this CTA
    const int tn = t + gridDim.x;
    uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
    if (tn < p.T) {
      const uint16_t* xr = x + static_cast<int64_t>(tn) * p.H;
      if (a0) n0 = ld_ro_v4(xr + h0);
      if (a1) n1 = ld_ro_v4(xr + h1);
    }
    // the row stage is free once the copies issued L.stages tokens ago have
    // read it (the first token's stage has had no copies)
    if (threadIdx.x == 0) bulk_wait_read_all_but(L.stages - 1);
    if (it > 0) __syncthreads();

    if constexpr (FP8) {
      float sc0, sc1;
      const uint2 q0 = quantize_piece(v0, sc0);
      const uint2 q1 = quantize_piece(v1, sc1);
      const bool scale_lane = (lane & (kLanesPerGroup - 1)) == 0;
      if (a0) {
        *reinterpret_cast<uint2*>(row + h0) = q0;
        if (scale_lane) sscale[h0 / kGroup] = sc0;
      }
      if (a1) {
        *reinterpret_cast<uint2*>(row + h1) = q1;
        if (scale_lane) sscale[h1 / kGroup] = sc1;
      }
    } else {
      if (a0) *reinterpret_cast<uint4*>(row + 2 * h0) = v0;
      if (a1) *reinterpret_cast<uint4*>(row + 2 * h1) = v1;
    }
    // the pairs' owners, rows and weights after the quantisation, as in
    // dispatch_tma_kernel
    if (warp == 0 && lane < p.k) {
      int o, r;
      peer_pair(p, row0, t, lane, o, r);
      srow[lane] = r;
      sowner[lane] = o;
      sw[lane] = p.topk_weights[static_cast<int64_t>(t) * p.k + lane];
    }
    // make the generic-proxy shared-memory writes visible to the bulk copies
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();

    if (threadIdx.x == 0) {
      const uint32_t src = static_cast<uint32_t>(__cvta_generic_to_shared(row));
      for (int j = 0; j < p.k; ++j) {
        const int r = srow[j];
        if (r >= 0)
          bulk_store_row(static_cast<uint8_t*>(rx.base[sowner[j]]) + static_cast<int64_t>(r) * row_bytes, src,
                         row_bytes);
      }
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    if constexpr (FP8) {
      for (int i = threadIdx.x; i < p.k * p.G; i += blockDim.x) {
        const int j = i / p.G, g = i - j * p.G;
        const int r = srow[j];
        if (r >= 0) static_cast<float*>(rscale.base[sowner[j]])[static_cast<int64_t>(r) * p.G + g] = sscale[g];
      }
    }
    if (threadIdx.x < p.k) {
      const int r = srow[threadIdx.x];
      float* wb = static_cast<float*>(rweight.base[sowner[threadIdx.x]]);
      if (r >= 0 && wb != nullptr) wb[r] = sw[threadIdx.x];
    }
    v0 = n0;
    v1 = n1;
  }
  if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// out[t] = bf16( chain over j of (WEIGHTED ? fmaf(w[t,j], y[slot], acc) : acc + y[slot]) ), acc = +0.0f,
// j = 0..k-1 in order: the single-GPU arithmetic, rows loaded from their owners.
template <bool WEIGHTED, bool RAGGED>
__global__ void __launch_bounds__(kMoveThreads)
gather_reduce_peers_kernel(PeerParams p, PeerRows y, uint16_t* __restrict__ out) {
  __shared__ unsigned long long base_of[kMaxE];
  pdl_allow_next();
  pdl_wait_prev();
  load_expert_bases(p, y, 2 * p.H, base_of);
  __syncthreads();
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t nunits = static_cast<int64_t>(p.T) * p.chunks;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp; u < nunits;
       u += static_cast<int64_t>(gridDim.x) * kMoveWarps) {
    const int t = static_cast<int>(u / p.chunks);
    const int c = static_cast<int>(u - static_cast<int64_t>(t) * p.chunks);
    const int h0 = piece_channel(c, lane), h1 = h0 + kHalfChunk;
    const bool a0 = !RAGGED || h0 < p.H, a1 = !RAGGED || h1 < p.H;
    unsigned long long my_row = 0;  // this lane's pair: the row's address, 0 if masked
    float my_w = 0.0f;
    if (lane < p.k) {
      my_row = peer_row_addr(p, base_of, t, lane, 2 * p.H);
      if (WEIGHTED) my_w = p.topk_weights[static_cast<int64_t>(t) * p.k + lane];
    }
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
    for (int jb = 0; jb < p.k; jb += 8) {  // all loads of a batch of 8 rows in flight, then the arithmetic
      uint4 v[8][2];
      unsigned long long src[8];
      float w[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = (jb + jj) & (kWarp - 1);
        src[jj] = __shfl_sync(0xffffffffu, my_row, j);
        w[jj] = __shfl_sync(0xffffffffu, my_w, j);
        if (jb + jj >= p.k) src[jj] = 0;
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        v[jj][0] = v[jj][1] = make_uint4(0, 0, 0, 0);
        if (src[jj] != 0) {
          const uint16_t* r = reinterpret_cast<const uint16_t*>(src[jj]);
          if (a0) v[jj][0] = *reinterpret_cast<const uint4*>(r + h0);
          if (a1) v[jj][1] = *reinterpret_cast<const uint4*>(r + h1);
        }
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (src[jj] == 0) continue;
        float f[16];
        unpack8(v[jj][0], f);
        unpack8(v[jj][1], f + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (WEIGHTED) acc[i] = fmaf(w[jj], f[i], acc[i]);
          else acc[i] = __fadd_rn(acc[i], f[i]);
        }
      }
    }
    uint16_t* dst = out + static_cast<int64_t>(t) * p.H;
    if (a0) st_v4(dst + h0, pack8_bf16(acc));
    if (a1) st_v4(dst + h1, pack8_bf16(acc + 8));
  }
}

// grad_y[slot] = bf16(w * g[t]) into the owner's buffer; grad_w[t, j] = g[t] . y[slot] with y from the owner:
// four chunks at a time with one fp32 partial sum per chunk slot, then xor shuffles across lanes (the
// single-GPU kernel's order).
template <bool RAGGED>
__global__ void __launch_bounds__(kMoveThreads)
combine_backward_peers_kernel(PeerParams p, const uint16_t* __restrict__ g, PeerRows y, PeerRows grad_y,
                              float* __restrict__ grad_w) {
  __shared__ unsigned long long y_of[kMaxE], gy_of[kMaxE];
  pdl_allow_next();
  pdl_wait_prev();
  load_expert_bases(p, y, 2 * p.H, y_of);
  load_expert_bases(p, grad_y, 2 * p.H, gy_of);
  __syncthreads();
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t npairs = static_cast<int64_t>(p.T) * p.k;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp; u < npairs;
       u += static_cast<int64_t>(gridDim.x) * kMoveWarps) {
    const int t = static_cast<int>(u / p.k), j = static_cast<int>(u - static_cast<int64_t>(t) * p.k);
    const int64_t ug = (static_cast<int64_t>(p.t_begin) + t) * p.k + j;
    const int s = p.slot_of_pair[ug];
    if (s < 0) {
      if (lane == 0) grad_w[u] = 0.0f;
      continue;
    }
    const int e = static_cast<int>(p.topk_idx[ug]);
    const unsigned long long off = static_cast<unsigned long long>(s) * static_cast<unsigned>(2 * p.H);
    const float w = p.topk_weights[u];
    const uint16_t* gr = g + static_cast<int64_t>(t) * p.H;
    const uint16_t* yr = reinterpret_cast<const uint16_t*>(y_of[e] + off);
    uint16_t* dr = reinterpret_cast<uint16_t*>(gy_of[e] + off);
    float d[kCbwdUnroll];
#pragma unroll
    for (int q = 0; q < kCbwdUnroll; ++q) d[q] = 0.0f;
    for (int c0 = 0; c0 < p.chunks; c0 += kCbwdUnroll) {
      uint4 gv[kCbwdUnroll][2], yv[kCbwdUnroll][2];
#pragma unroll
      for (int q = 0; q < kCbwdUnroll; ++q) {
        const int h0 = piece_channel(c0 + q, lane), h1 = h0 + kHalfChunk;
        gv[q][0] = gv[q][1] = yv[q][0] = yv[q][1] = make_uint4(0, 0, 0, 0);
        if (c0 + q < p.chunks) {
          if (!RAGGED || h0 < p.H) {
            gv[q][0] = ld_l1_v4(gr + h0);
            yv[q][0] = *reinterpret_cast<const uint4*>(yr + h0);
          }
          if (!RAGGED || h1 < p.H) {
            gv[q][1] = ld_l1_v4(gr + h1);
            yv[q][1] = *reinterpret_cast<const uint4*>(yr + h1);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < kCbwdUnroll; ++q) {
        const int h0 = piece_channel(c0 + q, lane), h1 = h0 + kHalfChunk;
        uint4 ov[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t gw[4] = {gv[q][h].x, gv[q][h].y, gv[q][h].z, gv[q][h].w};
          const uint32_t yw[4] = {yv[q][h].x, yv[q][h].y, yv[q][h].z, yv[q][h].w};
          uint32_t o4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float g0 = bf16_lo(gw[i]), g1 = bf16_hi(gw[i]);
            d[q] = fmaf(g0, bf16_lo(yw[i]), d[q]);
            d[q] = fmaf(g1, bf16_hi(yw[i]), d[q]);
            o4[i] = pack_bf16x2(__fmul_rn(w, g0), __fmul_rn(w, g1));
          }
          ov[h] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        if (c0 + q < p.chunks) {
          if (!RAGGED || h0 < p.H) st_v4(dr + h0, ov[0]);
          if (!RAGGED || h1 < p.H) st_v4(dr + h1, ov[1]);
        }
      }
    }
    float dot = (d[0] + d[1]) + (d[2] + d[3]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (lane == 0) grad_w[u] = dot;
  }
}

}  // namespace ep
