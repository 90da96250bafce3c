// Data movement: dispatch (BF16 copy or fused FP8 E4M3 quantisation), combine,
// combine backward and dispatch backward.
//
// Operations (pages: "DeepEP：MoE 专家并行 EP 通信 kernel 编译与使用指南",
// section 五 使用方法 and FAQ Q5 — dispatch scatters tokens to experts,
// combine gathers the expert outputs back and sums them, the forward handle
// serves both backward passes; FP8 dispatch + BF16 combine: blog.hotdry.top,
// section 五 实践建议; conversion fused into the movement: bjdmk.com.cn,
// section 3.2).
//
// All four kernels are HBM-bound streams.  Work unit = one warp x one token x
// one 512-channel chunk: each lane moves 16 channels (two 16-byte bf16
// vectors), so a warp reads or writes 1 KiB of bf16 (512 B of E4M3) per row
// with fully coalesced 16-byte accesses, and an FP8 scale group (128
// channels) is exactly 8 lanes.  Grids are capped at (SMs x resident CTAs)
// and stride over the units.  Read-only inputs use non-coherent,
// L1-no-allocate loads.
#pragma once

#include "common.cuh"

namespace ep {

struct MoveParams {
  int T, H, k, G;
  int chunks;  // ceil(H / kChunk)
  const int32_t* slot_of_pair;
  const float* topk_weights;
};

constexpr int kMoveThreads = 256;
constexpr int kMoveWarps = kMoveThreads / kWarp;

// ---------------------------------------------------------------- dispatch

// f[i] <- x_i / scale, rounded to nearest even in fp32, for 16 values of one
// 128-channel group (scale >= the group's amax / 448).
//
// Fast path (Markstein's division with a correctly rounded reciprocal, P.
// Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): r = RN(1/scale), q0 = RN(|x|*r),
// e = |x| - q0*scale (exact through the FMA), q = RN(q0 + e*r), sign copied
// back.  It gives the correctly rounded quotient unless the remainder
// underflows; for inputs that are bf16 values this holds whenever |x| >=
// 2^-105 and scale is a normal number with a finite reciprocal.  Every
// (x, amax) pair of bf16 values was checked: the resulting E4M3 codes equal
// those of the IEEE division.  Other elements (zeros excepted) take the IEEE
// division, which a warp executes only if one of its lanes needs it.
// The IEEE-division fallback of quotients_by_scale, out of line: it runs
// only for groups or elements outside the fast path's range.
struct Quot16 {
  float v[16];
};

__device__ __noinline__ Quot16 quotients_ieee(uint4 v0, uint4 v1, float scale, bool group_fast, Quot16 q) {
  float f[16];
  unpack8(v0, f);
  unpack8(v1, f + 8);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t mag = __float_as_uint(f[i]) & 0x7FFFFFFFu;
    if (!(group_fast && (mag >= 0x0B000000u || mag == 0u))) q.v[i] = __fdiv_rn(f[i], scale);
  }
  return q;
}

__device__ __forceinline__ void quotients_by_scale_ieee(const uint4& v0, const uint4& v1, float scale,
                                                        bool group_fast, float* q) {
  Quot16 in;
#pragma unroll
  for (int i = 0; i < 16; ++i) in.v[i] = q[i];
  const Quot16 out = quotients_ieee(v0, v1, scale, group_fast, in);
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = out.v[i];
}

__device__ __forceinline__ void quotients_by_scale(const uint4& v0, const uint4& v1, float scale,
                                                   float* q) {
  float f[16];
  unpack8(v0, f);
  unpack8(v1, f + 8);
  const float r = __frcp_rn(scale);
  const bool group_fast = scale >= 1.17549435e-38f && r <= 3.40282347e+38f;
  bool any_slow = false;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t b = __float_as_uint(f[i]);
    const uint32_t mag = b & 0x7FFFFFFFu;
    any_slow |= !(group_fast && (mag >= 0x0B000000u || mag == 0u));
    const float ax = __uint_as_float(mag);
    const float q0 = __fmul_rn(ax, r);
    const float e = fmaf(-q0, scale, ax);
    q[i] = __uint_as_float(__float_as_uint(fmaf(e, r, q0)) | (b & 0x80000000u));
  }
  if (__any_sync(0xffffffffu, any_slow)) quotients_by_scale_ieee(v0, v1, scale, group_fast, q);
}

template <bool FP8>
__global__ void __launch_bounds__(kMoveThreads)
dispatch_kernel(MoveParams p, const uint16_t* __restrict__ x, void* __restrict__ recv_x,
                float* __restrict__ recv_scale, float* __restrict__ recv_weight) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t nunits = static_cast<int64_t>(p.T) * p.chunks;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp; u < nunits;
       u += static_cast<int64_t>(gridDim.x) * kMoveWarps) {
    const int t = static_cast<int>(u / p.chunks);
    const int c = static_cast<int>(u - static_cast<int64_t>(t) * p.chunks);
    const int h0 = c * kChunk + lane * kLaneElems;
    const bool a0 = h0 < p.H, a1 = h0 + 8 < p.H;
    const uint16_t* xr = x + static_cast<int64_t>(t) * p.H + h0;
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    if (a0) v0 = ld_ro_v4(xr);
    if (a1) v1 = ld_ro_v4(xr + 8);
    int my_slot = -1;
    float my_w = 0.0f;
    if (lane < p.k) {
      my_slot = p.slot_of_pair[static_cast<int64_t>(t) * p.k + lane];
      my_w = p.topk_weights[static_cast<int64_t>(t) * p.k + lane];
    }
    if constexpr (FP8) {
      float amax = 0.0f;
      {
        float f[16];
        unpack8(v0, f);
        unpack8(v1, f + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
      }
      // 8 consecutive lanes hold one 128-channel group
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
      float scale = __fdiv_rn(amax, kE4M3Max);
      if (scale == 0.0f) scale = 1.0f;
      float f[16];
      quotients_by_scale(v0, v1, scale, f);
      uint32_t q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = pack_e4m3x2(f[4 * i + 0], f[4 * i + 1]);
        const uint32_t hi = pack_e4m3x2(f[4 * i + 2], f[4 * i + 3]);
        q[i] = lo | (hi << 16);
      }
      const uint4 qv = make_uint4(q[0], q[1], q[2], q[3]);
      uint8_t* rx = static_cast<uint8_t*>(recv_x);
      for (int j = 0; j < p.k; ++j) {
        const int s = __shfl_sync(0xffffffffu, my_slot, j);
        if (s >= 0 && a0) {
          st_v4(rx + static_cast<int64_t>(s) * p.H + h0, qv);
          if ((lane & (kLanesPerGroup - 1)) == 0)
            recv_scale[static_cast<int64_t>(s) * p.G + h0 / kGroup] = scale;
        }
      }
    } else {
      uint16_t* rx = static_cast<uint16_t*>(recv_x);
      for (int j = 0; j < p.k; ++j) {
        const int s = __shfl_sync(0xffffffffu, my_slot, j);
        if (s >= 0) {
          uint16_t* dst = rx + static_cast<int64_t>(s) * p.H + h0;
          if (a0) st_v4(dst, v0);
          if (a1) st_v4(dst + 8, v1);
        }
      }
    }
    if (recv_weight != nullptr && c == 0 && lane < p.k && my_slot >= 0) recv_weight[my_slot] = my_w;
  }
}

// -------------------------------------------- combine / dispatch backward
//
// out[t] = bf16( chain over j of (WEIGHTED ? fmaf(w[t,j], y[slot], acc) : acc + y[slot]) )
// with acc = +0.0f and j = 0..k-1 in order.  The k rows are fetched in
// batches of 8 (all loads of a batch issued before the arithmetic).

template <bool WEIGHTED>
__global__ void __launch_bounds__(kMoveThreads)
gather_reduce_kernel(MoveParams p, const uint16_t* __restrict__ y, uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t nunits = static_cast<int64_t>(p.T) * p.chunks;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp; u < nunits;
       u += static_cast<int64_t>(gridDim.x) * kMoveWarps) {
    const int t = static_cast<int>(u / p.chunks);
    const int c = static_cast<int>(u - static_cast<int64_t>(t) * p.chunks);
    const int h0 = c * kChunk + lane * kLaneElems;
    const bool a0 = h0 < p.H, a1 = h0 + 8 < p.H;
    int my_slot = -1;
    float my_w = 0.0f;
    if (lane < p.k) {
      my_slot = p.slot_of_pair[static_cast<int64_t>(t) * p.k + lane];
      if (WEIGHTED) my_w = p.topk_weights[static_cast<int64_t>(t) * p.k + lane];
    }
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
    for (int jb = 0; jb < p.k; jb += 8) {
      uint4 v[8][2];
      int s[8];
      float w[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = (jb + jj) & (kWarp - 1);
        s[jj] = __shfl_sync(0xffffffffu, my_slot, j);
        w[jj] = __shfl_sync(0xffffffffu, my_w, j);
        if (jb + jj >= p.k) s[jj] = -1;
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        v[jj][0] = make_uint4(0, 0, 0, 0);
        v[jj][1] = v[jj][0];
        if (s[jj] >= 0) {
          const uint16_t* src = y + static_cast<int64_t>(s[jj]) * p.H + h0;
          if (a0) v[jj][0] = ld_ro_v4(src);
          if (a1) v[jj][1] = ld_ro_v4(src + 8);
        }
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (s[jj] >= 0) {
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
    }
    uint16_t* dst = out + static_cast<int64_t>(t) * p.H + h0;
    if (a0) st_v4(dst, pack8_bf16(acc));
    if (a1) st_v4(dst + 8, pack8_bf16(acc + 8));
  }
}

// -------------------------------------------------------- combine backward
//
// One CTA per token (grid-stride).  Warps stride over the token's 512-channel
// chunks; for every pair j each lane writes grad_y = bf16(w_j * g) for its 16
// channels and accumulates the partial dot product g . y_j in fp32.  Partial
// sums are reduced across lanes (xor shuffles) and then across warps in warp
// order, so the result does not depend on scheduling.

template <int KMAX>  // 8 (k <= 8) or kMaxK
__global__ void __launch_bounds__(kMoveThreads)
combine_backward_kernel(MoveParams p, const uint16_t* __restrict__ g, const uint16_t* __restrict__ y,
                        uint16_t* __restrict__ grad_y, float* __restrict__ grad_w) {
  __shared__ float part[kMoveWarps][KMAX];
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
  for (int t = blockIdx.x; t < p.T; t += gridDim.x) {
    int my_slot = -1;
    float my_w = 0.0f;
    if (lane < p.k) {
      my_slot = p.slot_of_pair[static_cast<int64_t>(t) * p.k + lane];
      my_w = p.topk_weights[static_cast<int64_t>(t) * p.k + lane];
    }
    float dot[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) dot[j] = 0.0f;
    for (int c = warp; c < p.chunks; c += kMoveWarps) {
      const int h0 = c * kChunk + lane * kLaneElems;
      const bool a0 = h0 < p.H, a1 = h0 + 8 < p.H;
      const uint16_t* gr = g + static_cast<int64_t>(t) * p.H + h0;
      uint4 gv0 = make_uint4(0, 0, 0, 0), gv1 = gv0;
      if (a0) gv0 = ld_ro_v4(gr);
      if (a1) gv1 = ld_ro_v4(gr + 8);
      float gf[16];
      unpack8(gv0, gf);
      unpack8(gv1, gf + 8);
#pragma unroll
      for (int jb = 0; jb < KMAX; jb += 8) {
        if (jb < p.k) {
          uint4 v[8][2];
          int s[8];
          float w[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            s[jj] = __shfl_sync(0xffffffffu, my_slot, jb + jj);
            w[jj] = __shfl_sync(0xffffffffu, my_w, jb + jj);
            if (jb + jj >= p.k) s[jj] = -1;
          }
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            v[jj][0] = make_uint4(0, 0, 0, 0);
            v[jj][1] = v[jj][0];
            if (s[jj] >= 0) {
              const uint16_t* src = y + static_cast<int64_t>(s[jj]) * p.H + h0;
              if (a0) v[jj][0] = ld_ro_v4(src);
              if (a1) v[jj][1] = ld_ro_v4(src + 8);
            }
          }
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            if (s[jj] >= 0) {
              float yf[16], gy[16];
              unpack8(v[jj][0], yf);
              unpack8(v[jj][1], yf + 8);
              float d = dot[jb + jj];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                gy[i] = __fmul_rn(w[jj], gf[i]);
                d = fmaf(gf[i], yf[i], d);
              }
              dot[jb + jj] = d;
              uint16_t* dst = grad_y + static_cast<int64_t>(s[jj]) * p.H + h0;
              if (a0) st_v4(dst, pack8_bf16(gy));
              if (a1) st_v4(dst + 8, pack8_bf16(gy + 8));
            }
          }
        }
      }
    }
    // reduce the partial dot products: lanes, then warps in order
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < p.k) {
        float d = dot[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) part[warp][j] = d;
      }
    }
    __syncthreads();
    if (threadIdx.x < p.k) {
      const int j = threadIdx.x;
      float d = 0.0f;
      for (int w = 0; w < kMoveWarps; ++w) d += part[w][j];
      grad_w[static_cast<int64_t>(t) * p.k + j] = my_slot >= 0 ? d : 0.0f;
    }
    __syncthreads();
  }
}

}  // namespace ep
