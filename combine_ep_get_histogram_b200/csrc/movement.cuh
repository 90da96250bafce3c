// Data movement: dispatch (BF16 copy or fused FP8 E4M3 quantisation), combine,
// combine backward and dispatch backward.
//
// Operations (pages: "DeepEP：MoE 专家并行 EP 通信 kernel 编译与使用指南",
// section 五 使用方法 and FAQ Q5 — dispatch scatters tokens to experts,
// combine gathers the expert outputs back and sums them, the forward handle
// serves both backward passes; FP8 dispatch + BF16 combine:
// "deepep-expert-parallel-communication-library", section 五 实践建议;
// conversion fused into the movement: "DeepEP：专为MoE模型打造的All-to-All
// 通信库", section 3.2).
//
// All four kernels are HBM-bound streams.  Work unit = one warp x one token x
// one 512-channel chunk: each lane moves 16 channels as two 8-channel pieces
// half a chunk apart (piece_channel), so every 16-byte access of the warp
// covers 512 contiguous bytes of bf16 (256 of E4M3): 16 sectors per request.
// A warp reads or writes 1 KiB of bf16 (512 B of E4M3) per row, and an FP8
// scale group (128 channels) is one half-warp's pieces.  Grids are capped at
// (SMs x resident CTAs) and stride over the units.  Read-only inputs use
// non-coherent, L1-no-allocate loads.
#pragma once

#include "common.cuh"

namespace ep {

struct MoveParams {
  int T, H, k, G;
  int chunks;  // ceil(H / kChunk)
  int pdl;     // 1: launched with programmatic dependent launch: the kernel runs the
               // prologue of common.cuh (allow the next kernel, prefetch, wait);
               // 0: it skips it
  const int32_t* slot_of_pair;
  const float* topk_weights;
};

constexpr int kMoveThreads = 256;
constexpr int kMoveWarps = kMoveThreads / kWarp;

// ---------------------------------------------------------------- dispatch

// The IEEE-division fallback of quotients_by_scale, out of line: it runs
// only for groups or elements outside the fast path's range.
struct Quot8 {
  float v[8];
};

__device__ __noinline__ Quot8 quotients_ieee(uint4 v, float scale, bool group_fast, Quot8 q) {
  float f[8];
  unpack8(v, f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t mag = __float_as_uint(f[i]) & 0x7FFFFFFFu;
    if (!(group_fast && (mag >= 0x0B000000u || mag == 0u))) q.v[i] = __fdiv_rn(f[i], scale);
  }
  return q;
}

// q[i] <- x_i / scale, rounded to nearest even in fp32, for the 8 values of
// one piece (scale >= the group's amax / 448).  Every lane of the warp calls
// it together.
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
__device__ __forceinline__ void quotients_by_scale(const uint4& v, float scale, float* q) {
  float f[8];
  unpack8(v, f);
  const float r = __frcp_rn(scale);
  const bool group_fast = scale >= 1.17549435e-38f && r <= 3.40282347e+38f;
  bool any_slow = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t b = __float_as_uint(f[i]);
    const uint32_t mag = b & 0x7FFFFFFFu;
    any_slow |= !(group_fast && (mag >= 0x0B000000u || mag == 0u));
    const float ax = __uint_as_float(mag);
    const float q0 = __fmul_rn(ax, r);
    const float e = fmaf(-q0, scale, ax);
    q[i] = __uint_as_float(__float_as_uint(fmaf(e, r, q0)) | (b & 0x80000000u));
  }
  if (__any_sync(0xffffffffu, any_slow)) {
    Quot8 in;
#pragma unroll
    for (int i = 0; i < 8; ++i) in.v[i] = q[i];
    const Quot8 out = quotients_ieee(v, scale, group_fast, in);
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = out.v[i];
  }
}

// Largest |x| of the 128-channel group a piece belongs to: the piece's 8
// values, then the 16 lanes of the half-warp that hold the group.
__device__ __forceinline__ float group_amax(const uint4& v) {
  float f[8];
  unpack8(v, f);
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[i]));
#pragma unroll
  for (int o = 1; o < kLanesPerGroup; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  return a;
}

// The FP8 encoding of one piece: the group's scale (amax / 448, or 1 when
// amax / 448 is 0) and the 8 E4M3 codes of x / scale.
__device__ __forceinline__ uint2 quantize_piece(const uint4& v, float& scale) {
  scale = __fdiv_rn(group_amax(v), kE4M3Max);
  if (scale == 0.0f) scale = 1.0f;
  float f[8];
  quotients_by_scale(v, scale, f);
  return pack8_e4m3(f);
}

template <bool FP8>
__global__ void __launch_bounds__(kMoveThreads)
dispatch_kernel(MoveParams p, const uint16_t* __restrict__ x, void* __restrict__ recv_x,
                float* __restrict__ recv_scale, float* __restrict__ recv_weight) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t nunits = static_cast<int64_t>(p.T) * p.chunks;
  if (p.pdl) pdl_allow_next();
  if (p.pdl) pdl_wait_prev();
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
    int my_slot = -1;
    float my_w = 0.0f;
    if (lane < p.k) {
      my_slot = p.slot_of_pair[static_cast<int64_t>(t) * p.k + lane];
      my_w = p.topk_weights[static_cast<int64_t>(t) * p.k + lane];
    }
    if constexpr (FP8) {
      float sc0, sc1;
      const uint2 q0 = quantize_piece(v0, sc0);
      const uint2 q1 = quantize_piece(v1, sc1);
      const bool scale_lane = (lane & (kLanesPerGroup - 1)) == 0;
      uint8_t* rx = static_cast<uint8_t*>(recv_x);
      for (int j = 0; j < p.k; ++j) {
        const int s = __shfl_sync(0xffffffffu, my_slot, j);
        if (s < 0) continue;
        uint8_t* row = rx + static_cast<int64_t>(s) * p.H;
        float* srow = recv_scale + static_cast<int64_t>(s) * p.G;
        if (a0) {
          *reinterpret_cast<uint2*>(row + h0) = q0;
          if (scale_lane) srow[h0 / kGroup] = sc0;
        }
        if (a1) {
          *reinterpret_cast<uint2*>(row + h1) = q1;
          if (scale_lane) srow[h1 / kGroup] = sc1;
        }
      }
    } else {
      uint16_t* rx = static_cast<uint16_t*>(recv_x);
      for (int j = 0; j < p.k; ++j) {
        const int s = __shfl_sync(0xffffffffu, my_slot, j);
        if (s >= 0) {
          uint16_t* row = rx + static_cast<int64_t>(s) * p.H;
          if (a0) st_v4(row + h0, v0);
          if (a1) st_v4(row + h1, v1);
        }
      }
    }
    if (recv_weight != nullptr && c == 0 && lane < p.k && my_slot >= 0) recv_weight[my_slot] = my_w;
  }
}

// ------------------------------------------------- dispatch, TMA row stores
//
// One CTA per token (grid-stride over tokens), one warp per 512-channel chunk
// (4 <= chunks <= 16, i.e. 1536 < H <= 8192).  Each token's payload row (E4M3
// codes, or the bf16 row itself) is assembled in shared memory and written to
// its k receive rows by k TMA bulk copies (cp.async.bulk global <- shared)
// issued by one thread, so every destination row is written as one
// contiguous H- or 2H-byte transfer instead of 512-byte pieces from many
// warps.  2 or 3 row stages rotate; before a stage is rewritten, the issuing
// thread waits until the bulk copies that last read it have finished
// (cp.async.bulk.wait_group.read).  The next token's x is loaded into
// registers while the current one is quantised and stored.  Scales and gate
// weights are written with plain stores from shared memory.

constexpr int kTmaMinChunks = 4;
constexpr int kTmaMaxChunks = 16;

struct TmaSmemLayout {
  int row_bytes;   // payload row bytes, rounded up to 128
  int stages;      // payload row stages (2..3): as many as fit in kTmaRowBudget
  int nbuf;        // slot / weight / scale buffers: 2, or one per row stage (early form)
  int off_slot;    // int32 [nbuf][kMaxK]
  int off_w;       // float [nbuf][kMaxK]
  int off_scale;   // float [nbuf][G]
  int total;
};

constexpr int kTmaRowBudget = 40 * 1024;
constexpr int kTmaMaxStages = 3;

__host__ __device__ inline TmaSmemLayout tma_smem_layout(int H, bool fp8, bool early = false) {
  TmaSmemLayout L;
  const int row = fp8 ? H : 2 * H;
  L.row_bytes = (row + 127) / 128 * 128;
  L.stages = kTmaRowBudget / L.row_bytes;
  L.stages = L.stages < 2 ? 2 : (L.stages > kTmaMaxStages ? kTmaMaxStages : L.stages);
  L.nbuf = early ? L.stages : 2;
  L.off_slot = L.stages * L.row_bytes;
  L.off_w = L.off_slot + L.nbuf * kMaxK * 4;
  L.off_scale = L.off_w + L.nbuf * kMaxK * 4;
  L.total = L.off_scale + (fp8 ? L.nbuf * (H / kGroup) * 4 : 0);
  return L;
}

// Waits until at most stages-1 bulk-copy groups of this thread still read shared memory.
__device__ __forceinline__ void bulk_wait_read_all_but(int n) {
  if (n >= 3) asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory");
  else if (n == 2) asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory");
  else asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ void bulk_store_row(void* gdst, uint32_t ssrc, int bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               :: "l"(gdst), "r"(ssrc), "r"(bytes) : "memory");
}

// One token's x chunk, quantised (FP8) or copied (BF16) into its row stage,
// with its scales into sscale.
template <bool FP8>
__device__ __forceinline__ void tma_stage_row(uint8_t* row, float* sscale, const uint4& v0, const uint4& v1, int h0,
                                              int h1, bool a0, bool a1, int lane) {
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
}

// EARLY (the fused layout + dispatch call under programmatic launch): the
// kernel before this one is the call's own layout, which lets this kernel be
// scheduled only after its own wait, so every kernel before the call has
// completed and x is final; the layout does not write x.  Each CTA then loads
// and quantises its first tokens, one per row stage, before waiting for the
// layout, and sends them once their slots are known.
template <bool FP8, bool EARLY>
__global__ void __launch_bounds__(kTmaMaxChunks * kWarp, 3)
dispatch_tma_kernel(MoveParams p, const uint16_t* __restrict__ x, void* __restrict__ recv_x,
                    float* __restrict__ recv_scale, float* __restrict__ recv_weight) {
  extern __shared__ __align__(128) uint8_t tma_smem[];
  const TmaSmemLayout L = tma_smem_layout(p.H, FP8, EARLY);
  const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
  const int h0 = piece_channel(warp, lane), h1 = h0 + kHalfChunk;  // one chunk per warp
  const bool a0 = h0 < p.H, a1 = h1 < p.H;
  const int row_bytes = FP8 ? p.H : 2 * p.H;

  uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
  int t = blockIdx.x;
  int it0 = 0;
  // no prefetch in this prologue: its code cost the kernel a register spill
  // and 2-3 % at full batch
  if (p.pdl) pdl_allow_next();
  if constexpr (EARLY) {
    int n_pre = 0;  // this CTA's tokens staged before the wait (CTA-uniform)
    while (n_pre < L.stages && t + n_pre * static_cast<int>(gridDim.x) < p.T) ++n_pre;
    if (n_pre > 0) {
      const uint16_t* xr = x + static_cast<int64_t>(t) * p.H;
      if (a0) v0 = ld_ro_v4(xr + h0);
      if (a1) v1 = ld_ro_v4(xr + h1);
    }
    for (int i = 0; i < n_pre; ++i) {
      uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
      if (i + 1 < n_pre) {
        const uint16_t* xr = x + static_cast<int64_t>(t + (i + 1) * static_cast<int>(gridDim.x)) * p.H;
        if (a0) n0 = ld_ro_v4(xr + h0);
        if (a1) n1 = ld_ro_v4(xr + h1);
      }
      tma_stage_row<FP8>(tma_smem + i * L.row_bytes,
                         reinterpret_cast<float*>(tma_smem + L.off_scale) + i * p.G, v0, v1, h0, h1, a0, a1, lane);
      v0 = n0;
      v1 = n1;
    }
    if (p.pdl) pdl_wait_prev();
    if (n_pre > 0) {
      // warp i reads the slots and gate weights of staged token i
      if (warp < n_pre && lane < p.k) {
        const int64_t pr = static_cast<int64_t>(t + warp * static_cast<int>(gridDim.x)) * p.k + lane;
        reinterpret_cast<int32_t*>(tma_smem + L.off_slot)[warp * kMaxK + lane] = p.slot_of_pair[pr];
        reinterpret_cast<float*>(tma_smem + L.off_w)[warp * kMaxK + lane] = p.topk_weights[pr];
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      const int32_t* sslot = reinterpret_cast<const int32_t*>(tma_smem + L.off_slot);
      if (threadIdx.x == 0) {
        for (int i = 0; i < n_pre; ++i) {  // one bulk group per token, as in the loop below
          const uint32_t src = static_cast<uint32_t>(__cvta_generic_to_shared(tma_smem + i * L.row_bytes));
          for (int j = 0; j < p.k; ++j) {
            const int s = sslot[i * kMaxK + j];
            if (s >= 0) bulk_store_row(static_cast<uint8_t*>(recv_x) + static_cast<int64_t>(s) * row_bytes, src,
                                       row_bytes);
          }
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
      }
      if constexpr (FP8) {
        const float* sscale = reinterpret_cast<const float*>(tma_smem + L.off_scale);
        for (int i = threadIdx.x; i < n_pre * p.k * p.G; i += blockDim.x) {
          const int tj = i / p.G, g = i - tj * p.G;  // tj = token * k + j
          const int s = sslot[(tj / p.k) * kMaxK + tj % p.k];
          if (s >= 0) recv_scale[static_cast<int64_t>(s) * p.G + g] = sscale[(tj / p.k) * p.G + g];
        }
      }
      if (recv_weight != nullptr && threadIdx.x < n_pre * p.k) {
        const int i = threadIdx.x / p.k, j = threadIdx.x - i * p.k;
        const int s = sslot[i * kMaxK + j];
        if (s >= 0) recv_weight[s] = reinterpret_cast<const float*>(tma_smem + L.off_w)[i * kMaxK + j];
      }
    }
    it0 = n_pre;
    t += n_pre * static_cast<int>(gridDim.x);
    v0 = v1 = make_uint4(0, 0, 0, 0);
  } else {
    if (p.pdl) pdl_wait_prev();
  }
  if (t < p.T) {
    const uint16_t* xr = x + static_cast<int64_t>(t) * p.H;
    if (a0) v0 = ld_ro_v4(xr + h0);
    if (a1) v1 = ld_ro_v4(xr + h1);
  }
  for (int it = it0; t < p.T; ++it, t += gridDim.x) {
    const int stage = EARLY ? it % L.nbuf : (it & 1);
    uint8_t* row = tma_smem + (it % L.stages) * L.row_bytes;
    int32_t* sslot = reinterpret_cast<int32_t*>(tma_smem + L.off_slot) + stage * kMaxK;
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

    tma_stage_row<FP8>(row, sscale, v0, v1, h0, h1, a0, a1, lane);
    // the slots and weights after the quantisation: read before it, their
    // load held every warp at a barrier (decode dispatch 18.4 -> 16.9 us)
    if (warp == 0 && lane < p.k) {
      sslot[lane] = p.slot_of_pair[static_cast<int64_t>(t) * p.k + lane];
      sw[lane] = p.topk_weights[static_cast<int64_t>(t) * p.k + lane];
    }
    // make the generic-proxy shared-memory writes visible to the bulk copies
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();

    if (threadIdx.x == 0) {
      const uint32_t src = static_cast<uint32_t>(__cvta_generic_to_shared(row));
      for (int j = 0; j < p.k; ++j) {
        const int s = sslot[j];
        if (s >= 0) bulk_store_row(static_cast<uint8_t*>(recv_x) + static_cast<int64_t>(s) * row_bytes, src,
                                   row_bytes);
      }
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    if constexpr (FP8) {
      for (int i = threadIdx.x; i < p.k * p.G; i += blockDim.x) {
        const int j = i / p.G, g = i - j * p.G;
        const int s = sslot[j];
        if (s >= 0) recv_scale[static_cast<int64_t>(s) * p.G + g] = sscale[g];
      }
    }
    if (recv_weight != nullptr && threadIdx.x < p.k) {
      const int s = sslot[threadIdx.x];
      if (s >= 0) recv_weight[s] = sw[threadIdx.x];
    }
    v0 = n0;
    v1 = n1;
  }
  if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// -------------------------------------------- combine / dispatch backward
//
// out[t] = bf16( chain over j of (WEIGHTED ? fmaf(w[t,j], y[slot], acc) : acc + y[slot]) )
// with acc = +0.0f and j = 0..k-1 in order.  The k rows are fetched in
// batches of 8 (all loads of a batch issued before the arithmetic).

// RAGGED (H not a multiple of 512): every piece is checked against H.
// Otherwise every piece lies inside the row and no check is made; a kernel
// that carries both paths was measured slower even on full chunks, so the
// host launches the variant the shape needs.
template <bool WEIGHTED, bool RAGGED>
__global__ void __launch_bounds__(kMoveThreads)
gather_reduce_kernel(MoveParams p, const uint16_t* __restrict__ y, uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t nunits = static_cast<int64_t>(p.T) * p.chunks;
  if (p.pdl) pdl_allow_next();
  {  // the first unit's slots (and weights) are this warp's first loads
    const int64_t u0 = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp;
    if (p.pdl && u0 < nunits && lane == 0) {
      const int64_t pair0 = (u0 / p.chunks) * p.k;
      prefetch_l2(p.slot_of_pair + pair0, 4 * p.k, 0, 1);
      if (WEIGHTED) prefetch_l2(p.topk_weights + pair0, 4 * p.k, 0, 1);
    }
  }
  if (p.pdl) pdl_wait_prev();
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp; u < nunits;
       u += static_cast<int64_t>(gridDim.x) * kMoveWarps) {
    const int t = static_cast<int>(u / p.chunks);
    const int c = static_cast<int>(u - static_cast<int64_t>(t) * p.chunks);
    const int h0 = piece_channel(c, lane), h1 = h0 + kHalfChunk;
    const bool a0 = !RAGGED || h0 < p.H, a1 = !RAGGED || h1 < p.H;
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
          const uint16_t* src = y + static_cast<int64_t>(s[jj]) * p.H;
          if (a0) v[jj][0] = ld_ro_v4(src + h0);
          if (a1) v[jj][1] = ld_ro_v4(src + h1);
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
    uint16_t* dst = out + static_cast<int64_t>(t) * p.H;
    if (a0) st_v4(dst + h0, pack8_bf16(acc));
    if (a1) st_v4(dst + h1, pack8_bf16(acc + 8));
  }
}

// -------------------------------------------------------- combine backward
//
// One warp per (token t, top-k position j) pair, grid-stride over the pairs:
// the warp streams the whole y[slot] row in and the whole grad_y[slot] row
// out, kCbwdUnroll 512-channel chunks at a time, and reads g[t] through L1 (the
// k warps of one token usually share a CTA, so g comes from DRAM once).
// grad_y = bf16(w * g) (one fp32 product).  The dot product g . y[slot]
// keeps kCbwdUnroll fp32 partial sums per lane, one per chunk slot of an
// unrolled group (four independent fma chains instead of one: measured about
// 3 % faster at 7168 and 4096 channels), adds them, then reduces across lanes
// with xor shuffles, so grad_w needs no cross-warp reduction and does not
// depend on scheduling.  grad_y is written with an L2 evict-first policy: it is not read
// again here, and letting it leave L2 first keeps the y rows being read from
// being pushed out.

constexpr int kCbwdUnroll = 4;
static_assert(kCbwdUnroll == 4, "the partial sums below are added as two pairs");

// RAGGED (H not a multiple of 512): every piece is checked against H;
// otherwise one check per chunk covers both pieces (6 % faster than
// checking each piece, and the host launches the variant the shape needs).
template <bool RAGGED>
__global__ void __launch_bounds__(kMoveThreads)
combine_backward_kernel(MoveParams p, const uint16_t* __restrict__ g, const uint16_t* __restrict__ y,
                        uint16_t* __restrict__ grad_y, float* __restrict__ grad_w) {
  const uint64_t evict_first = l2_evict_first_policy();
  const int lane = threadIdx.x & (kWarp - 1);
  const int64_t npairs = static_cast<int64_t>(p.T) * p.k;
  if (p.pdl) pdl_allow_next();
  {  // the first pair's slot, weight and grad_out row are this warp's first loads
    const int64_t u0 = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp;
    if (p.pdl && u0 < npairs) {
      if (lane == 0) {
        prefetch_l2(p.slot_of_pair + u0, 4, 0, 1);
        prefetch_l2(p.topk_weights + u0, 4, 0, 1);
      }
      // one warp per token brings its grad_out row (the token's k pairs share it)
      if (u0 % p.k == 0 || threadIdx.x < kWarp)
        prefetch_l2(g + (u0 / p.k) * p.H, 2 * static_cast<int64_t>(p.H), lane, kWarp);
    }
  }
  if (p.pdl) pdl_wait_prev();
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kMoveWarps + threadIdx.x / kWarp; u < npairs;
       u += static_cast<int64_t>(gridDim.x) * kMoveWarps) {
    const int s = p.slot_of_pair[u];
    if (s < 0) {  // masked pair: no row, zero weight gradient
      if (lane == 0) grad_w[u] = 0.0f;
      continue;
    }
    const float w = p.topk_weights[u];
    const int t = static_cast<int>(u / p.k);
    const uint16_t* gr = g + static_cast<int64_t>(t) * p.H;
    const uint16_t* yr = y + static_cast<int64_t>(s) * p.H;
    uint16_t* dr = grad_y + static_cast<int64_t>(s) * p.H;
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
            yv[q][0] = ld_ro_v4(yr + h0);
          }
          if (!RAGGED || h1 < p.H) {
            gv[q][1] = ld_l1_v4(gr + h1);
            yv[q][1] = ld_ro_v4(yr + h1);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < kCbwdUnroll; ++q) {
        const int h0 = piece_channel(c0 + q, lane), h1 = h0 + kHalfChunk;
        uint4 out[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t gw[4] = {gv[q][h].x, gv[q][h].y, gv[q][h].z, gv[q][h].w};
          const uint32_t yw[4] = {yv[q][h].x, yv[q][h].y, yv[q][h].z, yv[q][h].w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float g0 = bf16_lo(gw[i]), g1 = bf16_hi(gw[i]);
            d[q] = fmaf(g0, bf16_lo(yw[i]), d[q]);
            d[q] = fmaf(g1, bf16_hi(yw[i]), d[q]);
            o[i] = pack_bf16x2(__fmul_rn(w, g0), __fmul_rn(w, g1));
          }
          out[h] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (c0 + q < p.chunks) {
          if (!RAGGED || h0 < p.H) st_v4_hint(dr + h0, out[0], evict_first);
          if (!RAGGED || h1 < p.H) st_v4_hint(dr + h1, out[1], evict_first);
        }
      }
    }
    float dot = (d[0] + d[1]) + (d[2] + d[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) grad_w[u] = dot;
  }
}

}  // namespace ep
