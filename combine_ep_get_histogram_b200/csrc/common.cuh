// Device helpers shared by the layout and data-movement kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ep {

constexpr int kWarp = 32;
constexpr int kMaxK = 32;
constexpr int kMaxE = 1024;
constexpr int kMaxR = 256;
constexpr int kGroup = 128;                   // channels per FP8 scale
constexpr int kLaneElems = 16;                // channels a lane moves per chunk
constexpr int kChunk = kWarp * kLaneElems;    // 512 channels per warp chunk
// A lane's 16 channels of a chunk are two 8-channel pieces (16 bytes of
// bf16 each) half a chunk apart: lane l holds [c*512 + 8l, +8) and
// [c*512 + 256 + 8l, +8), so each 16-byte load or store of the warp covers
// 512 contiguous bytes (16 sectors per request), and an FP8 scale group (128
// channels) is one half-warp's pieces.
constexpr int kPieceElems = 8;
constexpr int kHalfChunk = kChunk / 2;        // 256: offset of a lane's second piece
constexpr int kLanesPerGroup = kGroup / kPieceElems;  // 16
constexpr int kTilePairs = 1024;              // layout tile: pairs per CTA
constexpr int kTileFlagBytes = 32768;         // layout tile: tokens x ranks flag bytes
constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / kWarp;
constexpr int kMaxChunksPerWarp = (kTilePairs / kLayoutWarps + kWarp - 1) / kWarp;  // 4
constexpr int kPairsPerThread = kTilePairs / kLayoutThreads;                         // 4
constexpr float kE4M3Max = 448.0f;

// 16-byte load of data that no thread writes during the kernel: non-coherent
// path, no L1 allocation, 256-byte L2 prefetch (the aggressive load the pages
// describe, used only on read-only inputs).
__device__ __forceinline__ uint4 ld_ro_v4(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// 16-byte load of read-only data that other warps of the CTA read too: cached in L1.
__device__ __forceinline__ uint4 ld_l1_v4(const void* p) {
  uint4 v;
  asm("ld.global.ca.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  *reinterpret_cast<uint4*>(p) = v;
}

// L2 policy that marks written lines first in line for eviction.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte store with an L2 cache policy.  No memory clobber: callers use it
// only for outputs that no load of the same kernel reads.
__device__ __forceinline__ void st_v4_hint(void* p, uint4 v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1,%2,%3,%4}, %5;"
               :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(policy));
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Two fp32 values -> packed bf16x2 (round to nearest even); `lo` lands in the
// low half, which is the lower address in memory.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 values -> packed E4M3 codes (round to nearest even, saturating to
// +-448); `lo` lands in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ uint4 pack8_bf16(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                    pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}

// First channel of a lane's first piece in chunk c (the second is kHalfChunk further).
__device__ __forceinline__ int piece_channel(int c, int lane) { return c * kChunk + lane * kPieceElems; }

// Eight fp32 values -> eight E4M3 codes, channel order in memory order.
__device__ __forceinline__ uint2 pack8_e4m3(const float* f) {
  return make_uint2(pack_e4m3x2(f[0], f[1]) | (pack_e4m3x2(f[2], f[3]) << 16),
                    pack_e4m3x2(f[4], f[5]) | (pack_e4m3x2(f[6], f[7]) << 16));
}

// Programmatic dependent launch.  The host launches every kernel of the
// library with programmatic stream serialization (unless EP_PDL=0), and
// every kernel opens with the same three steps:
//   1. pdl_allow_next(): the next kernel on the stream may be scheduled now,
//      so its CTAs take SM slots as this grid's CTAs retire, instead of after
//      the last one;
//   2. optional L2 prefetches of the lines the kernel reads first: a prefetch
//      writes nothing and returns nothing to the thread, so it is harmless
//      while the previous kernel may still be writing those lines;
//   3. pdl_wait_prev(): blocks until the previous kernel on the stream has
//      completed and its memory writes are visible.
// Every global load and store of a kernel comes after step 3, so a kernel
// never reads data its predecessor has not finished writing, and never
// overwrites data its predecessor may still read.  Without the launch
// attribute both instructions do nothing.
__device__ __forceinline__ void pdl_allow_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_prev() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Brings the 128-byte lines of [p, p + bytes) into L2, one line per thread
// (thread `tid` of `nthreads`).  Every address lies inside the range.
__device__ __forceinline__ void prefetch_l2(const void* p, int64_t bytes, int tid, int nthreads) {
  if (bytes <= 0) return;
  const char* c = static_cast<const char*>(p);
  const int64_t first = reinterpret_cast<uintptr_t>(c) & 127;  // offset of p in its line
  for (int64_t off = static_cast<int64_t>(tid) * 128 - first; off < bytes; off += static_cast<int64_t>(nthreads) * 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(c + (off < 0 ? 0 : off)));
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

}  // namespace ep
