// C ABI of libep_b200.so (declared in include/ep.h): argument checks on the
// host, launch configuration, status codes.  Every step runs in the kernels of
// layout.cuh (routing layout), movement.cuh (dispatch, combine, backward
// passes), route.cuh (group-limited routing) and peers.cuh (the multi-GPU
// forms); nothing here touches data.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "ep.h"
#include "layout.cuh"
#include "movement.cuh"
#include "peers.cuh"
#include "route.cuh"

namespace {

using namespace ep;

thread_local char g_last_cuda_error[256] = "";

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return EP_OK;
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return EP_ERR_CUDA;
}

bool debug_mode() {
  static const bool on = [] {
    const char* s = std::getenv("EP_DEBUG");
    return s != nullptr && s[0] == '1';
  }();
  return on;
}

// Per-device facts, read once.
struct DeviceInfo {
  int sms = 0;
  bool supported = false;
  int occ_count = 0, occ_scan = 0, occ_assign = 0;
  int occ_disp_bf16 = 0, occ_disp_fp8 = 0;
  int occ_comb[2] = {}, occ_dbwd[2] = {};  // [ragged]
  int occ_tma[2][2][kTmaMaxChunks + 1] = {};  // [early][fp8][chunks], filled on first use
  int occ_tma_peers[2][kTmaMaxChunks + 1] = {};  // the same for dispatch_tma_peers_kernel
  int occ_cbwd[2] = {};  // [ragged]
  int occ_peer_disp[2] = {}, occ_peer_gather[2][2] = {}, occ_peer_cbwd[2] = {};  // [fp8], [weighted][ragged], [ragged]
  int occ_route[6] = {};          // route_group_limited_kernel<1, 2, 4, 8, 16, 32>
  int occ_route_aligned[6] = {};  // route_aligned_kernel<1, 2, 4, 8, 16, 32>
  int occ_route_compact[6][5] = {};  // route_compact_kernel<2^i, 2^j>, filled on first use
  int small_cluster = 0;             // cluster size of layout_small_kernel, chosen on first use
};

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_ready[kMaxDevices] = {};

int occupancy(const void* fn, int threads, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

// Cluster size of the one-launch layout on this device: the wide (16-CTA,
// non-portable) cluster when the device can hold one with the kernel's
// largest shared memory, else the portable 8.  The choice is made once per
// device, in the first context that runs the layout (EP_LAYOUT_CLUSTER=8
// keeps the portable size for a context with fewer SMs).  The non-portable
// size needs a function attribute, which belongs to the current context, so
// the launch sets it again every time.
int small_cluster_size(const DeviceInfo* d) {
  std::lock_guard<std::mutex> lock(g_dev_mu);
  int& c = const_cast<DeviceInfo*>(d)->small_cluster;
  if (c == 0) {
    const char* env = std::getenv("EP_LAYOUT_CLUSTER");  // "8": keep the portable size
    if (env != nullptr && std::strcmp(env, "8") == 0) return c = kClusterCtas;
    const cudaError_t before = cudaPeekAtLastError();
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kClusterCtasWide);
    cfg.blockDim = dim3(kSmallThreads);
    cfg.dynamicSmemBytes = kSmallMaxSmem;
    const bool ok = cudaFuncSetAttribute(layout_small_kernel<kClusterCtasWide>,
                                         cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
                    cudaOccupancyMaxActiveClusters(&n, layout_small_kernel<kClusterCtasWide>, &cfg) == cudaSuccess;
    if (!ok && before == cudaSuccess) (void)cudaGetLastError();  // the query's own error only
    c = ok && n > 0 ? kClusterCtasWide : kClusterCtas;
  }
  return c;
}

int device_info(const DeviceInfo** out) {
  int dev = 0;
  int st = cuda_status(cudaGetDevice(&dev));
  if (st != EP_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return EP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (!g_dev_ready[dev]) {
    DeviceInfo d;
    cudaDeviceProp prop;
    st = cuda_status(cudaGetDeviceProperties(&prop, dev));
    if (st != EP_OK) return st;
    d.sms = prop.multiProcessorCount;
    d.supported = prop.major == 10 && prop.minor == 0;
    if (d.supported) {
      cudaFuncSetAttribute(reinterpret_cast<const void*>(layout_padded_kernel<true>),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, kPadMaxSmem);
      cudaFuncSetAttribute(reinterpret_cast<const void*>(layout_padded_kernel<false>),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, kPadMaxSmem);
      d.occ_count = occupancy(reinterpret_cast<const void*>(layout_count_kernel), kLayoutThreads,
                              (kMaxE + kMaxR) * 4 + kTileFlagBytes);
      d.occ_disp_bf16 = occupancy(reinterpret_cast<const void*>(dispatch_kernel<false>), kMoveThreads, 0);
      d.occ_disp_fp8 = occupancy(reinterpret_cast<const void*>(dispatch_kernel<true>), kMoveThreads, 0);
      d.occ_comb[0] = occupancy(reinterpret_cast<const void*>(gather_reduce_kernel<true, false>), kMoveThreads, 0);
      d.occ_comb[1] = occupancy(reinterpret_cast<const void*>(gather_reduce_kernel<true, true>), kMoveThreads, 0);
      d.occ_dbwd[0] = occupancy(reinterpret_cast<const void*>(gather_reduce_kernel<false, false>), kMoveThreads, 0);
      d.occ_dbwd[1] = occupancy(reinterpret_cast<const void*>(gather_reduce_kernel<false, true>), kMoveThreads, 0);
      d.occ_cbwd[0] = occupancy(reinterpret_cast<const void*>(combine_backward_kernel<false>), kMoveThreads, 0);
      d.occ_cbwd[1] = occupancy(reinterpret_cast<const void*>(combine_backward_kernel<true>), kMoveThreads, 0);
      d.occ_peer_disp[0] = occupancy(reinterpret_cast<const void*>(dispatch_peers_kernel<false>), kMoveThreads, 0);
      d.occ_peer_disp[1] = occupancy(reinterpret_cast<const void*>(dispatch_peers_kernel<true>), kMoveThreads, 0);
      d.occ_peer_gather[0][0] =
          occupancy(reinterpret_cast<const void*>(gather_reduce_peers_kernel<false, false>), kMoveThreads, 0);
      d.occ_peer_gather[0][1] =
          occupancy(reinterpret_cast<const void*>(gather_reduce_peers_kernel<false, true>), kMoveThreads, 0);
      d.occ_peer_gather[1][0] =
          occupancy(reinterpret_cast<const void*>(gather_reduce_peers_kernel<true, false>), kMoveThreads, 0);
      d.occ_peer_gather[1][1] =
          occupancy(reinterpret_cast<const void*>(gather_reduce_peers_kernel<true, true>), kMoveThreads, 0);
      d.occ_peer_cbwd[0] =
          occupancy(reinterpret_cast<const void*>(combine_backward_peers_kernel<false>), kMoveThreads, 0);
      d.occ_peer_cbwd[1] =
          occupancy(reinterpret_cast<const void*>(combine_backward_peers_kernel<true>), kMoveThreads, 0);
      const void* route_fns[6] = {reinterpret_cast<const void*>(route_group_limited_kernel<1>),
                                  reinterpret_cast<const void*>(route_group_limited_kernel<2>),
                                  reinterpret_cast<const void*>(route_group_limited_kernel<4>),
                                  reinterpret_cast<const void*>(route_group_limited_kernel<8>),
                                  reinterpret_cast<const void*>(route_group_limited_kernel<16>),
                                  reinterpret_cast<const void*>(route_group_limited_kernel<32>)};
      const void* aligned_fns[6] = {reinterpret_cast<const void*>(route_aligned_kernel<1>),
                                    reinterpret_cast<const void*>(route_aligned_kernel<2>),
                                    reinterpret_cast<const void*>(route_aligned_kernel<4>),
                                    reinterpret_cast<const void*>(route_aligned_kernel<8>),
                                    reinterpret_cast<const void*>(route_aligned_kernel<16>),
                                    reinterpret_cast<const void*>(route_aligned_kernel<32>)};
      for (int i = 0; i < 6; ++i) {
        d.occ_route[i] = occupancy(route_fns[i], kRouteThreads, 0);
        d.occ_route_aligned[i] = occupancy(aligned_fns[i], kRouteThreads, 0);
      }
      cudaGetLastError();
    }
    g_dev[dev] = d;
    g_dev_ready[dev] = true;
  }
  if (!g_dev[dev].supported) return EP_ERR_UNSUPPORTED;
  *out = &g_dev[dev];
  return EP_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(const ep_shape_t* s) {
  if (s == nullptr) return EP_ERR_INVALID_ARG;
  if (s->T < 0 || s->k < 1 || s->k > kMaxK || s->E < 1 || s->E > kMaxE || s->R < 1 ||
      s->R > kMaxR || s->R > s->E || s->E % s->R != 0 || s->T % s->R != 0)
    return EP_ERR_INVALID_ARG;
  if (s->H < 8 || s->H % 8 != 0) return EP_ERR_INVALID_ARG;
  if (s->use_fp8 != 0 && s->use_fp8 != 1) return EP_ERR_INVALID_ARG;
  if (s->use_fp8 && s->H % kGroup != 0) return EP_ERR_INVALID_ARG;
  if (s->num_sms < 0) return EP_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s->T) * s->k > 0x7fffffffLL) return EP_ERR_INVALID_ARG;
  if (s->max_tokens_per_rank < 0) return EP_ERR_INVALID_ARG;
  if (s->max_tokens_per_rank > 0) {  // padded low-latency layout
    const int64_t Tr = s->T / s->R, M = s->max_tokens_per_rank;
    if (M < Tr || static_cast<int64_t>(s->E) * s->R * M > 0x7fffffffLL || Tr * s->k > kPadMaxPairs ||
        Tr * s->R > kPadMaxFlags)
      return EP_ERR_INVALID_ARG;
  }
  return EP_OK;
}

int64_t receive_rows(const ep_shape_t* s) {
  return s->max_tokens_per_rank > 0 ? static_cast<int64_t>(s->E) * s->R * s->max_tokens_per_rank
                                    : static_cast<int64_t>(s->T) * s->k;
}

int check_handle(const ep_shape_t* s, const ep_handle_t* h) {
  if (h == nullptr) return EP_ERR_INVALID_ARG;
  const void* arrays[] = {h->num_tokens_per_expert, h->expert_offset, h->num_tokens_per_rank,
                          h->count_src_rank_expert, h->src_rank_expert_offset, h->slot_of_pair,
                          h->src_of_slot, h->error_word};
  for (const void* a : arrays)
    if (a == nullptr || !aligned(a, 4)) return EP_ERR_INVALID_ARG;
  if (h->is_token_in_rank == nullptr && s->T > 0) return EP_ERR_INVALID_ARG;
  return EP_OK;
}

// Row arrays must be non-null (when they hold data) and 16-byte aligned.
bool rows_ok(const void* p, int64_t rows) { return rows == 0 || (p != nullptr && aligned(p, 16)); }
bool f32_ok(const void* p, int64_t n) { return n == 0 || (p != nullptr && aligned(p, 4)); }

int grid_cap(const DeviceInfo& d, const ep_shape_t* s, int occ) {
  const int sms = (s->num_sms > 0 && s->num_sms < d.sms) ? s->num_sms : d.sms;
  return sms * occ;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct LayoutGeometry {
  int tile_t, tiles_per_rank, nt, ncol;
  size_t colhist_bytes, coltotal_bytes, total_bytes;
};

LayoutGeometry layout_geometry(const ep_shape_t* s) {
  LayoutGeometry g;
  const int Tr = s->T / s->R;
  g.tile_t = kTilePairs / s->k;
  if (g.tile_t > kTileFlagBytes / s->R) g.tile_t = kTileFlagBytes / s->R;
  if (g.tile_t < 1) g.tile_t = 1;
  g.tiles_per_rank = static_cast<int>(ceil_div(Tr, g.tile_t));
  g.nt = s->R * g.tiles_per_rank;
  g.ncol = s->E + s->R;
  auto round256 = [](size_t b) { return (b + 255) / 256 * 256; };
  g.colhist_bytes = round256(static_cast<size_t>(g.ncol) * g.nt * 4);
  g.coltotal_bytes = round256(static_cast<size_t>(g.ncol) * 4);
  g.total_bytes = g.colhist_bytes + g.coltotal_bytes;
  return g;
}

MoveParams move_params(const ep_shape_t* s, const ep_handle_t* h, const float* w, bool pdl) {
  MoveParams p;
  p.pdl = pdl ? 1 : 0;
  p.T = s->T;
  p.H = s->H;
  p.k = s->k;
  p.G = s->H / kGroup;
  p.chunks = static_cast<int>(ceil_div(s->H, kChunk));
  p.slot_of_pair = h->slot_of_pair;
  p.topk_weights = w;
  return p;
}

int finish(const ep_handle_t* h, cudaStream_t stream) {
  int st = cuda_status(cudaGetLastError());
  if (st != EP_OK || !debug_mode()) return st;
  return ep_get_error(h, reinterpret_cast<ep_stream_t>(stream));
}

// Programmatic dependent launch (common.cuh): on unless EP_PDL=0.
bool pdl_enabled() {
  static const bool on = [] {
    const char* s = std::getenv("EP_PDL");
    return !(s != nullptr && s[0] == '0');
  }();
  return on;
}

// Fills the programmatic-serialization launch attribute (when `pdl`) at
// attrs[n] and returns the new attribute count.
unsigned pdl_attribute(cudaLaunchAttribute* attrs, unsigned n, bool pdl) {
  if (!pdl) return n;
  attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[n].val.programmaticStreamSerializationAllowed = 1;
  return n + 1;
}

// kernel<<<grid, block, smem, s>>>(args...), with programmatic stream
// serialization when `pdl`: the kernel may be scheduled while the previous
// kernel on the stream drains, and waits for it (griddepcontrol.wait) before
// any global access.  Launch errors are left for finish() to read, as with
// <<<>>>.
template <typename... KArgs, typename... Args>
void launch(bool pdl, void (*kernel)(KArgs...), int64_t grid, int block, size_t smem, cudaStream_t s,
            Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attrs[1];
  cfg.numAttrs = pdl_attribute(attrs, 0, pdl);
  cfg.attrs = attrs;
  (void)cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// finish() for calls without a handle (the router): launch errors, and with
// EP_DEBUG=1 a synchronisation that surfaces the kernel's own faults.
int finish_no_handle(cudaStream_t stream) {
  int st = cuda_status(cudaGetLastError());
  if (st != EP_OK || !debug_mode()) return st;
  return cuda_status(cudaStreamSynchronize(stream));
}

int movement_grid(const DeviceInfo& d, const ep_shape_t* s, int occ, int64_t units_per_warp_grid) {
  const int64_t need = ceil_div(units_per_warp_grid, kMoveWarps);
  const int64_t cap = grid_cap(d, s, occ);
  return static_cast<int>(need < cap ? need : cap);
}

// Tokens per CTA of the bulk-store dispatch on the whole GPU (ep_dispatch).
constexpr int64_t kTmaTokensPerCta = 2;

// From this many tokens per SM on, dispatch and combine backward launch
// oversubscribed grids on the whole GPU (below it, persistent ones measured
// as fast or faster).
constexpr int64_t kOversubscribeTokensPerSm = 16;

// Programmatic dependent launch for a call over `tokens` tokens: only below
// kOversubscribeTokensPerSm tokens per SM, where the grids are persistent and
// a call lasts tens of microseconds.  Measured on the decode shape (1024
// tokens): step 115.6 against 117.7 us without it.  On large batches it cost
// time instead (prefill step 2929 against 2886 us, backward workload 1832
// against 1815 us, same GPU), so they launch without it.
bool use_pdl(const DeviceInfo& d, int64_t tokens) {
  return pdl_enabled() && tokens < kOversubscribeTokensPerSm * d.sms;
}

// The budget is the whole GPU (no SM budget in force).
bool whole_gpu(const DeviceInfo& d, const ep_shape_t* s) { return s->num_sms <= 0 || s->num_sms >= d.sms; }

// Grid of the bulk-store dispatch (single-GPU and peer forms) for T tokens
// at occ resident CTAs per SM.
int tma_dispatch_grid(const DeviceInfo& d, const ep_shape_t* s, int64_t T, int occ) {
  const bool large = T >= kOversubscribeTokensPerSm * d.sms;
  if (large && whole_gpu(d, s)) {
    // kTmaTokensPerCta tokens per CTA, all resident slots in use: the block
    // scheduler refills each slot as a CTA retires, and a CTA's second token
    // loads while its first is quantised.  Measured against the persistent
    // grid: 54 / 56 us at 4096 tokens, 194 / 211 at 16384, 380 / 420 at
    // 32768.  Below 16 tokens per SM the persistent grid is as fast or faster
    // (a partial last wave costs more than it balances).
    return static_cast<int>(ceil_div(T, kTmaTokensPerCta));
  }
  // Persistent grid.  Large batches under an SM budget run 2 CTAs per SM
  // (fewer row copies in flight per SM measured faster at 32768 tokens);
  // small ones use every resident slot.
  if (large && occ > 2) occ = 2;
  const int64_t cap = grid_cap(d, s, occ);
  return static_cast<int>(T < cap ? T : cap);
}

// Combine backward on the whole GPU at 16 tokens per SM or more: about
// kCbwdPairsPerWarp pairs per warp, so the block scheduler balances the end of
// the kernel, never fewer CTAs than the persistent grid.  Measured against the
// persistent grid at H = 7168: 161 / 163 us at 4096 tokens, 314 / 320 at 8192,
// 617 / 635 at 16384, 1222 / 1262 at 32768 (and 702 / 723 at H = 4096); at
// 2048 tokens and below the persistent grid is as fast or faster.  Combine
// and dispatch backward measured fastest persistent at the prefill shape and
// keep movement_grid.  Under an SM budget the grid stays persistent: a budget
// caps the CTAs resident at once, which only a grid of that size guarantees.
constexpr int64_t kCbwdPairsPerWarp = 2;

int pair_grid(const DeviceInfo& d, const ep_shape_t* s, int occ, int64_t tokens, int64_t pairs) {
  if (!whole_gpu(d, s) || tokens < kOversubscribeTokensPerSm * d.sms) return movement_grid(d, s, occ, pairs);
  const int64_t need = ceil_div(pairs, kMoveWarps);
  const int64_t cap = grid_cap(d, s, occ);
  const int64_t want = ceil_div(pairs, kMoveWarps * kCbwdPairsPerWarp);
  const int64_t g = want > cap ? want : cap;
  return static_cast<int>(g < need ? g : need);
}

// route_compact_kernel<2^nq_log, 2^nc_log> (nc_log < nq_log <= 5).
const void* route_compact_fn(int nq_log, int nc_log) {
  switch (nq_log * 8 + nc_log) {
    case 8 + 0: return reinterpret_cast<const void*>(route_compact_kernel<2, 1>);
    case 16 + 0: return reinterpret_cast<const void*>(route_compact_kernel<4, 1>);
    case 16 + 1: return reinterpret_cast<const void*>(route_compact_kernel<4, 2>);
    case 24 + 0: return reinterpret_cast<const void*>(route_compact_kernel<8, 1>);
    case 24 + 1: return reinterpret_cast<const void*>(route_compact_kernel<8, 2>);
    case 24 + 2: return reinterpret_cast<const void*>(route_compact_kernel<8, 4>);
    case 32 + 0: return reinterpret_cast<const void*>(route_compact_kernel<16, 1>);
    case 32 + 1: return reinterpret_cast<const void*>(route_compact_kernel<16, 2>);
    case 32 + 2: return reinterpret_cast<const void*>(route_compact_kernel<16, 4>);
    case 32 + 3: return reinterpret_cast<const void*>(route_compact_kernel<16, 8>);
    case 40 + 0: return reinterpret_cast<const void*>(route_compact_kernel<32, 1>);
    case 40 + 1: return reinterpret_cast<const void*>(route_compact_kernel<32, 2>);
    case 40 + 2: return reinterpret_cast<const void*>(route_compact_kernel<32, 4>);
    case 40 + 3: return reinterpret_cast<const void*>(route_compact_kernel<32, 8>);
    case 40 + 4: return reinterpret_cast<const void*>(route_compact_kernel<32, 16>);
    default: return nullptr;
  }
}

static_assert(EP_MAX_PEERS == kMaxPeers, "peer tables of the C ABI and the kernels agree");

// Every owner's buffer given, non-null and aligned to `align` bytes.
bool peer_rows_ok(const ep_peer_rows_t* t, int R, size_t align) {
  if (t == nullptr) return false;
  for (int o = 0; o < R; ++o)
    if (t->rows[o] == nullptr || !aligned(t->rows[o], align)) return false;
  return true;
}

PeerRows peer_rows(const ep_peer_rows_t* t) {
  PeerRows r{};
  if (t != nullptr)
    for (int o = 0; o < kMaxPeers; ++o) r.base[o] = t->rows[o];
  return r;
}

// Checks common to the peer calls and the kernel parameters of this rank.
int peer_setup(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx, const ep_handle_t* handle,
               const float* topk_weights, PeerParams* p) {
  int st = check_shape(shape);
  if (st != EP_OK) return st;
  if ((st = check_handle(shape, handle)) != EP_OK) return st;
  if (shape->max_tokens_per_rank != 0 || shape->R > EP_MAX_PEERS || rank < 0 || rank >= shape->R)
    return EP_ERR_INVALID_ARG;
  const int64_t T = shape->T, Tl = T / shape->R;
  if (T > 0 && (topk_idx == nullptr || !aligned(topk_idx, 8))) return EP_ERR_INVALID_ARG;
  if (topk_weights != nullptr && !f32_ok(topk_weights, Tl * shape->k)) return EP_ERR_INVALID_ARG;
  p->T = static_cast<int>(Tl);
  p->H = shape->H;
  p->k = shape->k;
  p->G = shape->H / kGroup;
  p->chunks = static_cast<int>(ceil_div(shape->H, kChunk));
  p->t_begin = static_cast<int>(rank * Tl);
  p->Er = shape->E / shape->R;
  p->R = shape->R;
  p->slot_of_pair = handle->slot_of_pair;
  p->topk_idx = topk_idx;
  p->expert_offset = handle->expert_offset;
  p->topk_weights = topk_weights;
  return EP_OK;
}

// The layout kernels of one call, enqueued on s (arguments checked by the
// caller).  late: the last kernel lets the next one be scheduled only after
// its own programmatic-launch wait (LayoutParams::late_trigger).
int enqueue_layout(const ep_shape_t* shape, const int64_t* topk_idx, const ep_handle_t* handle, void* workspace,
                   const LayoutGeometry& g, const DeviceInfo* d, bool pdl, bool late, cudaStream_t s) {
  int st = EP_OK;
  LayoutParams p;
  p.topk_idx = topk_idx;
  p.T = shape->T;
  p.k = shape->k;
  p.E = shape->E;
  p.R = shape->R;
  p.Tr = shape->T / shape->R;
  p.Er = shape->E / shape->R;
  p.tile_t = g.tile_t;
  p.tiles_per_rank = g.tiles_per_rank;
  p.nt = g.nt;
  p.ncol = g.ncol;
  p.colhist = static_cast<int32_t*>(workspace);
  p.coltotal = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + g.colhist_bytes);
  p.num_tokens_per_expert = handle->num_tokens_per_expert;
  p.expert_offset = handle->expert_offset;
  p.num_tokens_per_rank = handle->num_tokens_per_rank;
  p.count_src_rank_expert = handle->count_src_rank_expert;
  p.src_rank_expert_offset = handle->src_rank_expert_offset;
  p.is_token_in_rank = handle->is_token_in_rank;
  p.slot_of_pair = handle->slot_of_pair;
  p.src_of_slot = handle->src_of_slot;
  p.error_word = handle->error_word;
  p.late_trigger = late ? 1 : 0;

  if (shape->max_tokens_per_rank > 0) {
    const size_t smem = layout_padded_smem(p.Tr, shape->E, shape->R);
    if (smem > 48 * 1024) {
      // a function attribute belongs to the current context (a reset or a
      // green context starts without it), so it is set before each launch
      const void* fn = shape->R <= kPadClusterMax ? reinterpret_cast<const void*>(layout_padded_kernel<true>)
                                                  : reinterpret_cast<const void*>(layout_padded_kernel<false>);
      if ((st = cuda_status(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem)))) != EP_OK)
        return st;
    }
    if (shape->R <= kPadClusterMax) {  // one cluster of R CTAs sums the totals itself
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(shape->R);
      cfg.blockDim = dim3(kPadThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = s;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = shape->R;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = pdl_attribute(attr, 1, pdl);
      return cuda_status(cudaLaunchKernelEx(&cfg, layout_padded_kernel<true>, p, shape->max_tokens_per_rank));
    }
    if ((st = cuda_status(cudaMemsetAsync(handle->num_tokens_per_expert, 0, shape->E * 4, s))) != EP_OK ||
        (st = cuda_status(cudaMemsetAsync(handle->num_tokens_per_rank, 0, shape->R * 4, s))) != EP_OK)
      return st;
    launch(pdl, layout_padded_kernel<false>, shape->R, kPadThreads, smem, s, p, shape->max_tokens_per_rank);
    return EP_OK;
  }
  if (layout_small_fits(shape->T, shape->k, shape->E, shape->R)) {
    if (small_cluster_size(d) == kClusterCtasWide) {
      if ((st = cuda_status(cudaFuncSetAttribute(layout_small_kernel<kClusterCtasWide>,
                                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1))) != EP_OK)
        return st;
      launch(pdl, layout_small_kernel<kClusterCtasWide>, kClusterCtasWide, kSmallThreads,
             layout_small_smem(shape->T, shape->E, shape->R, kClusterCtasWide), s, p);
    } else {
      launch(pdl, layout_small_kernel<kClusterCtas>, kClusterCtas, kSmallThreads,
             layout_small_smem(shape->T, shape->E, shape->R, kClusterCtas), s, p);
    }
    return EP_OK;
  }
  // only the last of the three kernels triggers late
  LayoutParams pe = p;
  pe.late_trigger = 0;
  if (g.nt > 0) {
    const size_t smem = static_cast<size_t>(g.ncol) * 4 + static_cast<size_t>(g.tile_t) * shape->R;
    launch(pdl, layout_count_kernel, g.nt, kLayoutThreads, smem, s, pe);
  }
  launch(pdl, layout_scan_kernel, g.ncol, kLayoutThreads, 0, s, pe);
  const size_t smem_assign = static_cast<size_t>(shape->E + 1 + kLayoutWarps * shape->E) * 4;
  launch(pdl, layout_assign_kernel, g.nt > 0 ? g.nt : 1, kLayoutThreads, smem_assign, s, p);
  return EP_OK;
}

// Argument checks of ep_dispatch.
int check_dispatch_args(const ep_shape_t* shape, const void* x, const float* topk_weights, const ep_handle_t* handle,
                        const void* recv_x, const float* recv_scale, const float* recv_weight) {
  int st = check_shape(shape);
  if (st != EP_OK) return st;
  if ((st = check_handle(shape, handle)) != EP_OK) return st;
  const int64_t T = shape->T, P = T * shape->k;
  if (!rows_ok(x, T) || !rows_ok(recv_x, P) || !f32_ok(topk_weights, P)) return EP_ERR_INVALID_ARG;
  if (shape->use_fp8 && !f32_ok(recv_scale, P)) return EP_ERR_INVALID_ARG;
  if (recv_weight != nullptr && !aligned(recv_weight, 4)) return EP_ERR_INVALID_ARG;
  return EP_OK;
}

// The bulk-store dispatch serves 4 to 16 chunks of 512 channels.
bool tma_dispatch_applies(const ep_shape_t* shape) {
  const int64_t chunks = ceil_div(shape->H, kChunk);
  return chunks >= kTmaMinChunks && chunks <= kTmaMaxChunks;
}

// The dispatch kernel of one call (arguments checked, T > 0).  early: the
// bulk-store kernel's EARLY form, only right after the fused call's layout.
void enqueue_dispatch(const ep_shape_t* shape, const void* x, const float* topk_weights, const ep_handle_t* handle,
                      void* recv_x, float* recv_scale, float* recv_weight, const DeviceInfo* d, bool pdl, bool early,
                      cudaStream_t s) {
  const MoveParams p = move_params(shape, handle, topk_weights, pdl);
  const int64_t units = shape->T * p.chunks;
  const uint16_t* xp = static_cast<const uint16_t*>(x);
  const bool fp8 = shape->use_fp8 != 0;
  if (tma_dispatch_applies(shape)) {
    const int threads = p.chunks * kWarp;
    const size_t smem = tma_smem_layout(shape->H, fp8, early).total;
    void (*fn)(MoveParams, const uint16_t*, void*, float*, float*) =
        fp8 ? (early ? dispatch_tma_kernel<true, true> : dispatch_tma_kernel<true, false>)
            : (early ? dispatch_tma_kernel<false, true> : dispatch_tma_kernel<false, false>);
    int occ;
    {
      std::lock_guard<std::mutex> lock(g_dev_mu);
      int& cached = const_cast<DeviceInfo*>(d)->occ_tma[early][fp8][p.chunks];
      if (cached == 0) cached = occupancy(reinterpret_cast<const void*>(fn), threads, smem);
      occ = cached;
    }
    const int grid = tma_dispatch_grid(*d, shape, shape->T, occ);
    launch(pdl, fn, grid, threads, smem, s, p, xp, recv_x, fp8 ? recv_scale : nullptr, recv_weight);
  } else if (fp8) {
    launch(pdl, dispatch_kernel<true>, movement_grid(*d, shape, d->occ_disp_fp8, units), kMoveThreads, 0, s, p, xp,
        recv_x, recv_scale, recv_weight);
  } else {
    launch(pdl, dispatch_kernel<false>, movement_grid(*d, shape, d->occ_disp_bf16, units), kMoveThreads, 0, s, p, xp,
        recv_x, nullptr, recv_weight);
  }
}

}  // namespace

// Argument checks of ep_get_dispatch_layout other than the workspace, shared
// with ep_get_dispatch_layout_noalloc (ep_noalloc.cu).  Not exported.
__attribute__((visibility("hidden"))) int ep_internal_check_layout_args(const ep_shape_t* shape,
                                                                        const int64_t* topk_idx,
                                                                        const ep_handle_t* handle) {
  int st = check_shape(shape);
  if (st != EP_OK) return st;
  if ((st = check_handle(shape, handle)) != EP_OK) return st;
  if (shape->T > 0 && (topk_idx == nullptr || !aligned(topk_idx, 8))) return EP_ERR_INVALID_ARG;
  return EP_OK;
}

extern "C" {

int ep_handle_sizes(const ep_shape_t* shape, int64_t counts[9]) {
  int st = check_shape(shape);
  if (st != EP_OK || counts == nullptr) return EP_ERR_INVALID_ARG;
  const int64_t T = shape->T, k = shape->k, E = shape->E, R = shape->R;
  const int64_t c[9] = {E, E + 1, R, R * E, R * E, T * R, T * k, receive_rows(shape), 1};
  for (int i = 0; i < 9; ++i) counts[i] = c[i];
  return EP_OK;
}

size_t ep_workspace_size(const ep_shape_t* shape) {
  if (check_shape(shape) != EP_OK) return 0;
  return layout_geometry(shape).total_bytes;
}

int ep_get_dispatch_layout(const ep_shape_t* shape, const int64_t* topk_idx, const ep_handle_t* handle,
                           void* workspace, size_t workspace_bytes, ep_stream_t stream) {
  int st = ep_internal_check_layout_args(shape, topk_idx, handle);
  if (st != EP_OK) return st;
  const LayoutGeometry g = layout_geometry(shape);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < g.total_bytes)
    return EP_ERR_INVALID_ARG;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != EP_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = enqueue_layout(shape, topk_idx, handle, workspace, g, d, use_pdl(*d, shape->T), false, s)) != EP_OK)
    return st;
  return finish(handle, s);
}

int ep_dispatch(const ep_shape_t* shape, const void* x, const float* topk_weights, const ep_handle_t* handle,
                void* recv_x, float* recv_scale, float* recv_weight, ep_stream_t stream) {
  int st = check_dispatch_args(shape, x, topk_weights, handle, recv_x, recv_scale, recv_weight);
  if (st != EP_OK) return st;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != EP_OK) return st;
  if (shape->T == 0) return EP_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  enqueue_dispatch(shape, x, topk_weights, handle, recv_x, recv_scale, recv_weight, d, use_pdl(*d, shape->T), false,
                   s);
  return finish(handle, s);
}

int ep_dispatch_with_layout(const ep_shape_t* shape, const int64_t* topk_idx, const void* x,
                            const float* topk_weights, const ep_handle_t* handle, void* workspace,
                            size_t workspace_bytes, void* recv_x, float* recv_scale, float* recv_weight,
                            ep_stream_t stream) {
  int st = ep_internal_check_layout_args(shape, topk_idx, handle);
  if (st != EP_OK) return st;
  if ((st = check_dispatch_args(shape, x, topk_weights, handle, recv_x, recv_scale, recv_weight)) != EP_OK) return st;
  const LayoutGeometry g = layout_geometry(shape);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < g.total_bytes)
    return EP_ERR_INVALID_ARG;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, shape->T);
  const bool early = pdl && shape->T > 0 && tma_dispatch_applies(shape);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = enqueue_layout(shape, topk_idx, handle, workspace, g, d, pdl, early, s)) != EP_OK) return st;
  if ((st = cuda_status(cudaGetLastError())) != EP_OK) return st;
  if (shape->T > 0)
    enqueue_dispatch(shape, x, topk_weights, handle, recv_x, recv_scale, recv_weight, d, pdl, early, s);
  return finish(handle, s);
}

int ep_combine(const ep_shape_t* shape, const void* y, const float* topk_weights, const ep_handle_t* handle,
               void* out, ep_stream_t stream) {
  int st = check_shape(shape);
  if (st != EP_OK) return st;
  if ((st = check_handle(shape, handle)) != EP_OK) return st;
  const int64_t T = shape->T, P = T * shape->k;
  if (!rows_ok(y, P) || !rows_ok(out, T) || !f32_ok(topk_weights, P)) return EP_ERR_INVALID_ARG;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, T);
  if (T == 0) return EP_OK;
  const MoveParams p = move_params(shape, handle, topk_weights, pdl);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool ragged = shape->H % kChunk != 0;
  const int grid = movement_grid(*d, shape, d->occ_comb[ragged], T * p.chunks);
  if (ragged)
    launch(pdl, gather_reduce_kernel<true, true>, grid, kMoveThreads, 0, s, p, static_cast<const uint16_t*>(y),
        static_cast<uint16_t*>(out));
  else
    launch(pdl, gather_reduce_kernel<true, false>, grid, kMoveThreads, 0, s, p, static_cast<const uint16_t*>(y),
        static_cast<uint16_t*>(out));
  return finish(handle, s);
}

int ep_combine_backward(const ep_shape_t* shape, const void* grad_out, const void* y,
                        const float* topk_weights, const ep_handle_t* handle, void* grad_y, float* grad_w,
                        ep_stream_t stream) {
  int st = check_shape(shape);
  if (st != EP_OK) return st;
  if ((st = check_handle(shape, handle)) != EP_OK) return st;
  const int64_t T = shape->T, P = T * shape->k;
  if (!rows_ok(grad_out, T) || !rows_ok(y, P) || !rows_ok(grad_y, P) || !f32_ok(topk_weights, P) ||
      !f32_ok(grad_w, P))
    return EP_ERR_INVALID_ARG;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, T);
  if (T == 0) return EP_OK;
  const MoveParams p = move_params(shape, handle, topk_weights, pdl);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool ragged = shape->H % kChunk != 0;
  const int grid = pair_grid(*d, shape, d->occ_cbwd[ragged], T, T * shape->k);
  const uint16_t* gp = static_cast<const uint16_t*>(grad_out);
  const uint16_t* yp = static_cast<const uint16_t*>(y);
  if (ragged)
    launch(pdl, combine_backward_kernel<true>, grid, kMoveThreads, 0, s, p, gp, yp, static_cast<uint16_t*>(grad_y),
        grad_w);
  else
    launch(pdl, combine_backward_kernel<false>, grid, kMoveThreads, 0, s, p, gp, yp, static_cast<uint16_t*>(grad_y),
        grad_w);
  return finish(handle, s);
}

int ep_dispatch_backward(const ep_shape_t* shape, const void* grad_recv, const ep_handle_t* handle,
                         void* grad_x, ep_stream_t stream) {
  int st = check_shape(shape);
  if (st != EP_OK) return st;
  if ((st = check_handle(shape, handle)) != EP_OK) return st;
  const int64_t T = shape->T, P = T * shape->k;
  if (!rows_ok(grad_recv, P) || !rows_ok(grad_x, T)) return EP_ERR_INVALID_ARG;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, T);
  if (T == 0) return EP_OK;
  const MoveParams p = move_params(shape, handle, nullptr, pdl);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool ragged = shape->H % kChunk != 0;
  const int grid = movement_grid(*d, shape, d->occ_dbwd[ragged], T * p.chunks);
  if (ragged)
    launch(pdl, gather_reduce_kernel<false, true>, grid, kMoveThreads, 0, s, p,
        static_cast<const uint16_t*>(grad_recv), static_cast<uint16_t*>(grad_x));
  else
    launch(pdl, gather_reduce_kernel<false, false>, grid, kMoveThreads, 0, s, p,
        static_cast<const uint16_t*>(grad_recv), static_cast<uint16_t*>(grad_x));
  return finish(handle, s);
}

int ep_route_group_limited(const ep_shape_t* shape, const float* scores, int n_groups, int topk_groups,
                           int64_t* topk_idx, float* topk_weights, ep_stream_t stream) {
  int st = check_shape(shape);
  if (st != EP_OK) return st;
  if (n_groups < 1 || n_groups > kRouteMaxGroups || shape->E % n_groups != 0 || topk_groups < 1 ||
      topk_groups > n_groups || shape->k > topk_groups * (shape->E / n_groups))
    return EP_ERR_INVALID_ARG;
  const int64_t T = shape->T;
  if (T > 0 && (!f32_ok(scores, T) || topk_idx == nullptr || !aligned(topk_idx, 8) || !f32_ok(topk_weights, T)))
    return EP_ERR_INVALID_ARG;
  const DeviceInfo* d = nullptr;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, T);
  if (T == 0) return EP_OK;
  RouteParams p{scores, shape->T, shape->E, shape->k, n_groups, topk_groups, topk_idx, topk_weights};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  constexpr int warps = kRouteThreads / kWarp;
  const int nq = static_cast<int>(ceil_div(shape->E, kWarp));
  const int variant = nq <= 1 ? 0 : nq <= 2 ? 1 : nq <= 4 ? 2 : nq <= 8 ? 3 : nq <= 16 ? 4 : 5;
  // groups on lane boundaries: a lane's experts share one group and a group
  // spans a power-of-two number of lanes
  const int per_lane = 1 << variant, per_group = shape->E / n_groups;
  const int lanes_per_group = per_group / per_lane;
  const bool on_lanes = shape->E % per_lane == 0 && per_group % per_lane == 0 &&
                        (lanes_per_group & (lanes_per_group - 1)) == 0;
  const int64_t need = ceil_div(T, warps);
  if (on_lanes) {
    // the chosen groups' experts onto all lanes, when that leaves fewer per lane
    const int64_t cand = static_cast<int64_t>(topk_groups) * per_group;
    int nc_log = 0;
    while ((int64_t{kWarp} << nc_log) < cand) ++nc_log;
    if (nc_log < variant) {
      const void* fn = route_compact_fn(variant, nc_log);
      int occ;
      {
        std::lock_guard<std::mutex> lock(g_dev_mu);
        int& cached = const_cast<DeviceInfo*>(d)->occ_route_compact[variant][nc_log];
        if (cached == 0) cached = occupancy(fn, kRouteThreads, 0);
        occ = cached;
      }
      const int64_t cap = grid_cap(*d, shape, occ);
      const int grid = static_cast<int>(need < cap ? need : cap);
      void* args[] = {&p};
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(grid);
      cfg.blockDim = dim3(kRouteThreads);
      cfg.stream = s;
      cudaLaunchAttribute attrs[1];
      cfg.numAttrs = pdl_attribute(attrs, 0, pdl);
      cfg.attrs = attrs;
      const int launched = cuda_status(cudaLaunchKernelExC(&cfg, fn, args));
      return launched != EP_OK ? launched : finish_no_handle(s);
    }
  }
  const int64_t cap = grid_cap(*d, shape, on_lanes ? d->occ_route_aligned[variant] : d->occ_route[variant]);
  const int grid = static_cast<int>(need < cap ? need : cap);
  if (on_lanes) {
    switch (variant) {
      case 0: launch(pdl, route_aligned_kernel<1>, grid, kRouteThreads, 0, s, p); break;
      case 1: launch(pdl, route_aligned_kernel<2>, grid, kRouteThreads, 0, s, p); break;
      case 2: launch(pdl, route_aligned_kernel<4>, grid, kRouteThreads, 0, s, p); break;
      case 3: launch(pdl, route_aligned_kernel<8>, grid, kRouteThreads, 0, s, p); break;
      case 4: launch(pdl, route_aligned_kernel<16>, grid, kRouteThreads, 0, s, p); break;
      default: launch(pdl, route_aligned_kernel<32>, grid, kRouteThreads, 0, s, p); break;
    }
    return finish_no_handle(s);
  }
  switch (variant) {
    case 0: launch(pdl, route_group_limited_kernel<1>, grid, kRouteThreads, 0, s, p); break;
    case 1: launch(pdl, route_group_limited_kernel<2>, grid, kRouteThreads, 0, s, p); break;
    case 2: launch(pdl, route_group_limited_kernel<4>, grid, kRouteThreads, 0, s, p); break;
    case 3: launch(pdl, route_group_limited_kernel<8>, grid, kRouteThreads, 0, s, p); break;
    case 4: launch(pdl, route_group_limited_kernel<16>, grid, kRouteThreads, 0, s, p); break;
    default: launch(pdl, route_group_limited_kernel<32>, grid, kRouteThreads, 0, s, p); break;
  }
  return finish_no_handle(s);
}

int ep_dispatch_peers(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx, const ep_handle_t* handle,
                      const void* x, const float* topk_weights, const ep_peer_rows_t* recv_x,
                      const ep_peer_rows_t* recv_scale, const ep_peer_rows_t* recv_weight, ep_stream_t stream) {
  PeerParams p;
  const DeviceInfo* d = nullptr;
  int st = peer_setup(shape, rank, topk_idx, handle, topk_weights, &p);
  if (st != EP_OK) return st;
  if (topk_weights == nullptr && p.T > 0) return EP_ERR_INVALID_ARG;
  const int R = shape->R;
  if (!rows_ok(x, p.T) || (p.T > 0 && !peer_rows_ok(recv_x, R, 16))) return EP_ERR_INVALID_ARG;
  if (shape->use_fp8 && p.T > 0 && !peer_rows_ok(recv_scale, R, 4)) return EP_ERR_INVALID_ARG;
  if (recv_weight != nullptr && p.T > 0 && !peer_rows_ok(recv_weight, R, 4)) return EP_ERR_INVALID_ARG;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, p.T);
  if (p.T == 0) return EP_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t units = static_cast<int64_t>(p.T) * p.chunks;
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  const PeerRows rx = peer_rows(recv_x), rs = peer_rows(recv_scale), rw = peer_rows(recv_weight);
  const bool fp8 = shape->use_fp8 != 0;
  if (p.chunks >= kTmaMinChunks && p.chunks <= kTmaMaxChunks) {
    const int threads = p.chunks * kWarp;
    const size_t smem = tma_smem_layout(shape->H, fp8).total;
    const void* fn = fp8 ? reinterpret_cast<const void*>(dispatch_tma_peers_kernel<true>)
                         : reinterpret_cast<const void*>(dispatch_tma_peers_kernel<false>);
    int occ;
    {
      std::lock_guard<std::mutex> lock(g_dev_mu);
      int& cached = const_cast<DeviceInfo*>(d)->occ_tma_peers[fp8][p.chunks];
      if (cached == 0) cached = occupancy(fn, threads, smem);
      occ = cached;
    }
    const int grid = tma_dispatch_grid(*d, shape, p.T, occ);
    if (fp8)
      launch(pdl, dispatch_tma_peers_kernel<true>, grid, threads, smem, s, p, xs, rx, rs, rw);
    else
      launch(pdl, dispatch_tma_peers_kernel<false>, grid, threads, smem, s, p, xs, rx, rs, rw);
  } else if (fp8) {
    launch(pdl, dispatch_peers_kernel<true>, movement_grid(*d, shape, d->occ_peer_disp[1], units), kMoveThreads, 0,
        s, p, xs, rx, rs, rw);
  } else {
    launch(pdl, dispatch_peers_kernel<false>, movement_grid(*d, shape, d->occ_peer_disp[0], units), kMoveThreads, 0,
        s, p, xs, rx, rs, rw);
  }
  return finish(handle, s);
}

int ep_combine_peers(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx, const ep_handle_t* handle,
                     const ep_peer_rows_t* y, const float* topk_weights, void* out, ep_stream_t stream) {
  PeerParams p;
  const DeviceInfo* d = nullptr;
  int st = peer_setup(shape, rank, topk_idx, handle, topk_weights, &p);
  if (st != EP_OK) return st;
  if (topk_weights == nullptr && p.T > 0) return EP_ERR_INVALID_ARG;
  if (!rows_ok(out, p.T) || (p.T > 0 && !peer_rows_ok(y, shape->R, 16))) return EP_ERR_INVALID_ARG;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, p.T);
  if (p.T == 0) return EP_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool ragged = shape->H % kChunk != 0;
  const int grid = movement_grid(*d, shape, d->occ_peer_gather[1][ragged], static_cast<int64_t>(p.T) * p.chunks);
  if (ragged)
    launch(pdl, gather_reduce_peers_kernel<true, true>, grid, kMoveThreads, 0, s, p, peer_rows(y),
        static_cast<uint16_t*>(out));
  else
    launch(pdl, gather_reduce_peers_kernel<true, false>, grid, kMoveThreads, 0, s, p, peer_rows(y),
        static_cast<uint16_t*>(out));
  return finish(handle, s);
}

int ep_combine_backward_peers(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx,
                              const ep_handle_t* handle, const void* grad_out, const ep_peer_rows_t* y,
                              const float* topk_weights, const ep_peer_rows_t* grad_y, float* grad_w,
                              ep_stream_t stream) {
  PeerParams p;
  const DeviceInfo* d = nullptr;
  int st = peer_setup(shape, rank, topk_idx, handle, topk_weights, &p);
  if (st != EP_OK) return st;
  if (topk_weights == nullptr && p.T > 0) return EP_ERR_INVALID_ARG;
  const int R = shape->R;
  if (!rows_ok(grad_out, p.T) || !f32_ok(grad_w, static_cast<int64_t>(p.T) * p.k) ||
      (p.T > 0 && (!peer_rows_ok(y, R, 16) || !peer_rows_ok(grad_y, R, 16))))
    return EP_ERR_INVALID_ARG;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, p.T);
  if (p.T == 0) return EP_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool ragged = shape->H % kChunk != 0;
  // persistent: with R ranks emulated side by side on one GPU, oversubscribed
  // grids measured slower (1210 against 1190 us a step at the prefill shape)
  const int grid = movement_grid(*d, shape, d->occ_peer_cbwd[ragged], static_cast<int64_t>(p.T) * p.k);
  const uint16_t* gp = static_cast<const uint16_t*>(grad_out);
  if (ragged)
    launch(pdl, combine_backward_peers_kernel<true>, grid, kMoveThreads, 0, s, p, gp, peer_rows(y), peer_rows(grad_y),
        grad_w);
  else
    launch(pdl, combine_backward_peers_kernel<false>, grid, kMoveThreads, 0, s, p, gp, peer_rows(y), peer_rows(grad_y),
        grad_w);
  return finish(handle, s);
}

int ep_dispatch_backward_peers(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx,
                               const ep_handle_t* handle, const ep_peer_rows_t* grad_recv, void* grad_x,
                               ep_stream_t stream) {
  PeerParams p;
  const DeviceInfo* d = nullptr;
  int st = peer_setup(shape, rank, topk_idx, handle, nullptr, &p);
  if (st != EP_OK) return st;
  if (!rows_ok(grad_x, p.T) || (p.T > 0 && !peer_rows_ok(grad_recv, shape->R, 16))) return EP_ERR_INVALID_ARG;
  if ((st = device_info(&d)) != EP_OK) return st;
  const bool pdl = use_pdl(*d, p.T);
  if (p.T == 0) return EP_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool ragged = shape->H % kChunk != 0;
  const int grid = movement_grid(*d, shape, d->occ_peer_gather[0][ragged], static_cast<int64_t>(p.T) * p.chunks);
  if (ragged)
    launch(pdl, gather_reduce_peers_kernel<false, true>, grid, kMoveThreads, 0, s, p, peer_rows(grad_recv),
        static_cast<uint16_t*>(grad_x));
  else
    launch(pdl, gather_reduce_peers_kernel<false, false>, grid, kMoveThreads, 0, s, p, peer_rows(grad_recv),
        static_cast<uint16_t*>(grad_x));
  return finish(handle, s);
}

int ep_get_error(const ep_handle_t* handle, ep_stream_t stream) {
  if (handle == nullptr || handle->error_word == nullptr) return EP_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t word = 0;
  int st = cuda_status(cudaStreamSynchronize(s));
  if (st != EP_OK) return st;
  if ((st = cuda_status(cudaMemcpyAsync(&word, handle->error_word, 4, cudaMemcpyDeviceToHost, s))) != EP_OK)
    return st;
  if ((st = cuda_status(cudaMemsetAsync(handle->error_word, 0, 4, s))) != EP_OK) return st;
  if ((st = cuda_status(cudaStreamSynchronize(s))) != EP_OK) return st;
  if (word & 1) return EP_ERR_BAD_INDEX;
  return (word & 2) ? EP_ERR_CAPACITY : EP_OK;
}

const char* ep_status_string(int status) {
  switch (status) {
    case EP_OK: return "EP_OK";
    case EP_ERR_INVALID_ARG: return "EP_ERR_INVALID_ARG: null or misaligned pointer, or shape outside the limits";
    case EP_ERR_BAD_INDEX: return "EP_ERR_BAD_INDEX: a topk_idx entry outside [-1, E)";
    case EP_ERR_CUDA: return "EP_ERR_CUDA: a CUDA call or kernel launch failed";
    case EP_ERR_UNSUPPORTED: return "EP_ERR_UNSUPPORTED: the current device is not an sm_100 GPU";
    case EP_ERR_SCRATCH_TOO_SMALL:
      return "EP_ERR_SCRATCH_TOO_SMALL: the shape needs more layout scratch than the no-alloc entry point's "
             "fixed array holds (ep_noalloc_scratch_bytes)";
    case EP_ERR_CAPACITY:
      return "EP_ERR_CAPACITY: a padded (source rank, expert) block received more than max_tokens_per_rank pairs";
    default: return "unknown ep status";
  }
}

const char* ep_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
