// ep_get_dispatch_layout_noalloc: the routing layout for callers that cannot
// allocate device memory.
//
// Some callers may not call cudaMalloc or any allocating library routine:
// code that runs inside another framework's memory pool or allocator hooks
// (allocating there re-enters the allocator), and embedded or real-time
// hosts whose device memory is fixed at start-up.  ep_get_dispatch_layout
// needs a scratch buffer for its tile histograms; this entry point takes that
// scratch from a fixed array that lives in the library itself, so the caller
// passes only its inputs and the handle.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kNoallocScratchBytes of it until the process exits.  In host
// code its name is only a host-side stand-in, so its device address is looked
// up with cudaGetSymbolAddress, with the caller's device and context current,
// by the first call made in that CUDA context.  The address belongs to the
// context that loaded the module (after cudaDeviceReset, or in a green or
// driver-API context, the same device has another address), so the lookups
// are cached per context, by the context's unique id.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ep.h"

// Argument checks of ep_get_dispatch_layout without the workspace (ep_api.cu;
// not exported).
int ep_internal_check_layout_args(const ep_shape_t* shape, const int64_t* topk_idx, const ep_handle_t* handle);

namespace {

constexpr size_t kNoallocScratchBytes = size_t(1) << 20;  // 1 MiB

static __device__ __align__(256) unsigned char g_layout_scratch[kNoallocScratchBytes];

// Driver entry points, found through the runtime (the library does not link
// libcuda itself).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct CachedAddress {
  unsigned long long ctx_id;
  void* ptr;
};

constexpr int kMaxContexts = 64;
std::mutex g_mu;
CachedAddress g_cache[kMaxContexts];
int g_cached = 0, g_next = 0;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
bool g_entry_points_tried = false;

// Unique id of the current context (false if there is none or the driver
// does not say).  Called with g_mu held.
bool current_context_id(unsigned long long* id) {
  if (!g_entry_points_tried) {
    g_entry_points_tried = true;
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa{}, qb{};
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &a, 12000, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &b, 12000, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
  }
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_layout_scratch in the current context.
int scratch_address(void** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = 0;
  if (current_context_id(&id)) {
    for (int i = 0; i < g_cached; ++i)
      if (g_cache[i].ctx_id == id) {
        *out = g_cache[i].ptr;
        return EP_OK;
      }
  }
  // First call in this context (or no context current yet): look the address
  // up; this also makes the runtime's context current if none was.
  const cudaError_t before = cudaPeekAtLastError();
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_layout_scratch);
  if (e != cudaSuccess || p == nullptr) {
    // clear the error this lookup left, but not one the caller had pending
    if (before == cudaSuccess) cudaGetLastError();
    return EP_ERR_CUDA;
  }
  if (current_context_id(&id)) {
    CachedAddress& slot = g_cached < kMaxContexts ? g_cache[g_cached++] : g_cache[g_next++ % kMaxContexts];
    slot.ctx_id = id;
    slot.ptr = p;
  }
  *out = p;
  return EP_OK;
}

}  // namespace

extern "C" {

size_t ep_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

int ep_get_dispatch_layout_noalloc(const ep_shape_t* shape, const int64_t* topk_idx,
                                   const ep_handle_t* handle, ep_stream_t stream) {
  int st = ep_internal_check_layout_args(shape, topk_idx, handle);
  if (st != EP_OK) return st;
  if (ep_workspace_size(shape) > kNoallocScratchBytes) return EP_ERR_SCRATCH_TOO_SMALL;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != EP_OK) return st;
  // The layout kernels overwrite every scratch word they read, so nothing in
  // the array has to start at zero, and the previous call's contents are harmless.
  return ep_get_dispatch_layout(shape, topk_idx, handle, scratch, kNoallocScratchBytes, stream);
}

}  // extern "C"
