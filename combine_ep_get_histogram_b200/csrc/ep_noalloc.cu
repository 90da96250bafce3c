// ep_get_dispatch_layout_noalloc: the routing layout for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocating library routine:
// code that runs while a CUDA graph is being captured, code inside another
// framework's memory pool or allocator hooks, and embedded or real-time hosts
// whose device memory is fixed at start-up.  ep_get_dispatch_layout needs a
// scratch buffer for its tile histograms; this entry point takes that scratch
// from a fixed array that lives in the library itself, so the caller passes
// only its inputs and the handle.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kNoallocScratchBytes of it until the process exits.  In host
// code its name is only a host-side stand-in, so its device address is looked
// up with cudaGetSymbolAddress, once per device, with that device current,
// on the first call made on that device.
#include <cuda_runtime.h>

#include <mutex>

#include "ep.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(1) << 20;  // 1 MiB

static __device__ __align__(256) unsigned char g_layout_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device (looked up once).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return EP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return EP_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return EP_OK;
}

}  // namespace

extern "C" {

size_t ep_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

int ep_get_dispatch_layout_noalloc(const ep_shape_t* shape, const int64_t* topk_idx,
                                   const ep_handle_t* handle, ep_stream_t stream) {
  const size_t need = ep_workspace_size(shape);
  if (need == 0) return EP_ERR_INVALID_ARG;  // shape outside the limits
  if (need > kNoallocScratchBytes) return EP_ERR_SCRATCH_TOO_SMALL;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != EP_OK) return st;
  // The layout kernels overwrite every scratch word they read, so nothing in
  // the array has to start at zero, and the previous call's contents are harmless.
  return ep_get_dispatch_layout(shape, topk_idx, handle, scratch, kNoallocScratchBytes, stream);
}

}  // extern "C"
