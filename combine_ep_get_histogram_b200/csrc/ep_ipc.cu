// Peer buffers between processes: the plumbing that turns another rank's
// device buffer into an address this process can pass in an ep_peer_rows_t
// (CUDA IPC).  The EP world is built from a process group, one process per
// GPU ("DeepEP：MoE 专家并行 EP 通信 kernel 编译与使用指南", section 五 使用方法:
// the buffer is created from the group), and inside one node the ranks reach
// each other's memory directly ("deepep-expert-parallel-communication-library",
// section 四: without NVSHMEM only intra-node communication is enabled).
//
// Export: the allocation that holds the buffer (CUDA IPC hands out whole
// cudaMalloc allocations, and a framework's caching allocator places many
// buffers in one) gets an IPC handle, and the buffer's offset inside it is
// recorded.  Open: the handle is mapped (a second open of the same
// allocation in this context returns the same mapping with its reference
// count raised) and the offset is added back.  Close: one cudaIpcCloseMemHandle
// per open.  Host-side only: no kernel, no allocation, no stream work.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "ep.h"

namespace {

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(((ep_ipc_buffer_t*)nullptr)->handle),
              "ep_ipc_buffer_t holds one cudaIpcMemHandle_t");

using MemGetAddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

std::mutex g_mu;
MemGetAddressRangeFn g_range = nullptr;
bool g_tried = false;

// cuMemGetAddressRange through the runtime (the library does not link libcuda).
MemGetAddressRangeFn address_range_fn() {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_tried) {
    g_tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_range = reinterpret_cast<MemGetAddressRangeFn>(f);
  }
  return g_range;
}

}  // namespace

extern "C" {

int ep_ipc_export(const void* ptr, ep_ipc_buffer_t* out) {
  if (ptr == nullptr || out == nullptr) return EP_ERR_INVALID_ARG;
  const MemGetAddressRangeFn range = address_range_fn();
  if (range == nullptr) return EP_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return EP_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  const cudaError_t before = cudaPeekAtLastError();
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    if (before == cudaSuccess) cudaGetLastError();  // clear only the error this call left
    return EP_ERR_CUDA;
  }
  std::memset(out, 0, sizeof(*out));
  std::memcpy(out->handle, &h, sizeof(h));
  out->offset = static_cast<uint64_t>(reinterpret_cast<CUdeviceptr>(ptr) - base);
  out->bytes = static_cast<uint64_t>(size) - out->offset;
  return EP_OK;
}

int ep_ipc_open(const ep_ipc_buffer_t* buf, void** mapped_base, void** ptr) {
  if (buf == nullptr || mapped_base == nullptr || ptr == nullptr) return EP_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, buf->handle, sizeof(h));
  void* base = nullptr;
  const cudaError_t before = cudaPeekAtLastError();
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess || base == nullptr) {
    if (before == cudaSuccess) cudaGetLastError();
    return EP_ERR_CUDA;
  }
  *mapped_base = base;
  *ptr = static_cast<char*>(base) + buf->offset;
  return EP_OK;
}

int ep_ipc_close(void* mapped_base) {
  if (mapped_base == nullptr) return EP_ERR_INVALID_ARG;
  const cudaError_t before = cudaPeekAtLastError();
  if (cudaIpcCloseMemHandle(mapped_base) != cudaSuccess) {
    if (before == cudaSuccess) cudaGetLastError();
    return EP_ERR_CUDA;
  }
  return EP_OK;
}

}  // extern "C"
