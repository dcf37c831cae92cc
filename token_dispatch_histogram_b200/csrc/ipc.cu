// Mapping a buffer of another process into this one, for the peer tables of
// the rank-local form (one rank per process).
//
// [GR] "Online planning, zero copy και στατικά σχήματα" (twodots.gr MoonEP
// article): dispatch writes each token row straight into its final
// expert-grouped row on the receiving rank, and the application reads views of
// that buffer.  Across processes that needs the receiving rank's buffer mapped
// into the sender's address space.  These host calls do that with CUDA IPC
// handles: the owner exports a handle for the allocation that holds its buffer
// (and the buffer's offset in it), the handle travels to the other processes
// (over any host channel, e.g. torch.distributed), and each opens it.  Once
// opened on a GPU other than the owner's, peer access is enabled lazily by the
// driver, and the address is used like any device pointer in the peer tables.
#include <cuda.h>

#include <cstring>

#include "common.cuh"

namespace {

using MemGetAddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

// The driver's cuMemGetAddressRange through the runtime's entry-point query
// (no link against the driver library).
MemGetAddressRangeFn address_range_fn() {
  static MemGetAddressRangeFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<MemGetAddressRangeFn>(f);
  }
  return fn;
}

}  // namespace

static_assert(sizeof(cudaIpcMemHandle_t) == EP_IPC_HANDLE_BYTES, "IPC handle size");

extern "C" int ep_ipc_export(const void* dev_ptr, void* handle, uint64_t* offset) {
  if (!dev_ptr || !handle || !offset) return EP_ERR_ARG;
  MemGetAddressRangeFn range = address_range_fn();
  if (!range) return EP_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS || !base) return EP_ERR_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return EP_ERR_CUDA;
  std::memcpy(handle, &h, sizeof(h));
  *offset = static_cast<uint64_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return EP_OK;
}

extern "C" int ep_ipc_open(const void* handle, uint64_t offset, void** base, void** dev_ptr) {
  if (!handle || !base || !dev_ptr) return EP_ERR_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* b = nullptr;
  if (cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess || !b) return EP_ERR_CUDA;
  *base = b;
  *dev_ptr = static_cast<char*>(b) + offset;
  return EP_OK;
}

extern "C" int ep_ipc_close(void* base) {
  if (!base) return EP_ERR_ARG;
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
