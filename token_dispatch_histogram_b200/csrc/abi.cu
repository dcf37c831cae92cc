// Library-wide entry points of libep.so: version, launch counter, status read,
// and the per-device SM count used to size persistent grids.
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace ep {

std::atomic<uint64_t> g_launches{0};

int num_sms() {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device, never lowering it: two host threads launching the same
// kernel with different sizes cannot undo each other's setting between a
// set and a launch.
bool raise_smem_limit(const void* fn, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> limits;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  size_t& cur = limits[std::make_pair(dev, fn)];
  if (bytes <= cur) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) return false;
  cur = bytes;
  return true;
}

}  // namespace ep

extern "C" const char* ep_version(void) { return "token_dispatch_histogram_b200 0.1 (sm_100a)"; }

extern "C" uint64_t ep_launch_count(void) { return ep::g_launches.load(std::memory_order_relaxed); }

extern "C" int ep_status_read(const int32_t* dev_status, int32_t* host_status, cudaStream_t stream) {
  if (!dev_status || !host_status) return EP_ERR_ARG;
  if (cudaMemcpyAsync(host_status, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return EP_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return EP_ERR_CUDA;
  return EP_OK;
}
