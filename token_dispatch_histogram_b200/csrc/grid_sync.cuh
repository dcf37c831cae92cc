// Grid-wide synchronisation for cooperative launches (all CTAs co-resident):
// a counting barrier and a flag wait on global words, every wait bounded by
// %globaltimer (WAIT_LIMIT_NS); a wait that runs out sets
// EP_DEV_LOOKBACK_TIMEOUT and lets the CTA go on, so no launch can hang.
#pragma once

#include "common.cuh"

namespace ep {

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Thread 0 waits (bounded) until *ctr >= target; the block follows.
static __device__ void wait_at_least(uint32_t* ctr, uint32_t target, int32_t* dev_status) {
  if (threadIdx.x == 0 && ld_acquire_u32(ctr) < target) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u32(ctr) < target) {
      __nanosleep(32);
      if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
        flag(dev_status, EP_DEV_LOOKBACK_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
}

// Barrier over all CTAs of the cooperative grid (they are co-resident).
static __device__ void grid_barrier(uint32_t* ctr, uint32_t target, int32_t* dev_status) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
  }
  wait_at_least(ctr, target, dev_status);
}

}  // namespace ep
