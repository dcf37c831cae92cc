// Shared device/host helpers of libep.so (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "ep.h"

namespace ep {

// ---------------------------------------------------------------- host side

extern std::atomic<uint64_t> g_launches;

inline void count_launch(uint64_t n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

inline int launch_status() { return cudaGetLastError() == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with programmatic dependent launch allowed: the kernel may be
// scheduled while its predecessor in the stream finishes, and must call
// wait_for_predecessor() before touching memory the predecessor writes or
// reads (the row movers do so first thing).
inline cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, void** args, size_t smem, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

int num_sms();  // cached per device
bool raise_smem_limit(const void* fn, size_t bytes);  // never lowers; thread-safe

// Pairs per tile of the histogram / rank scatter passes.  The largest of
// 2048, 4096, 8192 that still gives two tiles per SM (so small problems spread
// over the GPU and large ones amortise the per-tile scan), never below 2048.
inline int tile_pairs_for(int64_t P) {
  const int64_t want = 2 * 148;
  if (P >= want * 8192) return 8192;
  if (P >= want * 4096) return 4096;
  return 2048;
}

inline int64_t num_tiles(int64_t P, int tile) { return (P + tile - 1) / tile; }

// Workspace layout (bytes): [0,256) header (ticket counter), then the
// decoupled look-back words u64 [ntiles][E], then tile_excl i32 [ntiles][E],
// then loads i32 [E] (align-sort's own histogram).
struct WsLayout {
  size_t status_off, excl_off, loads_off, bytes, clear_bytes;
};
inline WsLayout ws_layout(int64_t P, int E) {
  const int tile = tile_pairs_for(P);
  const int64_t nt = num_tiles(P, tile);
  WsLayout l;
  l.status_off = 256;
  l.excl_off = l.status_off + (size_t)nt * E * 8;
  l.excl_off = (l.excl_off + 255) & ~(size_t)255;
  l.loads_off = l.excl_off + (size_t)nt * E * 4;
  l.loads_off = (l.loads_off + 255) & ~(size_t)255;
  l.bytes = l.loads_off + (size_t)E * 4 + 256;
  l.clear_bytes = l.status_off + (size_t)nt * E * 8;
  return l;
}

// Plan buffer layout: fills EpPlanLayout (offsets in int32 words).
void plan_layout(int E, int R, EpPlanLayout* L);

// Common argument checks for (T, K, E).
inline bool valid_tke(int64_t T, int K, int E) {
  if (T < 0 || K < 1 || K > 32 || E < 1 || E > EP_MAX_EXPERTS || K > E) return false;
  if (T * (int64_t)K >= ((int64_t)1 << 31)) return false;
  return true;
}

// ------------------------------------------------------------- device side

__device__ __forceinline__ void flag(int32_t* dev_status, int32_t bits) {
  if (dev_status) atomicOr(dev_status, bits);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Wall-clock bound for every wait inside a kernel (a look-back on another
// CTA, an mbarrier of an asynchronous copy): after it the kernel reports a
// timeout bit and goes on, so no wait can hang the device.
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Lanes of the warp holding the same key as this lane (the result of
// __match_any_sync), built from one ballot per key bit: for every bit, keep the
// lanes that agree with this lane on it.  Keys must lie in [0, 2^nbits).  A
// fixed, short run of pipelined ballots, whatever the number of distinct keys
// in the warp.  All 32 lanes must call it with the same nbits.
__device__ __forceinline__ uint32_t warp_match(uint32_t key, int nbits) {
  uint32_t m = 0xffffffffu;
  for (int b = 0; b < nbits; ++b) {
    const uint32_t bit = (key >> b) & 1u;
    const uint32_t bal = __ballot_sync(0xffffffffu, bit);
    m &= bit ? bal : ~bal;
  }
  return m;
}

// Bits needed for keys 0..n-1.
__host__ __device__ __forceinline__ int key_bits(int n) {
  int b = 1;
  while ((1 << b) < n) ++b;
  return b;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// --- mbarrier and bulk-copy (TMA) wrappers --------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Block until the preceding kernel in the stream has completed and its memory
// is visible (a no-op for a kernel not launched by launch_pdl).
__device__ __forceinline__ void wait_for_predecessor() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Wait (bounded by WAIT_LIMIT_NS) for phase `parity` of an mbarrier.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) return false;
  return true;
}

// global -> shared bulk copy completing on an mbarrier (bytes % 16 == 0,
// both addresses 16-byte aligned)
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// shared -> global bulk copy in the calling thread's bulk async-group
__device__ __forceinline__ void bulk_store(void* gmem_dst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
               "r"(smem_addr(smem_src)), "r"(bytes)
               : "memory");
}

// An L2 policy that marks the lines an access brings in as first to evict
// (for data written or read once).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// bulk_store with an L2 cache policy (from l2_evict_first_policy)
__device__ __forceinline__ void bulk_store_hint(void* gmem_dst, const void* smem_src, uint32_t bytes, uint64_t pol) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(gmem_dst),
               "r"(smem_addr(smem_src)), "r"(bytes), "l"(pol)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Two fp32 values to one packed bf16x2 word (lo in bits 0-15, hi in 16-31),
// each rounded to nearest, ties to even, by the hardware conversion (one
// instruction for both).  For every non-NaN input this is the IEEE rounding
// (overflow to Inf, subnormals kept); a NaN comes out as the canonical bf16
// NaN (a quiet NaN with its payload bits dropped).
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Rank-local form: address of global row g in the R ranks' buffers.  Ranks
// hold rows_per_rank rows each (rank_first == NULL: rank g / rows_per_rank), or
// rank r's rows start at rank_first[r] (ascending, rank_first[0] = 0) and fit
// in its buffer of rows_per_rank rows.  nullptr when the rank's table entry is
// zero or not 16-byte aligned, or the row falls past its rank's buffer.
__device__ __forceinline__ char* peer_row(const uint64_t* __restrict__ peers, const int32_t* __restrict__ rank_first,
                                          int R, int64_t rows_per_rank, int64_t g, int64_t row_bytes) {
  int64_t d, lr;
  if (rank_first) {
    int lo = 0, hi = R - 1;  // last rank whose first row is <= g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(rank_first + mid) <= g)
        lo = mid;
      else
        hi = mid - 1;
    }
    d = lo;
    lr = g - __ldg(rank_first + lo);
  } else {
    d = g / rows_per_rank;
    lr = g - d * rows_per_rank;
  }
  if (d < 0 || d >= R || lr < 0 || lr >= rows_per_rank) return nullptr;
  const uint64_t base = __ldg(peers + d);
  if (!base || (base & 15u)) return nullptr;
  return reinterpret_cast<char*>(base) + lr * row_bytes;
}

// 16-byte global loads that skip L1 allocation (streamed once)
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Block-wide exclusive scan of one int32 per thread (blockDim.x <= 1024,
// a multiple of 32).  `warp_sums` is shared scratch of 32 ints.  Returns the
// exclusive prefix; *total gets the block sum.  Contains __syncthreads.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_sums, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int32_t x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int32_t y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t s = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, s, d);
      if (lane >= d) s += y;
    }
    if (lane < nwarps) warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  int32_t base = warp > 0 ? warp_sums[warp - 1] : 0;
  int32_t tot = warp_sums[nwarps - 1];
  __syncthreads();
  if (total) *total = tot;
  return base + x - v;
}

// Block-wide exclusive scan of a[0..n) in shared memory (any n), in place;
// returns the total.  Each thread scans a contiguous segment.
__device__ __forceinline__ int32_t block_scan_array(int32_t* a, int n, int32_t* warp_sums) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b = threadIdx.x * per, e = min(n, b + per);
  int32_t s = 0;
  for (int i = b; i < e; ++i) s += a[i];
  int32_t total;
  int32_t run = block_exclusive_scan(s, warp_sums, &total);
  for (int i = b; i < e; ++i) {
    const int32_t v = a[i];
    a[i] = run;
    run += v;
  }
  __syncthreads();
  return total;
}

}  // namespace ep
