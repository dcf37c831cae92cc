// a1. Per-expert loads T_e and max_vio, plus the per-tile per-expert prefix
// counts that the stable layout and the align-sort scatter read back.
//
// [FR] "Pourquoi le parallélisme d'experts est-il nécessaire" (news.hamidun.com
// MoonEP article): max_vio = max_e(T_e / T̄) - 1, zero for perfect balance, T̄
// the mean load P/E.
//
// One kernel, one pass over topk_ids:
//  - each CTA takes a tile of consecutive flattened pairs (tile index from an
//    atomic ticket, so a CTA only ever waits on tiles that started earlier),
//  - builds the tile's histogram in shared memory (integer atomics: a sum, so
//    the order they are served in does not matter),
//  - publishes it and resolves its exclusive prefix over earlier tiles with a
//    decoupled look-back (Merrill & Garland, "Single-pass Parallel Prefix Scan
//    with Decoupled Look-back", 2016), one 64-bit {flag, value} word per
//    (tile, expert), every wait bounded,
//  - the last tile's inclusive prefix is T_e; it also reduces max_e T_e.
// Only integer adds feed the outputs, so they do not depend on scheduling.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace ep {

constexpr int HIST_THREADS = 512;
constexpr uint64_t FLAG_AGGREGATE = 1ull << 32;
constexpr uint64_t FLAG_PREFIX = 2ull << 32;

__global__ void __launch_bounds__(HIST_THREADS)
    k_hist_lookback(const int32_t* __restrict__ topk, int64_t P, int E, int tile, int ntiles, uint32_t* ticket,
                    uint64_t* status, int32_t* __restrict__ tile_excl, int32_t* __restrict__ loads,
                    double* __restrict__ max_vio, int32_t* dev_status) {
  extern __shared__ int32_t s_hist[];  // [E]
  __shared__ int s_tile, s_bad;
  __shared__ int32_t s_max[HIST_THREADS / 32];
  if (threadIdx.x == 0) {
    s_tile = (int)atomicAdd(ticket, 1u);
    s_bad = 0;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int t = s_tile;
  const int lane = threadIdx.x & 31;
  const int64_t p0 = (int64_t)t * tile;
  const int64_t p1 = min(P, p0 + tile);

  for (int64_t base = p0; base < p1; base += blockDim.x) {
    const int64_t p = base + threadIdx.x;
    if (p < p1) {
      const int e = __ldg(topk + p);
      if (e >= 0 && e < E)
        atomicAdd(&s_hist[e], 1);  // a sum: the order the lanes are served in does not matter
      else
        s_bad = 1;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_bad) flag(dev_status, EP_DEV_BAD_EXPERT_ID);

  int32_t my_max = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t agg = s_hist[e];
    int32_t excl = 0;
    uint64_t* mine = status + (int64_t)t * E + e;
    if (t == 0) {
      st_relaxed_u64(mine, FLAG_PREFIX | (uint32_t)agg);
    } else {
      st_relaxed_u64(mine, FLAG_AGGREGATE | (uint32_t)agg);
      int j = t - 1;
      int spins = 0;
      uint64_t t0 = 0;
      while (j >= 0) {
        const uint64_t w = ld_relaxed_u64(status + (int64_t)j * E + e);
        const uint64_t f = w & (3ull << 32);
        if (f == 0) {  // predecessor not published yet: bounded wait
          if (++spins > 32) {
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) {
              t0 = now;
            } else if (now - t0 > WAIT_LIMIT_NS) {
              flag(dev_status, EP_DEV_LOOKBACK_TIMEOUT);
              break;
            }
            __nanosleep(100);
          }
          continue;
        }
        excl += (int32_t)(uint32_t)w;
        if (f == FLAG_PREFIX) break;
        --j;
      }
      st_relaxed_u64(mine, FLAG_PREFIX | (uint32_t)(excl + agg));
    }
    tile_excl[(int64_t)t * E + e] = excl;
    if (t == ntiles - 1) {
      const int32_t total = excl + agg;
      if (loads) loads[e] = total;
      my_max = max(my_max, total);
    }
  }
  if (t == ntiles - 1 && max_vio) {
#pragma unroll
    for (int d = 16; d; d >>= 1) my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, d));
    if (lane == 0) s_max[threadIdx.x >> 5] = my_max;
    __syncthreads();
    if (threadIdx.x == 0) {
      int32_t m = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = max(m, s_max[w]);
      // (max_e T_e) * E / P - 1, fp64, each step rounded once (product exact)
      *max_vio = __dsub_rn(__ddiv_rn(__dmul_rn((double)m, (double)E), (double)P), 1.0);
    }
  }
}

// Histogram of topk_ids into ws (+ optional loads/max_vio).  Shared by
// ep_route_stats and ep_align_sort.
int run_hist(const int32_t* topk, int64_t P, int E, void* ws, int32_t* loads, double* max_vio, int32_t* dev_status,
             cudaStream_t st) {
  const WsLayout l = ws_layout(P, E);
  const int tile = tile_pairs_for(P);
  const int64_t nt = num_tiles(P, tile);
  if (nt == 0) {
    if (loads && cudaMemsetAsync(loads, 0, (size_t)E * 4, st) != cudaSuccess) return EP_ERR_CUDA;
    if (max_vio && cudaMemsetAsync(max_vio, 0, sizeof(double), st) != cudaSuccess) return EP_ERR_CUDA;
    return EP_OK;
  }
  char* w = static_cast<char*>(ws);
  if (cudaMemsetAsync(w, 0, l.clear_bytes, st) != cudaSuccess) return EP_ERR_CUDA;
  k_hist_lookback<<<(unsigned)nt, HIST_THREADS, (size_t)E * 4, st>>>(
      topk, P, E, tile, (int)nt, reinterpret_cast<uint32_t*>(w), reinterpret_cast<uint64_t*>(w + l.status_off),
      reinterpret_cast<int32_t*>(w + l.excl_off), loads, max_vio, dev_status);
  count_launch();
  return launch_status();
}

// Self-test of the bounded look-back: the tile counter starts at 1 and one CTA
// fewer is launched, so tile 0 is never processed and its flag is never set.
// Every later tile's wait on it runs out after WAIT_LIMIT_NS and reports
// EP_DEV_LOOKBACK_TIMEOUT; all accesses stay inside the workspace.
int run_hist_skip_first_tile(const int32_t* topk, int64_t P, int E, void* ws, int32_t* loads, double* max_vio,
                             int32_t* dev_status, cudaStream_t st) {
  const WsLayout l = ws_layout(P, E);
  const int tile = tile_pairs_for(P);
  const int64_t nt = num_tiles(P, tile);
  if (nt < 2) return EP_ERR_ARG;
  char* w = static_cast<char*>(ws);
  if (cudaMemsetAsync(w, 0, l.clear_bytes, st) != cudaSuccess) return EP_ERR_CUDA;
  const uint32_t one = 1;
  if (cudaMemcpyAsync(w, &one, sizeof(one), cudaMemcpyHostToDevice, st) != cudaSuccess) return EP_ERR_CUDA;
  k_hist_lookback<<<(unsigned)(nt - 1), HIST_THREADS, (size_t)E * 4, st>>>(
      topk, P, E, tile, (int)nt, reinterpret_cast<uint32_t*>(w), reinterpret_cast<uint64_t*>(w + l.status_off),
      reinterpret_cast<int32_t*>(w + l.excl_off), loads, max_vio, dev_status);
  count_launch();
  if (cudaStreamSynchronize(st) != cudaSuccess) return EP_ERR_CUDA;  // `one` lives on this stack frame
  return launch_status();
}

}  // namespace ep

using namespace ep;

extern "C" int ep_selftest_lookback_timeout(const int32_t* topk_ids, int64_t T, int K, int E, int32_t* loads,
                                            double* max_vio, void* ws, size_t ws_bytes, int32_t* dev_status,
                                            cudaStream_t stream) {
  if (!valid_tke(T, K, E) || !topk_ids || !loads || !max_vio || !ws || !dev_status) return EP_ERR_ARG;
  const int64_t P = T * K;
  if (ws_bytes < ws_layout(P, E).bytes) return EP_ERR_CAPACITY;
  return run_hist_skip_first_tile(topk_ids, P, E, ws, loads, max_vio, dev_status, stream);
}

extern "C" int ep_workspace_size(int64_t T, int K, int E, size_t* bytes) {
  if (!bytes || !valid_tke(T, K, E)) return EP_ERR_ARG;
  *bytes = ws_layout(T * K, E).bytes;
  return EP_OK;
}

extern "C" int ep_route_stats(const int32_t* topk_ids, int64_t T, int K, int E, int32_t* loads, double* max_vio,
                              void* ws, size_t ws_bytes, int32_t* dev_status, cudaStream_t stream) {
  if (!valid_tke(T, K, E) || !loads || !max_vio || !ws) return EP_ERR_ARG;
  const int64_t P = T * K;
  if (P > 0 && !topk_ids) return EP_ERR_ARG;
  if (ws_bytes < ws_layout(P, E).bytes) return EP_ERR_CAPACITY;
  return run_hist(topk_ids, P, E, ws, loads, max_vio, dev_status, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of ep_route_stats.
//
// Some callers cannot hand this library a scratch buffer: hosts that give a
// kernel only its input and output tensors at enqueue time and forbid device
// allocation there (plugin-style interfaces), or runtimes whose device memory is
// planned once up front.  For them ep_route_stats_noalloc keeps its scratch in
// the fixed array below, which exists on every GPU that loads this library
// until the process exits.  Its device address is looked up (cudaGetSymbolAddress)
// on the first call made in a CUDA context, with that context's device current,
// and cached per device together with the context's unique id; a call made in
// another context of the same device (after cudaDeviceReset, or under a context
// the caller created) looks it up again.  All calls share the array and it keeps
// the last call's contents; the part that must start at zero (the look-back
// words and the tile counter) is cleared on the call's stream, so calls must
// not overlap on the GPU: two calls running at the same time race on the array.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EP_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
struct NoallocEntry {
  unsigned long long ctx_id;
  void* addr;
};
NoallocEntry g_noalloc[64] = {};

// The driver's cuCtxGetCurrent / cuCtxGetId, reached through the runtime's
// entry-point query (so the library needs no link against the driver library).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

int current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || !f1)
      return EP_ERR_CUDA;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || !f2)
      return EP_ERR_CUDA;
    get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return EP_ERR_CUDA;
  *id = 0;  // no context current yet
  if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return EP_ERR_CUDA;
  return EP_OK;
}

int noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return EP_ERR_CUDA;
  if (dev < 0 || dev >= 64) return EP_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long id = 0;
  int rc = current_context_id(&id);
  if (rc != EP_OK) return rc;
  NoallocEntry& ent = g_noalloc[dev];
  if (!ent.addr || id == 0 || ent.ctx_id != id) {
    void* p = nullptr;  // the lookup makes the device's context current if none was
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return EP_ERR_CUDA;
    rc = current_context_id(&id);
    if (rc != EP_OK) return rc;
    ent.addr = p;
    ent.ctx_id = id;
  }
  *out = ent.addr;
  return EP_OK;
}
}  // namespace


extern "C" int ep_route_stats_noalloc(const int32_t* topk_ids, int64_t T, int K, int E, int32_t* loads,
                                      double* max_vio, int32_t* dev_status, cudaStream_t stream) {
  using namespace ep;
  if (!valid_tke(T, K, E) || !loads || !max_vio) return EP_ERR_ARG;
  const int64_t P = T * K;
  if (P > 0 && !topk_ids) return EP_ERR_ARG;
  if (ws_layout(P, E).bytes > (size_t)EP_NOALLOC_SCRATCH_BYTES) return EP_ERR_CAPACITY;
  void* scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc != EP_OK) return rc;
  return run_hist(topk_ids, P, E, scratch, loads, max_vio, dev_status, stream);
}
