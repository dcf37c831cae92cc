// The stable-rank walk over one tile of routed pairs, shared by the layout,
// align-sort and quota-layout kernels: a pair's rank among all pairs of its
// expert = (pairs of that expert before the tile) + (pairs of it in earlier
// warps of the tile) + (earlier pairs of it in this warp's sub-tile).  The last
// term comes from a warp match over 32 consecutive pairs (one ballot per key
// bit) plus a per-warp running counter.  The per-warp counts behind the second
// term are summed with shared-memory integer atomics (a sum, so the order the
// lanes are served in does not matter); no atomic feeds a rank directly.
#pragma once

#include "common.cuh"

namespace ep {

constexpr int SCAT_THREADS = 512;
constexpr int SCAT_WARPS = SCAT_THREADS / 32;

// Stable ranks of the n pairs p0 .. p0+n-1 (one tile, n <= tile, tile a
// multiple of 32 * SCAT_WARPS); excl_row[e] = pairs of e before p0.  Calls
// emit(p, e, g) for every valid pair (g = rank of p among all pairs of expert
// e) and bad(p) for pairs whose id is outside [0, E).  s_ids: [tile] ints,
// s_whist: [SCAT_WARPS][E] ints.  Two halves: tile_ranks_prepare (loads the
// ids, counts them per warp and turns the counts into each warp's first rank
// per expert) and tile_ranks_walk (the ranks themselves, emitted in order),
// so a caller can run the first before the data emit needs is ready.
__device__ __forceinline__ void tile_ranks_prepare(const int32_t* __restrict__ topk, int E, int tile, int64_t p0,
                                                   int n, const int32_t* __restrict__ excl_row, int32_t* s_ids,
                                                   int32_t* s_whist) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < tile; i += blockDim.x) {
    int e = -1;
    if (i < n) {
      e = __ldg(topk + p0 + i);
      if (e < 0 || e >= E) e = -2;  // invalid id (reported by bad())
    }
    s_ids[i] = e;
  }
  for (int i = threadIdx.x; i < SCAT_WARPS * E; i += blockDim.x) s_whist[i] = 0;
  __syncthreads();

  const int sub = tile / SCAT_WARPS;  // pairs per warp, a multiple of 32
  int32_t* my = s_whist + warp * E;
  for (int c = 0; c < sub; c += 32) {  // counts only: integer atomics (order-free) into the warp's own row
    const int e = s_ids[warp * sub + c + lane];
    if (e >= 0) atomicAdd(my + e, 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = excl_row[e];
#pragma unroll 4
    for (int w = 0; w < SCAT_WARPS; ++w) {
      const int32_t c = s_whist[w * E + e];
      s_whist[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
}

template <class Emit, class Bad>
__device__ __forceinline__ void tile_ranks_walk(int E, int tile, int64_t p0, int n, const int32_t* s_ids,
                                                int32_t* s_whist, Emit emit, Bad bad) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = tile / SCAT_WARPS;
  const int nbits = key_bits(E + 2);
  int32_t* my = s_whist + warp * E;
  const uint32_t lt = lanemask_lt();
  for (int c = 0; c < sub; c += 32) {
    const int i = warp * sub + c + lane;
    const int e = s_ids[i];
    const uint32_t peers = warp_match((uint32_t)(e + 2), nbits);
    int32_t base = 0;
    if (e >= 0) base = my[e];
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) my[e] = base + __popc(peers);
    __syncwarp();
    if (i < n) {
      if (e >= 0)
        emit(p0 + i, e, base + __popc(peers & lt));
      else
        bad(p0 + i);
    }
  }
}

template <class Emit, class Bad>
__device__ __forceinline__ void tile_stable_ranks(const int32_t* __restrict__ topk, int E, int tile, int64_t p0, int n,
                                                  const int32_t* __restrict__ excl_row, int32_t* s_ids,
                                                  int32_t* s_whist, Emit emit, Bad bad) {
  tile_ranks_prepare(topk, E, tile, p0, n, excl_row, s_ids, s_whist);
  tile_ranks_walk(E, tile, p0, n, s_ids, s_whist, emit, bad);
}

}  // namespace ep
