// a3. Layout and a4. MoE Align & Sort: a stable counting sort by expert.
//
// Both steps place each routed pair at (start of its expert's group) + (its
// stable rank among the pairs of that expert), ties in flattened (rank, token,
// k) order.  The histogram pass (stats.cu) left, per tile of consecutive pairs
// and per expert, the number of that expert's pairs in all earlier tiles
// (tile_excl).  Here each CTA re-reads its tile, recounts per warp, scans the
// per-warp counts, and walks its pairs in order: a pair's stable rank is
//   tile_excl[tile][e] + (pairs of e in earlier warps of the tile)
//                      + (pairs of e earlier in this warp's sub-tile).
// The last term comes from a warp match over 32 consecutive pairs (one ballot
// per key bit, common.cuh) plus a per-warp running counter.  No atomics feed any output.
//
// Layout  ([GR] "Online planning, zero copy και στατικά σχήματα", twodots.gr
// MoonEP article): an expert's home copy takes its first home_count pairs, its
// replicas the following ranges in match order; the plan gives each copy's
// first row.  Outputs pos (pair -> row), src (row -> pair), pair_slot.
// Align & Sort ([ZH] MoE Align & Sort report): groups padded to block_m;
// sorted_token_ids[off_e + rank] = p; padding and tail hold the sentinel P.
#include "tile_ranks.cuh"

namespace ep {

int run_hist(const int32_t* topk, int64_t P, int E, void* ws, int32_t* loads, double* max_vio, int32_t* dev_status,
             cudaStream_t st);

// base_counts == NULL: the pairs are the whole problem (rows in [0, P)).
// Otherwise (rank-local form) they are source rank base_rank's pairs, counts
// [R, E] is the gathered load matrix, each expert's list position is offset by
// the pairs of that expert on lower source ranks, rows lie in [0, rows_total),
// and src may be NULL.
__global__ void __launch_bounds__(SCAT_THREADS)
    k_layout(const int32_t* __restrict__ topk, int64_t P, int E, int tile, const int32_t* __restrict__ tile_excl,
             const int32_t* __restrict__ base_counts, int base_rank, int64_t rows_total,
             const int32_t* __restrict__ plan, EpPlanLayout L, int32_t* __restrict__ pos, int32_t* __restrict__ src,
             int32_t* __restrict__ pair_slot, int32_t* dev_status) {
  extern __shared__ int32_t sm[];
  const int cap = L.cap;
  int32_t* s_ids = sm;                            // [tile]
  int32_t* s_whist = s_ids + tile;                // [SCAT_WARPS * E]
  int32_t* s_hc = s_whist + SCAT_WARPS * E;       // [E] home_count
  int32_t* s_hb = s_hc + E;                       // [E] home_base
  int32_t* s_cf = s_hb + E;                       // [E] copy_first
  int32_t* s_cc = s_cf + E;                       // [E] copy_cnt
  int32_t* s_rb = s_cc + E;                       // [cap] rep_begin
  int32_t* s_rc = s_rb + cap;                     // [cap] rep_count
  int32_t* s_rbase = s_rc + cap;                  // [cap] rep_base
  int32_t* s_excl = s_rbase + cap;                // [E] (rank-local form) list offset of the tile
  __shared__ int s_flags;
  if (threadIdx.x == 0) s_flags = 0;
  const int32_t* excl_row = tile_excl + (int64_t)blockIdx.x * E;
  if (base_counts) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int32_t b = excl_row[e];
      for (int r = 0; r < base_rank; ++r) b += base_counts[(int64_t)r * E + e];
      s_excl[e] = b;
    }
    excl_row = s_excl;  // read by tile_stable_ranks after its first barrier
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    s_hc[e] = plan[L.home_count + e];
    s_hb[e] = plan[L.home_base + e];
    s_cf[e] = plan[L.copy_first + e];
    s_cc[e] = plan[L.copy_cnt + e];
  }
  const int n_rep = min(plan[L.n_rep], cap);
  for (int m = threadIdx.x; m < n_rep; m += blockDim.x) {
    s_rb[m] = plan[L.rep_begin + m];
    s_rc[m] = plan[L.rep_count + m];
    s_rbase[m] = plan[L.rep_base + m];
  }
  // (tile_stable_ranks begins with __syncthreads after its own loads)
  auto emit = [&](int64_t p, int e, int32_t g) {
    int32_t row = -1, slot = -1;
    if (g < s_hc[e]) {
      row = s_hb[e] + g;
      slot = e;
    } else if (s_cc[e] > 0) {
      int lo = s_cf[e], hi = s_cf[e] + s_cc[e] - 1;  // last replica m with rep_begin[m] <= g
      if (lo >= 0 && hi < n_rep) {
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (s_rb[mid] <= g)
            lo = mid;
          else
            hi = mid - 1;
        }
        const int32_t off = g - s_rb[lo];
        if (off >= 0 && off < s_rc[lo]) {
          row = s_rbase[lo] + off;
          slot = E + lo;
        }
      }
    }
    if (row < 0 || row >= rows_total) {
      atomicOr(&s_flags, EP_DEV_BAD_ROW);
      pos[p] = -1;
      if (pair_slot) pair_slot[p] = -1;
      return;
    }
    pos[p] = row;
    if (src) src[row] = (int32_t)p;
    if (pair_slot) pair_slot[p] = slot;
  };
  auto bad = [&](int64_t p) {
    atomicOr(&s_flags, EP_DEV_BAD_EXPERT_ID);
    pos[p] = -1;
    if (pair_slot) pair_slot[p] = -1;
  };
  const int64_t p0 = (int64_t)blockIdx.x * tile;
  tile_stable_ranks(topk, E, tile, p0, (int)min((int64_t)tile, P - p0), excl_row, s_ids, s_whist, emit, bad);
  __syncthreads();
  if (threadIdx.x == 0 && s_flags) flag(dev_status, s_flags);
}

__global__ void __launch_bounds__(SCAT_THREADS)
    k_align_scatter(const int32_t* __restrict__ topk, int64_t P, int E, int tile, const int32_t* __restrict__ tile_excl,
                    const int32_t* __restrict__ counts, int block_m, int32_t* __restrict__ sorted_ids,
                    int64_t sorted_cap, int32_t* __restrict__ expert_ids, int64_t expert_ids_cap,
                    int32_t* __restrict__ num_post_pad, int32_t* dev_status) {
  extern __shared__ int32_t sm[];
  int32_t* s_ids = sm;                      // [tile]
  int32_t* s_whist = s_ids + tile;          // [SCAT_WARPS * E]
  int32_t* s_off = s_whist + SCAT_WARPS * E;  // [E + 1] padded group offsets
  int32_t* s_cnt = s_off + E + 1;           // [E]
  __shared__ int32_t warp_sums[32];
  __shared__ int s_flags;
  if (threadIdx.x == 0) s_flags = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t c = counts[e];
    s_cnt[e] = c;
    s_off[e] = (c + block_m - 1) / block_m * block_m;
  }
  __syncthreads();
  const int32_t total = block_scan_array(s_off, E, warp_sums);
  if (threadIdx.x == 0) s_off[E] = total;
  // valid entries
  auto emit = [&](int64_t p, int e, int32_t g) { sorted_ids[s_off[e] + g] = (int32_t)p; };
  auto bad = [&](int64_t) { atomicOr(&s_flags, EP_DEV_BAD_EXPERT_ID); };
  const int ntiles = (int)((P + tile - 1) / tile);
  if ((int)blockIdx.x < ntiles) {
    const int64_t p0 = (int64_t)blockIdx.x * tile;
    tile_stable_ranks(topk, E, tile, p0, (int)min((int64_t)tile, P - p0), tile_excl + (int64_t)blockIdx.x * E, s_ids,
                      s_whist, emit, bad);
  }
  __syncthreads();
  // padding of each group, the tail past the padded total, and expert_ids
  const int32_t sentinel = (int32_t)P;
  for (int e = blockIdx.x; e < E; e += gridDim.x)
    for (int32_t i = s_off[e] + s_cnt[e] + threadIdx.x; i < s_off[e + 1]; i += blockDim.x) sorted_ids[i] = sentinel;
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, gstride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = total + gtid; i < sorted_cap; i += gstride) sorted_ids[i] = sentinel;
  const int64_t nblocks = total / block_m;
  for (int64_t b = gtid; b < expert_ids_cap; b += gstride) {
    int32_t owner = -1;
    if (b < nblocks) {
      const int32_t v = (int32_t)(b * block_m);
      int lo = 0, hi = E - 1;  // last e with off[e] <= v (groups with no block share off with the next)
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= v)
          lo = mid;
        else
          hi = mid - 1;
      }
      owner = lo;
    }
    expert_ids[b] = owner;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *num_post_pad = total;
  __syncthreads();
  if (threadIdx.x == 0 && s_flags) flag(dev_status, s_flags);
}

size_t scatter_smem_base(int tile, int E) { return sizeof(int32_t) * ((size_t)tile + (size_t)SCAT_WARPS * E); }

static int run_layout(const int32_t* topk, int64_t P, int E, int tile, int64_t nt, const int32_t* tile_excl,
                      const int32_t* base_counts, int base_rank, int64_t rows_total, const int32_t* plan,
                      const EpPlanLayout& L, int32_t* pos, int32_t* src, int32_t* pair_slot, int32_t* dev_status,
                      cudaStream_t stream) {
  const size_t smem = scatter_smem_base(tile, E) + sizeof(int32_t) * (5 * (size_t)E + 3 * (size_t)L.cap);
  if (smem > 48 * 1024 &&
      !raise_smem_limit((const void*)k_layout, smem))
    return EP_ERR_CUDA;
  k_layout<<<(unsigned)nt, SCAT_THREADS, smem, stream>>>(topk, P, E, tile, tile_excl, base_counts, base_rank,
                                                         rows_total, plan, L, pos, src, pair_slot, dev_status);
  count_launch();
  return launch_status();
}

}  // namespace ep

using namespace ep;

extern "C" int ep_layout(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, const int32_t* plan,
                         size_t plan_words, const void* ws, size_t ws_bytes, int32_t* pos, int32_t* src,
                         int32_t* pair_slot, int32_t* dev_status, cudaStream_t stream) {
  if (!valid_tke(T, K, E) || R < 1 || R > EP_MAX_RANKS || E % R || S < 0 || (int64_t)R * S != T) return EP_ERR_ARG;
  if (!plan || !ws) return EP_ERR_ARG;
  const int64_t P = T * K;
  if (P > 0 && (!topk_ids || !pos || !src)) return EP_ERR_ARG;
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  const WsLayout wl = ws_layout(P, E);
  if (ws_bytes < wl.bytes) return EP_ERR_CAPACITY;
  if (P == 0) return EP_OK;
  const int tile = tile_pairs_for(P);
  const int64_t nt = num_tiles(P, tile);
  const char* w = static_cast<const char*>(ws);
  return run_layout(topk_ids, P, E, tile, nt, reinterpret_cast<const int32_t*>(w + wl.excl_off), nullptr, 0, P, plan, L,
                    pos, src, pair_slot, dev_status, stream);
}

extern "C" int ep_layout_rank(const int32_t* topk_local, int64_t S, int K, int E, int R, int rank,
                              const int32_t* counts, const int32_t* plan, size_t plan_words, const void* ws,
                              size_t ws_bytes, int32_t* pos_local, int32_t* pair_slot, int32_t* dev_status,
                              cudaStream_t stream) {
  if (!valid_tke(S, K, E) || R < 1 || R > EP_MAX_RANKS || E % R || rank < 0 || rank >= R) return EP_ERR_ARG;
  if ((int64_t)R * S * K >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  if (!plan || !ws || !counts) return EP_ERR_ARG;
  const int64_t P = S * K;
  if (P > 0 && (!topk_local || !pos_local)) return EP_ERR_ARG;
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  const WsLayout wl = ws_layout(P, E);
  if (ws_bytes < wl.bytes) return EP_ERR_CAPACITY;
  if (P == 0) return EP_OK;
  const int tile = tile_pairs_for(P);
  const int64_t nt = num_tiles(P, tile);
  const char* w = static_cast<const char*>(ws);
  return run_layout(topk_local, P, E, tile, nt, reinterpret_cast<const int32_t*>(w + wl.excl_off), counts, rank,
                    (int64_t)R * P, plan, L, pos_local, nullptr, pair_slot, dev_status, stream);
}

extern "C" int ep_align_sort(const int32_t* topk_ids, int64_t T, int K, int E, int block_m,
                             int32_t* sorted_token_ids, int64_t sorted_cap, int32_t* expert_ids,
                             int64_t expert_ids_cap, int32_t* num_tokens_post_pad, void* ws, size_t ws_bytes,
                             int32_t* dev_status, cudaStream_t stream) {
  if (!valid_tke(T, K, E) || block_m < 1 || block_m > (1 << 16)) return EP_ERR_ARG;
  if (!sorted_token_ids || !expert_ids || !num_tokens_post_pad || !ws) return EP_ERR_ARG;
  const int64_t P = T * K;
  if (P > 0 && !topk_ids) return EP_ERR_ARG;
  const int64_t need = P + (int64_t)E * (block_m - 1);
  if (need >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  if (sorted_cap < need || expert_ids_cap < (sorted_cap + block_m - 1) / block_m) return EP_ERR_CAPACITY;
  const WsLayout wl = ws_layout(P, E);
  if (ws_bytes < wl.bytes) return EP_ERR_CAPACITY;
  char* w = static_cast<char*>(ws);
  int32_t* counts = reinterpret_cast<int32_t*>(w + wl.loads_off);
  int rc = run_hist(topk_ids, P, E, ws, counts, nullptr, dev_status, stream);
  if (rc != EP_OK) return rc;
  const int tile = tile_pairs_for(P);
  const int64_t nt = num_tiles(P, tile);
  int grid = (int)std::max<int64_t>(nt, 2 * num_sms());
  const size_t smem = scatter_smem_base(tile, E) + sizeof(int32_t) * (2 * (size_t)E + 1);
  if (smem > 48 * 1024 &&
      !raise_smem_limit((const void*)k_align_scatter, smem))
    return EP_ERR_CUDA;
  k_align_scatter<<<grid, SCAT_THREADS, smem, stream>>>(topk_ids, P, E, tile,
                                                        reinterpret_cast<const int32_t*>(w + wl.excl_off), counts,
                                                        block_m, sorted_token_ids, sorted_cap, expert_ids,
                                                        expert_ids_cap, num_tokens_post_pad, dev_status);
  count_launch();
  return launch_status();
}
