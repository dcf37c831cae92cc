// The whole route phase -- a1 stats, a2 plan, a3 layout, a4 align-sort -- in
// ONE cooperative launch.  Same outputs as ep_route_stats + ep_plan + ep_layout
// + ep_align_sort, bit for bit.
//
// Why: every step of the route phase moves only a few MB (4-12 bytes per pair),
// so on B200 it is bound by latency chains, not HBM: launch gaps, the serial
// look-back, one CTA planning while the GPU idles.  Here all CTAs stay resident
// (cooperative launch) and meet at grid barriers instead:
//   1. each CTA counts its tile per warp (shared-memory integer atomics into
//      the warp's own row), writes the tile's per-expert counts, column-major
//      [E][tiles], and adds them into the totals T_e (integer atomics: the
//      sums do not depend on order);
//   -- grid barrier --
//   2. one extra CTA with no tile reads T_e and runs the planner
//      (plan_block.cuh) and max_vio at once, then raises a flag; meanwhile the
//      tile CTAs scan the per-expert columns in parallel (exclusive tile
//      prefixes), meet at a second barrier of their own, and write what the
//      align-sort needs no rank for (group offsets, padding, block experts);
//   4. after the flag, every CTA walks its tile once: each pair's stable rank
//      within its expert gives both its align-sort slot (sorted ids) and its
//      layout row (pos / src / pair_slot from the plan).
// A pair's stable rank within its expert = (its tile's prefix) + (earlier warps
// of the tile) + (earlier chunks of its warp) + popc(peers & lanemask_lt):
// integer adds only, so nothing depends on scheduling.  Every wait is bounded.
// Large tiles (STAGE_MIN_TILE pairs and more) stage the walk's pairs in shared
// memory in (expert, rank) order and write the align-sort ids and src from a
// sweep over the experts' runs, as consecutive words instead of scattered ones.
//
// Fused layout + dispatch (ep_route_dispatch_fused, DISPATCH = true): once a
// tile CTA has written its pairs' rows (step 4), it copies the hidden rows of
// the tokens its tile touches straight to those rows -- the dispatch kernel's
// scheme (one TMA bulk load per token row into a shared-memory stage, one bulk
// store per pair) run by a few warps of the CTA, with the pair rows read back
// from pos.  A token whose pairs straddle two tiles is loaded by both CTAs,
// each storing only its own pairs.  Same outputs as ep_route_fused followed by
// ep_dispatch, bit for bit; no launch and no grid-wide wait between them.
#include <algorithm>

#include "grid_sync.cuh"
#include "plan_block.cuh"

namespace ep {

int fused_route_separate(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, int32_t* loads,
                         double* max_vio, int32_t* plan, size_t plan_words, int32_t* pos, int32_t* src,
                         int32_t* pair_slot, int block_m, int32_t* sorted_ids, int64_t sorted_cap,
                         int32_t* expert_ids, int64_t expert_ids_cap, int32_t* ntpp, void* ws, size_t ws_bytes,
                         int32_t* dev_status, cudaStream_t stream);
bool dispatch_shape_ok(int64_t H, int K);  // rows.cu

constexpr int FUSED_THREADS = 512;
constexpr int FUSED_WARPS = FUSED_THREADS / 32;

struct FusedArgs {
  const int32_t* topk;
  int64_t P;
  int E, R;
  int32_t SK;
  int tile, ntiles;
  uint32_t* sync;  // [0] barrier arrivals, [1] plan-ready flag (zeroed by the host)
  int32_t* counts; // [E][ntiles] tile counts, then exclusive tile prefixes
  int32_t* tot;    // [E] T_e, summed by atomics (zeroed by the host)
  int32_t* loads;
  double* max_vio;
  int32_t* plan;
  EpPlanLayout L;
  int32_t* pos;
  int32_t* src;
  int32_t* pair_slot;
  int block_m;
  int32_t* sorted_ids;
  int64_t sorted_cap;
  int32_t* expert_ids;
  int64_t expert_ids_cap;
  int32_t* ntpp;
  int32_t* dev_status;
  int stage;            // tile CTAs stage their pairs in shared memory; src and sorted ids go out in runs
  // fused dispatch (DISPATCH = true only)
  const uint8_t* x;     // [T, row_bytes] token rows
  uint8_t* buf;         // [buf_rows, row_bytes]
  int64_t buf_rows;
  uint32_t row_bytes;
  int K;
  int copy_warps;       // warps of each tile CTA that copy rows
  int copy_stages;      // shared-memory row stages per copying warp
  uint32_t copy_off;    // byte offset of the copy region in dynamic shared memory
};

constexpr int WALK_UNROLL = 8;  // tile loads each lane keeps in flight during a walk
constexpr int SWEEP_RUN = 256;  // entries of an expert's run its own warp writes; the rest, all warps

// A pair's layout row from its expert e and stable rank g within e (the plan
// in shared memory): the home copy takes ranks [0, home_count), then the
// expert's replicas in order, replica m ranks [rep_begin, rep_begin +
// rep_count).  slot = e (home) or E + m; -1 when g lies outside every copy.
struct RowMap {
  const int32_t *hc, *hb, *cf, *cc, *rb, *rc, *rbase;
  int n_rep, E;
  __device__ __forceinline__ int32_t row(int e, int32_t g, int32_t* slot) const {
    if (g < hc[e]) {
      *slot = e;
      return hb[e] + g;
    }
    if (cc[e] > 0) {
      int lo = cf[e], hi = cf[e] + cc[e] - 1;  // last replica with rep_begin <= g
      if (lo >= 0 && hi < n_rep) {
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (rb[mid] <= g)
            lo = mid;
          else
            hi = mid - 1;
        }
        const int32_t off = g - rb[lo];
        if (off >= 0 && off < rc[lo]) {
          *slot = E + lo;
          return rbase[lo] + off;
        }
      }
    }
    *slot = -1;
    return -1;
  }
};

// Walk this warp's part of the tile in flattened order; `run` is the warp's
// running per-expert count (initialised to the rank of its first pair).  Ids
// are loaded WALK_UNROLL chunks at a time so the loads overlap.
template <class Emit>
__device__ __forceinline__ void walk_warp(const int32_t* __restrict__ topk, int64_t P, int E, int64_t wp0, int sub,
                                          int32_t* run, Emit emit, int* s_bad) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  const int nbits = key_bits(E + 2);
  for (int c0 = 0; c0 < sub; c0 += 32 * WALK_UNROLL) {
    int ids[WALK_UNROLL];
#pragma unroll
    for (int u = 0; u < WALK_UNROLL; ++u) {
      const int64_t p = wp0 + c0 + u * 32 + lane;
      ids[u] = (c0 + u * 32 < sub && p < P) ? __ldg(topk + p) : 0;
    }
#pragma unroll
    for (int u = 0; u < WALK_UNROLL; ++u) {
      if (c0 + u * 32 >= sub) break;  // warp-uniform
      const int64_t p = wp0 + c0 + u * 32 + lane;
      int e = ids[u];
      if (p >= P)
        e = -1;
      else if (e < 0 || e >= E)
        e = -2;
      const uint32_t peers = warp_match((uint32_t)(e + 2), nbits);
      int32_t base = 0;
      if (e >= 0) base = run[e];
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) run[e] = base + __popc(peers);
      __syncwarp();
      if (e >= 0)
        emit(p, e, base + __popc(peers & lt));
      else if (e == -2)
        *s_bad = 1;
    }
  }
}

// Copy the rows of the tokens that pairs [pb, pe) belong to: buf[pos[p]] =
// x[p / K] for every p in [pb, pe).  Warps 0 .. copy_warps-1 take the tokens in
// turn, each with a ring of copy_stages row stages (TMA bulk load of the token
// row, completion on an mbarrier; one bulk store per pair of the range, with
// an L2 evict-first policy as in the dispatch kernel).  pos is read back with
// L2 loads: this CTA wrote it, before a block barrier.  Rows outside
// [0, buf_rows) (pos = -1 for an invalid id) are reported, never written.
__device__ void route_copy_rows(const FusedArgs& a, int64_t pb, int64_t pe, uint8_t* cs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= a.copy_warps || pe <= pb) return;
  const int K = a.K, stages = a.copy_stages, nw = a.copy_warps;
  const uint32_t row_bytes = a.row_bytes;
  const uint32_t stride_b = (row_bytes + 127u) & ~127u;
  uint8_t* st0 = cs + (size_t)warp * stages * stride_b;
  uint64_t* bars = reinterpret_cast<uint64_t*>(cs + (size_t)nw * stages * stride_b) + (size_t)warp * stages;
  int32_t* ring = reinterpret_cast<int32_t*>(cs + (size_t)nw * stages * (stride_b + 8)) + (size_t)warp * stages * K;
  const uint64_t evict_first = l2_evict_first_policy();
  if (lane == 0)
    for (int s = 0; s < stages; ++s) mbar_init(&bars[s], 1);
  fence_mbar_init();
  __syncwarp();

  constexpr int32_t NOT_MINE = INT32_MIN;  // a pair of the token outside [pb, pe)
  const int64_t t_lo = pb / K, t_hi = (pe - 1) / K + 1;
  const int64_t first = t_lo + warp;
  const int64_t njobs = first < t_hi ? (t_hi - first + nw - 1) / nw : 0;
  auto issue = [&](int64_t j) {
    const int s = (int)(j % stages);
    const int64_t t = first + j * nw;
    if (lane < K) {
      const int64_t p = t * K + lane;
      ring[s * K + lane] = (p >= pb && p < pe) ? __ldcg(a.pos + p) : NOT_MINE;
    }
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[s], row_bytes);
      bulk_load(st0 + (size_t)s * stride_b, a.x + t * (int64_t)row_bytes, row_bytes, &bars[s]);
    }
  };
  const int64_t pro = njobs < stages ? njobs : (int64_t)stages;
  for (int64_t j = 0; j < pro; ++j) issue(j);
  int64_t issued = pro;

  int32_t bad = 0;
  bool ok = true;
  int64_t j = 0;
  for (; j < njobs; ++j) {
    const int s = (int)(j % stages);
    const uint32_t parity = (uint32_t)((j / stages) & 1);
    const bool landed = mbar_wait_bounded(&bars[s], parity);
    if (!__all_sync(0xffffffffu, landed)) {
      ok = false;
      break;
    }
    if (lane < K) {
      const int32_t row = ring[s * K + lane];
      if (row != NOT_MINE) {
        if (row >= 0 && row < a.buf_rows)
          bulk_store_hint(a.buf + (int64_t)row * row_bytes, st0 + (size_t)s * stride_b, row_bytes, evict_first);
        else
          bad = EP_DEV_BAD_ROW;
      }
    }
    bulk_commit();
    if (j >= 1 && issued < njobs) {  // refill the previous job's stage once its stores have read it
      bulk_wait_read<1>();
      __syncwarp();
      issue(issued);
      ++issued;
    }
  }
  if (!ok) {  // a row did not land in time: report, and give the loads in flight a bounded chance to land
    if (lane == 0) flag(a.dev_status, EP_DEV_COPY_TIMEOUT);
    for (int64_t q = j; q < issued; ++q) mbar_wait_bounded(&bars[(int)(q % stages)], (uint32_t)((q / stages) & 1));
  }
  bulk_wait_all();
  if (bad) flag(a.dev_status, bad);
}

template <bool DISPATCH>
__global__ void __launch_bounds__(FUSED_THREADS) k_route_fused(FusedArgs a) {
  extern __shared__ __align__(128) int32_t sm[];
  // CTAs 0..NT-1 own one tile each; the last CTA (NT) owns none and runs the
  // planner, so the plan overlaps the align-sort walks of the others.
  const int E = a.E, tile = a.tile, G = gridDim.x, NT = a.ntiles, t = blockIdx.x, tid = threadIdx.x;
  const bool has_tile = t < NT, planner = t == NT;
  const int warp = tid >> 5, lane = tid & 31;
  const int sub = tile / FUSED_WARPS;
  const int cap = a.L.cap;
  const int region_a = max(FUSED_WARPS * E, plan_work_words(E, a.R));
  int32_t* s_wb = sm;                          // [16][E] per-warp exclusive counts within the tile
  int32_t* s_run = s_wb + FUSED_WARPS * E;     // region A: running counters, or the planner's work space
  int32_t* s_loads = s_run + region_a;         // [E]
  int32_t* s_excl = s_loads + E;               // [E] this tile's prefix per expert
  int32_t* s_off = s_excl + E;                 // [E + 1] align-sort group offsets
  int32_t* s_hc = s_off + E + 1;               // [E] home_count
  int32_t* s_hb = s_hc + E;                    // [E] home_base
  int32_t* s_cf = s_hb + E;                    // [E] copy_first
  int32_t* s_cc = s_cf + E;                    // [E] copy_cnt
  int32_t* s_rb = s_cc + E;                    // [cap] rep_begin
  int32_t* s_rc = s_rb + cap;                  // [cap] rep_count
  int32_t* s_rbase = s_rc + cap;               // [cap] rep_base
  // staged sweep only: tile count per expert, its run's base in the stage
  // (less the tile prefix), experts with runs longer than SWEEP_RUN, and the
  // tile's pairs (offsets from the tile's first pair) in (expert, rank) order
  int32_t* s_tc = s_rbase + cap;               // [E]
  int32_t* s_tb = s_tc + E;                    // [E]
  int32_t* s_long = s_tb + E;                  // [E]
  uint16_t* s_stage = reinterpret_cast<uint16_t*>(s_long + E);  // [tile]
  __shared__ int32_t warp_sums[32];
  __shared__ int s_bad, s_badrow, s_nlong;
  __shared__ int32_t s_max[FUSED_WARPS];
  const int64_t p0 = (int64_t)t * tile;
  const int64_t wp0 = p0 + (int64_t)warp * sub;

  // ---- 1. per-warp counts of this tile
  if (tid == 0) {
    s_bad = 0;
    s_badrow = 0;
  }
  for (int i = tid; i < FUSED_WARPS * E; i += FUSED_THREADS) s_wb[i] = 0;
  __syncthreads();
  if (has_tile) {
    // counts only: shared-memory integer atomics into the warp's own row (the
    // sum does not depend on the order the lanes are served in)
    int32_t* my = s_wb + warp * E;
    for (int c0 = 0; c0 < sub; c0 += 32 * WALK_UNROLL) {
      int ids[WALK_UNROLL];
#pragma unroll
      for (int u = 0; u < WALK_UNROLL; ++u) {
        const int64_t p = wp0 + c0 + u * 32 + lane;
        ids[u] = (c0 + u * 32 + lane < sub && p < a.P) ? __ldg(a.topk + p) : -1;
      }
#pragma unroll
      for (int u = 0; u < WALK_UNROLL; ++u)
        if (ids[u] >= 0 && ids[u] < E) atomicAdd(my + ids[u], 1);
    }
  }
  __syncthreads();
  if (has_tile) {
    for (int e = tid; e < E; e += FUSED_THREADS) {
      int32_t run = 0;
      for (int w = 0; w < FUSED_WARPS; ++w) {
        const int32_t c = s_wb[w * E + e];
        s_wb[w * E + e] = run;
        run += c;
      }
      a.counts[(int64_t)e * NT + t] = run;
      if (a.stage) s_tc[e] = run;
      if (run) atomicAdd(a.tot + e, run);
    }
  }
  grid_barrier(a.sync, (uint32_t)G, a.dev_status);

  // ---- 2. the planner CTA plans from T_e at once; the tile CTAs scan every
  // expert column over the tiles (exclusive prefixes; totals = T_e again) and
  // meet at a barrier of their own
  if (planner) {
    for (int e = tid; e < E; e += FUSED_THREADS) s_loads[e] = __ldcg(a.tot + e);
    __syncthreads();
  } else {
    for (int e = t; e < E; e += NT) {
      const int32_t total = block_scan_inplace(a.counts + (int64_t)e * NT, NT, warp_sums);
      if (tid == 0) a.loads[e] = total;
    }
    grid_barrier(a.sync, (uint32_t)(G + NT), a.dev_status);
    for (int e = tid; e < E; e += FUSED_THREADS) {
      s_loads[e] = __ldcg(a.loads + e);
      s_excl[e] = __ldcg(a.counts + (int64_t)e * NT + t);
    }
    __syncthreads();
  }

  // ---- 3. planner on the last CTA; the align-sort's group offsets, padding
  // and block experts on the tile CTAs
  if (planner) {
    int32_t m = 0;
    for (int e = tid; e < E; e += FUSED_THREADS) m = max(m, s_loads[e]);
#pragma unroll
    for (int d = 16; d; d >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, d));
    if (lane == 0) s_max[warp] = m;
    __syncthreads();
    if (tid == 0) {
      int32_t mx = 0;
      for (int w = 0; w < FUSED_WARPS; ++w) mx = max(mx, s_max[w]);
      *a.max_vio = a.P > 0 ? __dsub_rn(__ddiv_rn(__dmul_rn((double)mx, (double)E), (double)a.P), 1.0) : 0.0;
    }
    plan_block(s_loads, a.R, a.SK, E, a.plan, a.L, s_run, a.dev_status);
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      st_release_u32(a.sync + 1, 1u);
    }
  }
  if (a.sorted_ids && has_tile) {
    const int bm = a.block_m;
    for (int e = tid; e < E; e += FUSED_THREADS) s_off[e] = (s_loads[e] + bm - 1) / bm * bm;
    __syncthreads();
    const int32_t total = block_scan_inplace(s_off, E, warp_sums);
    if (tid == 0) s_off[E] = total;
    __syncthreads();
    // the pairs' own ids go out in the layout walk below (same stable rank);
    // here only what needs no rank: the padding, the block experts, the total
    int32_t* sorted_ids = a.sorted_ids;
    const int32_t sentinel = (int32_t)a.P;
    for (int e = t; e < E; e += NT)
      for (int32_t i = s_off[e] + s_loads[e] + tid; i < s_off[e + 1]; i += FUSED_THREADS) sorted_ids[i] = sentinel;
    const int64_t gt = (int64_t)t * FUSED_THREADS + tid, gs = (int64_t)NT * FUSED_THREADS;
    for (int64_t i = total + gt; i < a.sorted_cap; i += gs) sorted_ids[i] = sentinel;
    const int64_t nblocks = total / bm;
    for (int64_t b = gt; b < a.expert_ids_cap; b += gs) {
      int32_t owner = -1;
      if (b < nblocks) {
        const int32_t v = (int32_t)(b * bm);
        int lo = 0, hi = E - 1;  // last expert whose group starts at or before v
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (s_off[mid] <= v)
            lo = mid;
          else
            hi = mid - 1;
        }
        owner = lo;
      }
      a.expert_ids[b] = owner;
    }
    if (t == 0 && tid == 0) *a.ntpp = total;  // tile 0 always exists when P > 0
    __syncthreads();
  }
  if (a.stage && has_tile) {
    // where each expert's run starts in the stage: an exclusive scan of the
    // tile counts, less the tile prefix (so a pair of rank g sits at s_tb[e] + g)
    for (int e = tid; e < E; e += FUSED_THREADS) s_tb[e] = s_tc[e];
    if (tid == 0) s_nlong = 0;
    __syncthreads();
    block_scan_inplace(s_tb, E, warp_sums);
    for (int e = tid; e < E; e += FUSED_THREADS) {
      s_tb[e] -= s_excl[e];
      if (s_tc[e] > SWEEP_RUN) s_long[atomicAdd(&s_nlong, 1)] = e;  // list order is free: writes are disjoint
    }
  }

  // ---- 4. layout ranks once the plan is out
  if (!has_tile) return;
  wait_at_least(a.sync + 1, 1u, a.dev_status);
  const EpPlanLayout& L = a.L;
  const int n_rep = min(max(__ldcg(a.plan + L.n_rep), 0), cap);
  for (int e = tid; e < E; e += FUSED_THREADS) {
    s_hc[e] = __ldcg(a.plan + L.home_count + e);
    s_hb[e] = __ldcg(a.plan + L.home_base + e);
    s_cf[e] = __ldcg(a.plan + L.copy_first + e);
    s_cc[e] = __ldcg(a.plan + L.copy_cnt + e);
  }
  for (int m = tid; m < n_rep; m += FUSED_THREADS) {
    s_rb[m] = __ldcg(a.plan + L.rep_begin + m);
    s_rc[m] = __ldcg(a.plan + L.rep_count + m);
    s_rbase[m] = __ldcg(a.plan + L.rep_base + m);
  }
  for (int i = tid; i < FUSED_WARPS * E; i += FUSED_THREADS) s_run[i] = s_wb[i] + s_excl[i % E];
  __syncthreads();
  int32_t* pos = a.pos;
  int32_t* src = a.src;
  int32_t* pair_slot = a.pair_slot;
  int32_t* sorted_ids = a.sorted_ids;
  const int64_t P = a.P;
  const RowMap rm{s_hc, s_hb, s_cf, s_cc, s_rb, s_rc, s_rbase, n_rep, E};
  const bool stage = a.stage != 0;
  const int32_t p0_32 = (int32_t)p0;  // P < 2^31
  walk_warp(a.topk, P, E, wp0, sub, s_run + warp * E,
            [&](int64_t p, int e, int32_t g) {
              if (stage) {  // sorted id and src: the sweep below (q < tile by the count pass; checked)
                const int32_t q = s_tb[e] + g;
                if ((uint32_t)q < (uint32_t)a.tile) s_stage[q] = (uint16_t)((int32_t)p - p0_32);
              } else if (sorted_ids)
                sorted_ids[s_off[e] + g] = (int32_t)p;  // align-sort: same rank within the expert
              int32_t slot;
              const int32_t row = rm.row(e, g, &slot);
              if (row < 0 || row >= P) {
                s_badrow = 1;
                pos[p] = -1;
                if (pair_slot) pair_slot[p] = -1;
                return;
              }
              pos[p] = row;
              if (!stage) src[row] = (int32_t)p;
              if (pair_slot) pair_slot[p] = slot;
            },
            &s_bad);
  // pairs with an invalid id: pos = -1 (their rank walk skipped them)
  __syncthreads();
  if (s_bad) {
    for (int64_t p = wp0 + lane, c = 0; c < sub; c += 32, p += 32) {
      if (p >= P) break;
      const int e = __ldg(a.topk + p);
      if (e < 0 || e >= E) {
        pos[p] = -1;
        if (pair_slot) pair_slot[p] = -1;
      }
    }
  }
  if (stage) {
    // the staged sweep: each expert's run of this tile holds consecutive
    // ranks, so its align-sort ids and (within one copy) its src rows are
    // consecutive words; a warp writes its own experts' runs up to SWEEP_RUN
    // entries, then all warps write the rest of the longer runs
    auto put = [&](int e, int32_t i, int32_t qbase, int32_t g0, int32_t so) {
      const int32_t p = p0_32 + (int32_t)s_stage[qbase + i];
      const int32_t g = g0 + i;
      if (sorted_ids) sorted_ids[so + g] = p;
      int32_t slot;
      const int32_t row = rm.row(e, g, &slot);
      if (row >= 0 && row < P) src[row] = p;
    };
    for (int e = warp; e < E; e += FUSED_WARPS) {
      const int32_t n = min(s_tc[e], SWEEP_RUN);
      const int32_t g0 = s_excl[e], qbase = s_tb[e] + g0, so = sorted_ids ? s_off[e] : 0;
      for (int32_t i = lane; i < n; i += 32) put(e, i, qbase, g0, so);
    }
    const int nlong = s_nlong;
    for (int j = 0; j < nlong; ++j) {
      const int e = s_long[j];
      const int32_t n = s_tc[e];
      const int32_t g0 = s_excl[e], qbase = s_tb[e] + g0, so = sorted_ids ? s_off[e] : 0;
      for (int32_t i = SWEEP_RUN + tid; i < n; i += FUSED_THREADS) put(e, i, qbase, g0, so);
    }
  }
  if (tid == 0) {
    if (s_bad) flag(a.dev_status, EP_DEV_BAD_EXPERT_ID);
    if (s_badrow) flag(a.dev_status, EP_DEV_BAD_ROW);
  }
  if constexpr (DISPATCH) {
    __syncthreads();  // every pos of this tile is written (the walk and the fix-up above)
    route_copy_rows(a, p0, min(p0 + (int64_t)tile, P), reinterpret_cast<uint8_t*>(sm) + a.copy_off);
  }
}

// stage_tile > 0: with the staged sweep's tables and a tile of that many pairs
size_t fused_smem_bytes(int E, int R, int64_t stage_tile = 0) {
  const int cap = E + R - 1;
  size_t words = (size_t)FUSED_WARPS * E + std::max(FUSED_WARPS * E, plan_work_words(E, R)) + 3 * (size_t)E +
                 1 + 4 * (size_t)E + 3 * (size_t)cap;
  if (stage_tile > 0) words += 3 * (size_t)E + ((size_t)stage_tile + 1) / 2;
  return words * sizeof(int32_t);
}

}  // namespace ep

using namespace ep;

namespace ep {

// Rows in flight for the fused copy, as the dispatch kernel sizes them: about
// 32 KB of row loads per SM (4 stages per warp for rows up to 1 KB, else 2),
// split over the CTAs of an SM.
struct CopyShape {
  int warps = 0, stages = 0;
  size_t bytes = 0;
};

static CopyShape copy_shape(uint32_t row_bytes, int K, int per_sm) {
  const uint32_t stride_b = (row_bytes + 127u) & ~127u;
  const uint32_t target = 32u * 1024u;
  const int stages = stride_b * 2u * 16u <= target ? 4 : 2;
  const int ctas = (int)std::min<uint32_t>(32, std::max<uint32_t>(1, (target + stages * stride_b - 1) / (stages * stride_b)));
  const int rows_cta = std::max(1, stages * ctas / std::max(1, per_sm));
  CopyShape c;
  c.stages = std::min(stages, rows_cta);
  c.warps = std::min(FUSED_WARPS, std::max(1, rows_cta / c.stages));
  c.bytes = (size_t)c.warps * c.stages * (stride_b + 8 + 4 * (size_t)K);
  return c;
}

// Smallest tile that stages its pairs.  Measured on B200 with the L2 flushed
// before each route (as in a step, where dispatch and combine stream far more
// than the L2 between routes): tiles of 14,336 pairs (4.2M pairs, E = 384)
// 104.4 -> 90.1 us per route; tiles of 7,168 (2.1M pairs, E = 256) 53.4 ->
// 57.2 us and of 3,584 (1M pairs) 34.8 -> 43.1 us, the sweep costing more
// than the scattered stores it replaces.
constexpr int64_t STAGE_MIN_TILE = 12288;

// ep_route_fused, and with x != nullptr the dispatch of x into buf in the
// same launch (ep_route_dispatch_fused).
static int route_fused(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, int32_t* loads,
                       double* max_vio, int32_t* plan, size_t plan_words, int32_t* pos, int32_t* src,
                       int32_t* pair_slot, int block_m, int32_t* sorted_token_ids, int64_t sorted_cap,
                       int32_t* expert_ids, int64_t expert_ids_cap, int32_t* num_tokens_post_pad,
                       const uint16_t* x, int64_t H, uint16_t* buf, int64_t buf_rows, void* ws, size_t ws_bytes,
                       int32_t* dev_status, cudaStream_t stream) {
  if (!valid_tke(T, K, E) || R < 1 || R > EP_MAX_RANKS || E % R || S < 0 || (int64_t)R * S != T) return EP_ERR_ARG;
  if (!loads || !max_vio || !plan || !ws) return EP_ERR_ARG;
  const int64_t P = T * K;
  if (P > 0 && (!topk_ids || !pos || !src)) return EP_ERR_ARG;
  const bool align = sorted_token_ids != nullptr;
  if (align) {
    if (!expert_ids || !num_tokens_post_pad || block_m < 1 || block_m > (1 << 16)) return EP_ERR_ARG;
    const int64_t need = P + (int64_t)E * (block_m - 1);
    if (need >= ((int64_t)1 << 31)) return EP_ERR_ARG;
    if (sorted_cap < need || expert_ids_cap < (sorted_cap + block_m - 1) / block_m) return EP_ERR_CAPACITY;
  }
  const bool dispatch = x != nullptr;
  if (dispatch) {  // as ep_dispatch (its fallback must accept the same rows)
    if (!dispatch_shape_ok(H, K) || buf_rows < 0) return EP_ERR_ARG;
    if (T > 0 && (!buf || !aligned16(x) || !aligned16(buf))) return EP_ERR_ARG;
  }
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  const WsLayout wl = ws_layout(P, E);
  if (ws_bytes < wl.bytes) return EP_ERR_CAPACITY;

  // grid: one or two resident CTAs per SM, tiles a multiple of 512 pairs; the
  // fused copy adds its row stages to each CTA's shared memory
  const void* fn = dispatch ? (const void*)k_route_fused<true> : (const void*)k_route_fused<false>;
  const uint32_t row_bytes = dispatch ? (uint32_t)(H * 2) : 0u;
  const size_t route_smem = (fused_smem_bytes(E, R) + 127) & ~(size_t)127;
  auto smem_for = [&](int ps) { return route_smem + (dispatch ? copy_shape(row_bytes, K, ps).bytes : 0); };
  auto resident_ok = [&](int ps, size_t smem) {
    if (smem > 227 * 1024) return false;
    if (smem > 48 * 1024 &&
        !raise_smem_limit(fn, smem))
      return false;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, FUSED_THREADS, smem) != cudaSuccess) return false;
    return occ >= ps;
  };
  int per_sm = 0;
  if (P > 0) {
    if (resident_ok(2, smem_for(2)))
      per_sm = 2;
    else if (resident_ok(1, smem_for(1)))
      per_sm = 1;
  }
  // One CTA per SM while that keeps tiles at 2048 pairs or fewer: the planner
  // CTA then has an SM to itself (measured on B200 at 196,608 pairs: kernel span
  // 17.9 -> 15.9 us); larger problems keep two per SM (one per SM measured
  // slower there: the longer tile walks outweigh the faster plan).
  if (per_sm == 2 && num_sms() > 1) {
    const int64_t t1 = ((P + num_sms() - 2) / (num_sms() - 1) + 511) / 512 * 512;
    if (t1 <= 2048 && resident_ok(1, smem_for(1))) per_sm = 1;
  }
  size_t smem = per_sm ? smem_for(per_sm) : 0;
  const int64_t resident = (int64_t)num_sms() * per_sm;
  int64_t tile = 0, ntiles = 0;
  if (resident > 1) {  // one CTA per tile plus the planner CTA
    tile = (P + resident - 2) / (resident - 1);
    tile = std::max<int64_t>(512, (tile + 511) / 512 * 512);
    ntiles = (P + tile - 1) / tile;
  }
  // Large tiles stage their pairs in shared memory (16-bit offsets) when that
  // still leaves the grid resident: the walk's scattered 4-byte stores of src
  // and the align-sort ids become runs of consecutive words.
  bool stage = false;
  if (!dispatch && per_sm > 0 && tile >= STAGE_MIN_TILE && tile <= 65536) {
    const size_t ss = (fused_smem_bytes(E, R, tile) + 127) & ~(size_t)127;
    if (resident_ok(per_sm, ss)) {
      stage = true;
      smem = ss;
    }
  }
  // the [E][tiles] counts must fit below T_e (the separate path's regions are unused here)
  const bool fits = resident > 1 && ntiles + 1 <= resident && tile <= (1 << 20) &&
                    (size_t)E * ntiles * 4 <= wl.loads_off;
  if (!fits) {
    int rc = fused_route_separate(topk_ids, T, K, E, R, S, loads, max_vio, plan, plan_words, pos, src, pair_slot,
                                  block_m, sorted_token_ids, sorted_cap, expert_ids, expert_ids_cap,
                                  num_tokens_post_pad, ws, ws_bytes, dev_status, stream);
    if (rc == EP_OK && dispatch) rc = ep_dispatch(x, T, K, H, pos, buf, buf_rows, dev_status, stream);
    return rc;
  }
  // workspace: counts [E][tiles] from byte 0; T_e [E] where ep_align_sort
  // keeps its histogram, then the two sync words (in the slack after it);
  // one memset zeroes T_e and the sync words
  char* w = static_cast<char*>(ws);
  const size_t tot_bytes = ((size_t)E * 4 + 15) & ~(size_t)15;
  if (cudaMemsetAsync(w + wl.loads_off, 0, tot_bytes + 16, stream) != cudaSuccess) return EP_ERR_CUDA;
  FusedArgs args = {};
  args.topk = topk_ids;
  args.P = P;
  args.E = E;
  args.R = R;
  args.SK = (int32_t)(S * K);
  args.tile = (int)tile;
  args.ntiles = (int)ntiles;
  args.sync = reinterpret_cast<uint32_t*>(w + wl.loads_off + tot_bytes);
  args.counts = reinterpret_cast<int32_t*>(w);
  args.tot = reinterpret_cast<int32_t*>(w + wl.loads_off);
  args.loads = loads;
  args.max_vio = max_vio;
  args.plan = plan;
  args.L = L;
  args.pos = pos;
  args.src = src;
  args.pair_slot = pair_slot;
  args.block_m = block_m;
  args.sorted_ids = align ? sorted_token_ids : nullptr;
  args.sorted_cap = sorted_cap;
  args.expert_ids = expert_ids;
  args.expert_ids_cap = expert_ids_cap;
  args.ntpp = num_tokens_post_pad;
  args.dev_status = dev_status;
  args.stage = stage ? 1 : 0;
  if (dispatch) {
    const CopyShape c = copy_shape(row_bytes, K, per_sm);
    args.x = reinterpret_cast<const uint8_t*>(x);
    args.buf = reinterpret_cast<uint8_t*>(buf);
    args.buf_rows = buf_rows;
    args.row_bytes = row_bytes;
    args.K = K;
    args.copy_warps = c.warps;
    args.copy_stages = c.stages;
    args.copy_off = (uint32_t)route_smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ntiles + 1);
  cfg.blockDim = dim3(FUSED_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t err = dispatch ? cudaLaunchKernelEx(&cfg, k_route_fused<true>, args)
                                   : cudaLaunchKernelEx(&cfg, k_route_fused<false>, args);
  if (err != cudaSuccess) return EP_ERR_CUDA;
  count_launch();
  return launch_status();
}

}  // namespace ep

extern "C" int ep_route_fused(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, int32_t* loads,
                              double* max_vio, int32_t* plan, size_t plan_words, int32_t* pos, int32_t* src,
                              int32_t* pair_slot, int block_m, int32_t* sorted_token_ids, int64_t sorted_cap,
                              int32_t* expert_ids, int64_t expert_ids_cap, int32_t* num_tokens_post_pad, void* ws,
                              size_t ws_bytes, int32_t* dev_status, cudaStream_t stream) {
  return route_fused(topk_ids, T, K, E, R, S, loads, max_vio, plan, plan_words, pos, src, pair_slot, block_m,
                     sorted_token_ids, sorted_cap, expert_ids, expert_ids_cap, num_tokens_post_pad, nullptr, 0,
                     nullptr, 0, ws, ws_bytes, dev_status, stream);
}

extern "C" int ep_route_dispatch_fused(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S,
                                       int32_t* loads, double* max_vio, int32_t* plan, size_t plan_words,
                                       int32_t* pos, int32_t* src, int32_t* pair_slot, int block_m,
                                       int32_t* sorted_token_ids, int64_t sorted_cap, int32_t* expert_ids,
                                       int64_t expert_ids_cap, int32_t* num_tokens_post_pad, const uint16_t* x,
                                       int64_t H, uint16_t* buf, int64_t buf_rows, void* ws, size_t ws_bytes,
                                       int32_t* dev_status, cudaStream_t stream) {
  if (!x && T > 0) return EP_ERR_ARG;  // (T = 0: nothing to copy, x may be NULL)
  return route_fused(topk_ids, T, K, E, R, S, loads, max_vio, plan, plan_words, pos, src, pair_slot, block_m,
                     sorted_token_ids, sorted_cap, expert_ids, expert_ids_cap, num_tokens_post_pad, x, H, buf,
                     buf_rows, ws, ws_bytes, dev_status, stream);
}

namespace ep {

// Same outputs through the separate entry points (when the cooperative grid
// cannot be resident, or P == 0).
int fused_route_separate(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, int32_t* loads,
                         double* max_vio, int32_t* plan, size_t plan_words, int32_t* pos, int32_t* src,
                         int32_t* pair_slot, int block_m, int32_t* sorted_ids, int64_t sorted_cap,
                         int32_t* expert_ids, int64_t expert_ids_cap, int32_t* ntpp, void* ws, size_t ws_bytes,
                         int32_t* dev_status, cudaStream_t stream) {
  int rc = ep_route_stats(topk_ids, T, K, E, loads, max_vio, ws, ws_bytes, dev_status, stream);
  if (rc == EP_OK) rc = ep_plan(loads, R, S, K, E, plan, plan_words, dev_status, stream);
  if (rc == EP_OK)
    rc = ep_layout(topk_ids, T, K, E, R, S, plan, plan_words, ws, ws_bytes, pos, src, pair_slot, dev_status, stream);
  if (rc == EP_OK && sorted_ids)
    rc = ep_align_sort(topk_ids, T, K, E, block_m, sorted_ids, sorted_cap, expert_ids, expert_ids_cap, ntpp, ws,
                       ws_bytes, dev_status, stream);
  return rc;
}

}  // namespace ep
