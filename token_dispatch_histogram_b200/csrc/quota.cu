// Quota-driven replica planning with a per-rank replica budget B.
//
// [JA] "その仕組みは高速なエキスパート複製に依存する" (remio.ai UltraEP
// article): planning starts from the exact load matrix after routing, searches
// for a load threshold every rank can stay under within the replica slots, and
// gives each expert instance a quota; pairs use a local instance first and the
// rest is placed by lookup on cumulative quotas, all on the GPU.  The rule (a
// reading; the page prints none) is stated with ep_quota_route in ep.h.
//
// Four launches, integer work only:
//  1. k_q_count: per-tile expert histogram over RANK-ALIGNED tiles (a tile
//     never straddles two source ranks), so the load matrix L[s][e] and each
//     pair's rank among the pairs of (source rank, expert) come out of one
//     column scan.
//  2. k_q_scan: one warp per expert scans its column of tile counts into
//     exclusive per-tile prefixes (row ntiles holds T_e).  The last CTA to
//     finish computes the rank loads H_r, each rank's experts heaviest first,
//     and the threshold range [ceil(P/R), max(ceil(P/R), max H_r)].
//  3. k_q_search: every thread of the grid tests one threshold at a time, the
//     smallest candidates first; a feasible one is folded into an atomicMin, so
//     the result is the smallest feasible threshold whatever the order.  A
//     test is the sequential chunk/room walk, O(chunks + R), on shared-memory
//     copies of H, T and the order.  The last CTA to finish builds the plan at
//     tau*: one thread repeats the walk and emits the replicas, the CTA then
//     fills quotas, locality counts, rows, slots and cu_seqlens in parallel.
//  4. k_q_layout: the stable-rank walk of the layout pass (tile_ranks.cuh);
//     each pair goes to the instance of its expert on its own source rank while
//     that instance's local share lasts, else to the instance whose cumulative
//     looked-up range holds its rank among the non-local pairs of the expert.
#include <algorithm>

#include "tile_ranks.cuh"

namespace ep {

int num_sms();

constexpr int Q_SCAN_THREADS = 256;
constexpr int Q_SEARCH_THREADS = 256;

// header words of the quota workspace
enum : int { QH_TICKET_SCAN = 0, QH_TICKET_SEARCH = 1, QH_BEST = 2, QH_TAU_LO = 3, QH_TAU_HI = 4, QH_VALID = 5 };

struct QTiles {
  int tile;       // pairs per tile, a multiple of 512
  int tpr;        // tiles per source rank
  int64_t ntiles; // R * tpr
};

// Largest tile of 8192 .. 512 pairs that still gives two tiles per SM.
inline QTiles q_tiles(int64_t SK, int R) {
  QTiles q;
  const int64_t want = 2 * (int64_t)num_sms();
  q.tile = 512;
  for (int sz = 8192; sz >= 512; sz >>= 1) {
    if ((int64_t)R * ((SK + sz - 1) / sz) >= want) {
      q.tile = sz;
      break;
    }
  }
  q.tpr = SK > 0 ? (int)((SK + q.tile - 1) / q.tile) : 0;
  q.ntiles = (int64_t)R * q.tpr;
  return q;
}

struct QWs {
  size_t hdr, cnt, excl, H, ord, bytes;
};
inline QWs q_ws(int64_t ntiles, int E, int R) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  QWs w;
  w.hdr = 0;
  w.cnt = 256;
  w.excl = al(w.cnt + sizeof(int32_t) * (size_t)E * (size_t)std::max<int64_t>(ntiles, 1));
  w.H = al(w.excl + sizeof(int32_t) * (size_t)E * (size_t)(ntiles + 1));
  w.ord = al(w.H + sizeof(int32_t) * (size_t)R);
  w.bytes = al(w.ord + sizeof(int32_t) * (size_t)E);
  return w;
}

void quota_layout(int E, int R, EpQuotaLayout* L) {
  const int cap = E + R - 1;
  int32_t o = 0;
  auto take = [&](int32_t n) {
    const int32_t at = o;
    o += (n + 7) & ~7;
    return at;
  };
  L->cap = cap;
  L->tau = take(1);
  L->n_rep = take(1);
  L->n_local = take(1);
  L->rank_load = take(R);
  L->rank_off = take(R);
  L->rank_nrep = take(R);
  L->rank_rep_first = take(R);
  L->home_quota = take(E);
  L->rep_first = take(E);
  L->rep_cnt = take(E);
  L->rep_expert = take(cap);
  L->rep_rank = take(cap);
  L->rep_count = take(cap);
  L->inst_local = take(E + cap);
  L->inst_cum = take(E + cap);
  L->inst_base = take(E + cap);
  L->inst_lpre = take(E + cap);
  L->slot_order = take(E + cap);
  L->cu_seqlens = take(E + cap + 1);
  L->words = o;
}

// ------------------------------------------------------------------ 1. count

__global__ void __launch_bounds__(SCAT_THREADS)
    k_q_count(const int32_t* __restrict__ topk, int64_t SK, int E, int tile, int tpr, int64_t ntiles,
              int32_t* __restrict__ cnt, uint32_t* __restrict__ hdr, int32_t* dev_status) {
  extern __shared__ int32_t s_hist[];  // [E]
  __shared__ int s_bad;
  const int64_t t = blockIdx.x;
  if (t == 0 && threadIdx.x == 0) {
    hdr[QH_TICKET_SCAN] = 0;
    hdr[QH_TICKET_SEARCH] = 0;
  }
  if (t >= ntiles) return;
  if (threadIdx.x == 0) s_bad = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int64_t r = t / tpr, lt = t % tpr;
  const int64_t p0 = r * SK + lt * tile;
  const int n = (int)min((int64_t)tile, SK - lt * tile);
  const int lane = threadIdx.x & 31;
  const int nbits = key_bits(E + 1);
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < n) {
      e = __ldg(topk + p0 + i);
      if (e < 0 || e >= E) {
        e = -1;
        s_bad = 1;
      }
    }
    const uint32_t peers = warp_match((uint32_t)(e + 1), nbits);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&s_hist[e], __popc(peers));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[(int64_t)e * ntiles + t] = s_hist[e];
  if (threadIdx.x == 0 && s_bad) flag(dev_status, EP_DEV_BAD_EXPERT_ID);
}

// ------------------------------------------------------------------- 2. scan

__global__ void __launch_bounds__(Q_SCAN_THREADS)
    k_q_scan(const int32_t* __restrict__ cnt, int64_t ntiles, int E, int R, int64_t P, int32_t* __restrict__ excl,
             int32_t* __restrict__ loads, int32_t* __restrict__ H_out, int32_t* __restrict__ ord,
             uint32_t* __restrict__ hdr) {
  extern __shared__ int32_t sm[];
  int32_t* s_T = sm;      // [E]
  int32_t* s_H = sm + E;  // [R]
  __shared__ int s_last;
  __shared__ unsigned long long s_total;
  __shared__ int s_maxH;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e = blockIdx.x * (Q_SCAN_THREADS / 32) + warp;
  if (e < E) {
    int32_t run = 0;
    for (int64_t b = 0; b < ntiles; b += 32) {
      const int64_t t = b + lane;
      const int32_t v = t < ntiles ? cnt[(int64_t)e * ntiles + t] : 0;
      int32_t x = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
      }
      if (t < ntiles) excl[t * E + e] = run + x - v;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) {
      excl[ntiles * E + e] = run;
      loads[e] = run;
    }
  }
  // the last CTA to finish prepares the threshold search
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&hdr[QH_TICKET_SCAN], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x == 0) {
    s_total = 0;
    s_maxH = 0;
  }
  for (int r = threadIdx.x; r < R; r += blockDim.x) s_H[r] = 0;
  __syncthreads();
  const int ER = E / R;
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    const int32_t v = __ldcg(loads + x);
    s_T[x] = v;
    atomicAdd(&s_total, (unsigned long long)v);
    atomicAdd(&s_H[x / ER], v);
  }
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    H_out[r] = s_H[r];
    atomicMax(&s_maxH, s_H[r]);
  }
  // each rank's experts heaviest first, ties to the lower id
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    const int r = x / ER;
    const int32_t v = s_T[x];
    int k = 0;
    for (int y = r * ER; y < (r + 1) * ER; ++y) {
      const int32_t w = s_T[y];
      k += (w > v) || (w == v && y < x);
    }
    ord[r * ER + k] = x;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int64_t lo = (P + R - 1) / R;
    const int64_t hi = (int64_t)s_maxH > lo ? (int64_t)s_maxH : lo;
    hdr[QH_TAU_LO] = (uint32_t)lo;
    hdr[QH_TAU_HI] = (uint32_t)hi;
    hdr[QH_BEST] = (uint32_t)hi;
    hdr[QH_VALID] = s_total == (unsigned long long)P;
    hdr[QH_TICKET_SCAN] = 0;
  }
}

// --------------------------------------------------------- 3. search + build

// Whether every chunk finds room at threshold tau (the chunk/room walk).
__device__ bool q_feasible(int64_t tau, const int32_t* s_T, const int32_t* s_H, const int32_t* s_ord, int R, int ER,
                           int B) {
  int j = 0;
  while (j < R && s_H[j] >= tau) ++j;
  int64_t room = j < R ? tau - s_H[j] : 0;
  int pieces = 0;
  for (int r = 0; r < R; ++r) {
    int64_t rem = (int64_t)s_H[r] - tau;
    for (int i = 0; i < ER && rem > 0; ++i) {
      int64_t c = min((int64_t)s_T[s_ord[r * ER + i]], rem);
      if (c <= 0) break;
      rem -= c;
      while (c > 0) {
        if (j >= R || B <= 0) return false;
        const int64_t take = min(c, room);
        c -= take;
        room -= take;
        if (++pieces == B || room == 0) {
          ++j;
          while (j < R && s_H[j] >= tau) ++j;
          room = j < R ? tau - s_H[j] : 0;
          pieces = 0;
        }
      }
    }
  }
  return true;
}

__global__ void __launch_bounds__(Q_SEARCH_THREADS)
    k_q_search(const int32_t* __restrict__ loads, const int32_t* __restrict__ H_in, const int32_t* __restrict__ ord,
               const int32_t* __restrict__ excl, int tpr, int E, int R, int B, int64_t P, uint32_t* hdr,
               int32_t* __restrict__ plan, EpQuotaLayout L) {
  extern __shared__ int32_t sm[];
  int32_t* s_T = sm;            // [E]
  int32_t* s_ord = s_T + E;     // [E]
  int32_t* s_rfirst = s_ord + E;  // [E] (build)
  int32_t* s_rcnt = s_rfirst + E;  // [E] (build)
  int32_t* s_hq = s_rcnt + E;   // [E] (build)
  int32_t* s_H = s_hq + E;      // [R]
  int32_t* s_rnrep = s_H + R;   // [R] (build)
  int32_t* s_rrf = s_rnrep + R;  // [R] (build)
  int32_t* s_rl = s_rrf + R;    // [R] (build)
  __shared__ int s_last, s_nrep;
  __shared__ int32_t warp_sums[32];
  __shared__ unsigned long long s_local;
  const int ER = E / R;
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    s_T[x] = loads[x];
    s_ord[x] = ord[x];
  }
  for (int r = threadIdx.x; r < R; r += blockDim.x) s_H[r] = H_in[r];
  __syncthreads();
  const int64_t lo = hdr[QH_TAU_LO], hi = hdr[QH_TAU_HI];
  const bool valid = hdr[QH_VALID] != 0;
  if (valid) {
    const int64_t N = (int64_t)gridDim.x * blockDim.x;
    volatile uint32_t* best = hdr + QH_BEST;
    for (int64_t tau = lo + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; tau < hi; tau += N) {
      if (tau >= (int64_t)*best) break;
      if (q_feasible(tau, s_T, s_H, s_ord, R, ER, B)) {
        atomicMin(hdr + QH_BEST, (uint32_t)tau);
        break;
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&hdr[QH_TICKET_SEARCH], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- the plan at tau*, by the last CTA
  const int cap = L.cap;
  const int64_t tau = valid ? (int64_t)atomicAdd(hdr + QH_BEST, 0u) : -1;
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    s_rfirst[x] = 0;
    s_rcnt[x] = 0;
  }
  for (int r = threadIdx.x; r < R; r += blockDim.x) s_rnrep[r] = 0;
  if (threadIdx.x == 0) {
    s_nrep = 0;
    s_local = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0 && valid) {  // the walk at tau*, emitting one replica per piece
    int n = 0, j = 0, pieces = 0;
    while (j < R && s_H[j] >= tau) ++j;
    int64_t room = j < R ? tau - s_H[j] : 0;
    for (int r = 0; r < R; ++r) {
      int64_t rem = (int64_t)s_H[r] - tau;
      for (int i = 0; i < ER && rem > 0; ++i) {
        const int e = s_ord[r * ER + i];
        int64_t c = min((int64_t)s_T[e], rem);
        if (c <= 0) break;
        rem -= c;
        s_rfirst[e] = n;
        while (c > 0 && j < R && B > 0 && n < cap) {
          const int64_t take = min(c, room);
          plan[L.rep_expert + n] = e;
          plan[L.rep_rank + n] = j;
          plan[L.rep_count + n] = (int32_t)take;
          ++n;
          s_rcnt[e] += 1;
          s_rnrep[j] += 1;
          c -= take;
          room -= take;
          if (++pieces == B || room == 0) {
            ++j;
            while (j < R && s_H[j] >= tau) ++j;
            room = j < R ? tau - s_H[j] : 0;
            pieces = 0;
          }
        }
      }
    }
    s_nrep = n;
  }
  __syncthreads();
  const int n_rep = s_nrep;
  for (int m = n_rep + threadIdx.x; m < cap; m += blockDim.x) {
    plan[L.rep_expert + m] = -1;
    plan[L.rep_rank + m] = -1;
    plan[L.rep_count + m] = 0;
  }
  // home quotas, replica ranges per expert
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int32_t q = valid ? s_T[x] : 0;
    for (int k = 0; k < s_rcnt[x]; ++k) q -= plan[L.rep_count + s_rfirst[x] + k];
    s_hq[x] = q;
    plan[L.home_quota + x] = q;
    plan[L.rep_first + x] = s_rfirst[x];
    plan[L.rep_cnt + x] = s_rcnt[x];
  }
  for (int r = threadIdx.x; r < R; r += blockDim.x) s_rrf[r] = s_rnrep[r];
  __syncthreads();
  block_scan_array(s_rrf, R, warp_sums);  // replicas received by lower ranks
  // rank loads
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    int32_t l = 0;
    for (int x = r * ER; x < (r + 1) * ER; ++x) l += s_hq[x];
    for (int k = 0; k < s_rnrep[r]; ++k) l += plan[L.rep_count + s_rrf[r] + k];
    s_rl[r] = l;
    plan[L.rank_load + r] = l;
    plan[L.rank_nrep + r] = s_rnrep[r];
    plan[L.rank_rep_first + r] = s_rrf[r];
  }
  __syncthreads();
  block_scan_array(s_rl, R, warp_sums);  // now the first row of each rank
  // rows of every instance, rank by rank: home experts by id, then replicas
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    int32_t row = s_rl[r];
    plan[L.rank_off + r] = row;
    for (int x = r * ER; x < (r + 1) * ER; ++x) {
      plan[L.inst_base + x] = row;
      const int slot = x + s_rrf[r];
      plan[L.slot_order + slot] = x;
      row += s_hq[x];
      plan[L.cu_seqlens + slot + 1] = row;
    }
    for (int k = 0; k < s_rnrep[r]; ++k) {
      const int m = s_rrf[r] + k;
      plan[L.inst_base + E + m] = row;
      const int slot = (r + 1) * ER + m;
      plan[L.slot_order + slot] = E + m;
      row += plan[L.rep_count + m];
      plan[L.cu_seqlens + slot + 1] = row;
    }
  }
  for (int slot = E + n_rep + threadIdx.x; slot < E + cap; slot += blockDim.x) {
    plan[L.slot_order + slot] = -1;
    plan[L.cu_seqlens + slot + 1] = valid ? (int32_t)P : 0;
  }
  if (threadIdx.x == 0) plan[L.cu_seqlens] = 0;
  // locality: instance i on rank r takes the first min(q_i, L[r][e]) pairs of
  // e from source rank r; the rest of e's pairs fill the instances' remaining
  // quotas in instance order (home, then replicas in match order)
  const int64_t Eq = E;
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int32_t cum = 0;
    for (int k = 0; k <= s_rcnt[x]; ++k) {
      const int i = k == 0 ? x : E + s_rfirst[x] + k - 1;
      const int r = k == 0 ? x / ER : plan[L.rep_rank + s_rfirst[x] + k - 1];
      const int32_t q = k == 0 ? s_hq[x] : plan[L.rep_count + s_rfirst[x] + k - 1];
      const int32_t lpre = excl[(int64_t)r * tpr * Eq + x];
      const int32_t lsrc = excl[(int64_t)(r + 1) * tpr * Eq + x] - lpre;
      const int32_t loc = valid ? min(q, lsrc) : 0;
      plan[L.inst_local + i] = loc;
      plan[L.inst_cum + i] = cum;
      plan[L.inst_lpre + i] = lpre;
      cum += q - loc;
      atomicAdd(&s_local, (unsigned long long)loc);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    plan[L.tau] = (int32_t)tau;
    plan[L.n_rep] = n_rep;
    plan[L.n_local] = (int32_t)s_local;
    hdr[QH_TICKET_SEARCH] = 0;
  }
}

// ----------------------------------------------------------------- 4. layout

__global__ void __launch_bounds__(SCAT_THREADS)
    k_q_layout(const int32_t* __restrict__ topk, int64_t SK, int E, int R, int tile, int tpr,
               const int32_t* __restrict__ excl, const int32_t* __restrict__ plan, EpQuotaLayout L,
               int32_t* __restrict__ pos, int32_t* __restrict__ src, int32_t* dev_status) {
  extern __shared__ int32_t sm[];
  int32_t* s_ids = sm;              // [tile]
  int32_t* s_whist = s_ids + tile;  // [SCAT_WARPS * E]
  __shared__ int s_flags;
  const int64_t t = blockIdx.x;
  const int rs = (int)(t / tpr);
  const int64_t lt = t % tpr;
  const int64_t p0 = (int64_t)rs * SK + lt * tile;
  const int n = (int)min((int64_t)tile, SK - lt * tile);
  const int ER = E / R;
  const int64_t P = (int64_t)R * SK;
  const int32_t tau = plan[L.tau];
  if (threadIdx.x == 0) s_flags = 0;
  if (tau < 0) {  // no plan (bad input): nothing is placed
    for (int i = threadIdx.x; i < n; i += blockDim.x) pos[p0 + i] = -1;
    return;
  }
  const int32_t* lpre_src = excl + (int64_t)rs * tpr * E;  // pairs of e from source ranks below rs
  auto emit = [&](int64_t p, int e, int32_t g) {
    const int rf = __ldg(plan + L.rep_first + e), rc = __ldg(plan + L.rep_cnt + e);
    // the instance of e on the pair's own source rank, if any (e's replicas
    // sit on ascending ranks)
    int inst = -1;
    if (e / ER == rs) {
      inst = e;
    } else if (rc > 0) {
      int a = rf, b = rf + rc - 1;
      while (a < b) {
        const int mid = (a + b) >> 1;
        if (__ldg(plan + L.rep_rank + mid) < rs)
          a = mid + 1;
        else
          b = mid;
      }
      if (__ldg(plan + L.rep_rank + a) == rs) inst = E + a;
    }
    const int32_t ls = g - __ldg(lpre_src + e);
    int32_t row = -1;
    if (inst >= 0 && ls < __ldg(plan + L.inst_local + inst)) {
      row = __ldg(plan + L.inst_base + inst) + ls;
    } else {
      // rank among e's pairs that are not placed locally
      int32_t j = g;
      for (int k = 0; k <= rc; ++k) {
        const int i = k == 0 ? e : E + rf + k - 1;
        const int32_t d = g - __ldg(plan + L.inst_lpre + i);
        const int32_t loc = __ldg(plan + L.inst_local + i);
        j -= d <= 0 ? 0 : (d < loc ? d : loc);
      }
      // the last instance whose cumulative start is <= j
      int a = 0, b = rc;
      while (a < b) {
        const int mid = (a + b + 1) >> 1;
        const int i = mid == 0 ? e : E + rf + mid - 1;
        if (__ldg(plan + L.inst_cum + i) <= j)
          a = mid;
        else
          b = mid - 1;
      }
      const int i = a == 0 ? e : E + rf + a - 1;
      const int32_t q = a == 0 ? __ldg(plan + L.home_quota + e) : __ldg(plan + L.rep_count + rf + a - 1);
      const int32_t loc = __ldg(plan + L.inst_local + i);
      const int32_t off = j - __ldg(plan + L.inst_cum + i);
      if (off >= 0 && off < q - loc) row = __ldg(plan + L.inst_base + i) + loc + off;
    }
    if (row < 0 || row >= P) {
      atomicOr(&s_flags, EP_DEV_BAD_ROW);
      pos[p] = -1;
      return;
    }
    pos[p] = row;
    src[row] = (int32_t)p;
  };
  auto bad = [&](int64_t p) {
    atomicOr(&s_flags, EP_DEV_BAD_EXPERT_ID);
    pos[p] = -1;
  };
  tile_stable_ranks(topk, E, tile, p0, n, excl + t * E, s_ids, s_whist, emit, bad);
  __syncthreads();
  if (threadIdx.x == 0 && s_flags) flag(dev_status, s_flags);
}

}  // namespace ep

using namespace ep;

extern "C" int ep_quota_plan_layout(int E, int R, EpQuotaLayout* layout) {
  if (!layout || R < 1 || R > EP_MAX_RANKS || E < 1 || E > EP_MAX_EXPERTS || E % R) return EP_ERR_ARG;
  quota_layout(E, R, layout);
  return EP_OK;
}

extern "C" int ep_quota_workspace_size(int64_t T, int K, int E, int R, size_t* bytes) {
  if (!bytes || !valid_tke(T, K, E) || R < 1 || R > EP_MAX_RANKS || E % R || T % R) return EP_ERR_ARG;
  const QTiles q = q_tiles(T / R * K, R);
  *bytes = q_ws(q.ntiles, E, R).bytes;
  return EP_OK;
}

extern "C" int ep_quota_route(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, int B,
                              int32_t* loads, int32_t* plan, size_t plan_words, int32_t* pos, int32_t* src, void* ws,
                              size_t ws_bytes, int32_t* dev_status, cudaStream_t stream) {
  if (!valid_tke(T, K, E) || R < 1 || R > EP_MAX_RANKS || E % R || S < 0 || (int64_t)R * S != T || B < 0)
    return EP_ERR_ARG;
  if (!loads || !plan || !ws) return EP_ERR_ARG;
  const int64_t P = T * K, SK = S * K;
  if (P > 0 && (!topk_ids || !pos || !src)) return EP_ERR_ARG;
  EpQuotaLayout L;
  quota_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  const QTiles q = q_tiles(SK, R);
  const QWs w = q_ws(q.ntiles, E, R);
  if (ws_bytes < w.bytes) return EP_ERR_CAPACITY;
  char* base = static_cast<char*>(ws);
  uint32_t* hdr = reinterpret_cast<uint32_t*>(base + w.hdr);
  int32_t* cnt = reinterpret_cast<int32_t*>(base + w.cnt);
  int32_t* excl = reinterpret_cast<int32_t*>(base + w.excl);
  int32_t* H = reinterpret_cast<int32_t*>(base + w.H);
  int32_t* ord = reinterpret_cast<int32_t*>(base + w.ord);

  k_q_count<<<(unsigned)std::max<int64_t>(q.ntiles, 1), SCAT_THREADS, sizeof(int32_t) * E, stream>>>(
      topk_ids, SK, E, q.tile, q.tpr, q.ntiles, cnt, hdr, dev_status);
  const int scan_grid = (E + Q_SCAN_THREADS / 32 - 1) / (Q_SCAN_THREADS / 32);
  k_q_scan<<<scan_grid, Q_SCAN_THREADS, sizeof(int32_t) * (E + R), stream>>>(cnt, q.ntiles, E, R, P, excl, loads, H,
                                                                              ord, hdr);
  const size_t search_smem = sizeof(int32_t) * (5 * (size_t)E + 4 * (size_t)R);
  k_q_search<<<2 * num_sms(), Q_SEARCH_THREADS, search_smem, stream>>>(loads, H, ord, excl, q.tpr, E, R, B, P, hdr,
                                                                       plan, L);
  count_launch(3);
  if (q.ntiles > 0) {
    const size_t smem = sizeof(int32_t) * ((size_t)q.tile + (size_t)SCAT_WARPS * E);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(k_q_layout, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return EP_ERR_CUDA;
    k_q_layout<<<(unsigned)q.ntiles, SCAT_THREADS, smem, stream>>>(topk_ids, SK, E, R, q.tile, q.tpr, excl, plan, L,
                                                                   pos, src, dev_status);
    count_launch();
  }
  return launch_status();
}
