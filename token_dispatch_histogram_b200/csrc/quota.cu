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
//  2. k_q_scan: every expert column of tile counts is scanned into
//     exclusive per-tile prefixes (row ntiles holds T_e) by 128 threads, one
//     short tile range each, 8 columns per CTA.
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

#include "grid_sync.cuh"
#include "tile_ranks.cuh"

namespace ep {

int num_sms();

constexpr int Q_SCAN_THREADS = 1024;
constexpr int Q_SEARCH_THREADS = 256;

// header words of the quota workspace
enum : int { QH_TICKET_SEARCH = 0, QH_BEST = 1, QH_BARRIER = 2, QH_FLAG = 3 };

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

// Workspace: header words, T_e (the one-launch route's atomic sums; the
// header and T_e are zeroed together), tile counts [ntiles][E], exclusive
// tile prefixes [ntiles + 1][E].
struct QWs {
  size_t hdr, tot, cnt, excl, bytes;
};
inline QWs q_ws(int64_t ntiles, int E, int R) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  QWs w;
  w.hdr = 0;
  w.tot = 256;
  w.cnt = al(w.tot + sizeof(int32_t) * (size_t)E);
  w.excl = al(w.cnt + sizeof(int32_t) * (size_t)E * (size_t)std::max<int64_t>(ntiles, 1));
  w.bytes = al(w.excl + sizeof(int32_t) * (size_t)E * (size_t)(ntiles + 1));
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
  L->n_chunks = take(1);
  L->rank_load = take(R);
  L->rank_off = take(R);
  L->rank_nrep = take(R);
  L->rank_rep_first = take(R);
  L->home_quota = take(E);
  L->rep_first = take(E);
  L->rep_cnt = take(E);
  L->rep_experts = take(E);
  L->rep_expert = take(cap);
  L->rep_rank = take(cap);
  L->rep_count = take(cap);
  L->inst_local = take(E + cap);
  L->inst_cum = take(E + cap);
  L->inst_base = take(E + cap);
  L->inst_lpre = take(E + cap);
  L->rep_local_incl = take(cap);
  L->slot_order = take(E + cap);
  L->cu_seqlens = take(E + cap + 1);
  L->words = o;
}

// ------------------------------------------------------------------ 1. count

constexpr int Q_ITEMS = 16;  // keys per thread per round: 512 * 16 = 8192 pairs

// Per-expert counts of tile t (rank-aligned): cnt[t*E + e]; with tot != NULL
// also added into tot[e] (integer atomics, so the sums do not depend on
// order).  Counts are order-free, so plain shared-memory adds do.  s_hist: [E].
__device__ void q_count_tile(const int32_t* __restrict__ topk, int64_t SK, int E, int tile, int tpr, int64_t t,
                             int32_t* __restrict__ cnt, int32_t* __restrict__ tot, int32_t* s_hist,
                             int32_t* dev_status) {
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  const int64_t r = t / tpr, lt = t % tpr;
  const int64_t p0 = r * SK + lt * tile;
  const int n = (int)min((int64_t)tile, SK - lt * tile);
  __syncthreads();
  bool bad = false;
  for (int c0 = 0; c0 < n; c0 += Q_ITEMS * SCAT_THREADS) {
    int key[Q_ITEMS];
#pragma unroll
    for (int k = 0; k < Q_ITEMS; ++k) {  // every load issued before the first add
      const int i = c0 + k * SCAT_THREADS + threadIdx.x;
      key[k] = i < n ? __ldg(topk + p0 + i) : 0;
    }
#pragma unroll
    for (int k = 0; k < Q_ITEMS; ++k) {
      const int i = c0 + k * SCAT_THREADS + threadIdx.x;
      if (i < n) {
        const int e = key[k];
        if (e >= 0 && e < E)
          atomicAdd(&s_hist[e], 1);
        else
          bad = true;
      }
    }
  }
  if (bad) s_bad = 1;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t v = s_hist[e];
    cnt[t * E + e] = v;
    if (tot && v) atomicAdd(tot + e, v);
  }
  if (threadIdx.x == 0 && s_bad) flag(dev_status, EP_DEV_BAD_EXPERT_ID);
}

__global__ void __launch_bounds__(SCAT_THREADS)
    k_q_count(const int32_t* __restrict__ topk, int64_t SK, int E, int tile, int tpr, int64_t ntiles,
              int32_t* __restrict__ cnt, uint32_t* __restrict__ hdr, int32_t* dev_status) {
  extern __shared__ int32_t s_hist[];  // [E]
  const int64_t t = blockIdx.x;
  if (t == 0 && threadIdx.x == 0) {
    hdr[QH_TICKET_SEARCH] = 0;
    hdr[QH_BEST] = 0xffffffffu;
  }
  if (t >= ntiles) return;
  q_count_tile(topk, SK, E, tile, tpr, t, cnt, nullptr, s_hist, dev_status);
}

// ------------------------------------------------------------------- 2. scan

constexpr int Q_SCAN_EXPERTS = 8;                              // expert columns per CTA
constexpr int Q_SCAN_GROUPS = Q_SCAN_THREADS / Q_SCAN_EXPERTS;  // tile ranges per column

// Threads = (tile range g, expert j): 8 consecutive experts of one tile are 8
// consecutive words, read by 8 consecutive threads.  Each thread sums its tile
// range; warp j then scans column j's range sums (each lane four consecutive
// ranges, one warp scan); each thread walks its range again writing the
// exclusive prefixes.  Row ntiles of excl and loads get T_e.  Many CTAs with
// one short range each keep the dependent load chains short.
__global__ void __launch_bounds__(Q_SCAN_THREADS)
    k_q_scan(const int32_t* __restrict__ cnt, int64_t ntiles, int E, int32_t* __restrict__ excl,
             int32_t* __restrict__ loads) {
  static_assert(Q_SCAN_GROUPS == 128 && Q_SCAN_EXPERTS <= Q_SCAN_THREADS / 32, "one warp scans 4 ranges per lane");
  __shared__ int32_t s_part[Q_SCAN_GROUPS][Q_SCAN_EXPERTS];
  const int j = threadIdx.x % Q_SCAN_EXPERTS, g = threadIdx.x / Q_SCAN_EXPERTS;
  const int e = blockIdx.x * Q_SCAN_EXPERTS + j;
  const int64_t span = (ntiles + Q_SCAN_GROUPS - 1) / Q_SCAN_GROUPS;
  const int64_t t0 = min(ntiles, g * span), t1 = min(ntiles, t0 + span);
  int32_t sum = 0;
  if (e < E) {
#pragma unroll 4
    for (int64_t t = t0; t < t1; ++t) sum += cnt[t * E + e];
  }
  s_part[g][j] = sum;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp < Q_SCAN_EXPERTS) {  // warp `warp` scans column `warp`: lane owns ranges 4*lane .. 4*lane+3
    int32_t v[4], tot = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[q] = s_part[4 * lane + q][warp];
      tot += v[q];
    }
    int32_t inc = tot;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += y;
    }
    int32_t run = inc - tot;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      s_part[4 * lane + q][warp] = run;
      run += v[q];
    }
    const int ew = blockIdx.x * Q_SCAN_EXPERTS + warp;
    if (lane == 31 && ew < E) {
      excl[ntiles * E + ew] = inc;
      loads[ew] = inc;
    }
  }
  __syncthreads();
  if (e < E) {
    int32_t run = s_part[g][j];
#pragma unroll 4
    for (int64_t t = t0; t < t1; ++t) {
      const int32_t v = cnt[t * E + e];
      excl[t * E + e] = run;
      run += v;
    }
  }
}

// Rank-local form: the gathered load matrix counts [R, E] (row s = source rank
// s's pairs per expert) as the per-rank prefixes the search reads with one
// "tile" per rank: pre[s][e] = sum_{s' < s} counts[s'][e], pre[R][e] = T_e =
// loads[e].  A column with a negative entry or a sum past int32 gets -1, so
// the loads do not add up and the search writes no plan.  Also resets the
// search's ticket and best threshold.
__global__ void __launch_bounds__(256)
    k_q_counts_prefix(const int32_t* __restrict__ counts, int R, int E, int32_t* __restrict__ pre,
                      int32_t* __restrict__ loads, uint32_t* __restrict__ hdr) {
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    hdr[QH_TICKET_SEARCH] = 0;
    hdr[QH_BEST] = 0xffffffffu;
  }
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  int64_t run = 0;
  bool ok = true;
  for (int r = 0; r < R; ++r) {
    const int32_t c = counts[(int64_t)r * E + e];
    pre[(int64_t)r * E + e] = (int32_t)run;
    ok = ok && c >= 0;
    run += c;
    ok = ok && run <= INT32_MAX;
    if (!ok) run = 0;
  }
  const int32_t tot = ok ? (int32_t)run : -1;
  pre[(int64_t)R * E + e] = tot;
  loads[e] = tot;
}

// --------------------------------------------------------- 3. search + build

// Whether every chunk finds room at threshold tau: the chunk/room walk over
// this CTA's lists of possibly overloaded ranks (H and offset of its sorted
// loads) and possible rooms (H), both in ascending rank order.  All values fit
// in 32 bits (they are at most P < 2^31).
__device__ __forceinline__ bool q_feasible(int32_t tau, const int32_t* s_sT, const int32_t* s_oH,
                                           const int32_t* s_oOff, int novr, const int32_t* s_mH, int nroom, int ER,
                                           int B) {
  if (B <= 0) {
    for (int a = 0; a < novr; ++a)
      if (s_oH[a] > tau) return false;
    return true;
  }
  int j = 0;
  while (j < nroom && s_mH[j] >= tau) ++j;
  int32_t room = j < nroom ? tau - s_mH[j] : 0;
  int pieces = 0;
  for (int a = 0; a < novr; ++a) {
    int32_t rem = s_oH[a] - tau;
    const int32_t* st = s_sT + s_oOff[a];
    for (int i = 0; i < ER && rem > 0; ++i) {
      int32_t c = min(st[i], rem);
      if (c <= 0) break;
      rem -= c;
      while (c > 0) {
        if (j >= nroom) return false;
        const int32_t take = min(c, room);
        c -= take;
        room -= take;
        if (++pieces == B || room == 0) {
          ++j;
          while (j < nroom && s_mH[j] >= tau) ++j;
          room = j < nroom ? tau - s_mH[j] : 0;
          pieces = 0;
        }
      }
    }
  }
  return true;
}

inline size_t q_search_smem(int E, int R) {
  const size_t cap = (size_t)E + R - 1;
  return sizeof(int32_t) * (9 * (size_t)E + 12 * (size_t)R + 3 * cap + ((size_t)E + cap));
}

// What a call of q_search_build does: the threshold search (every CTA: its
// own view of the loads, then its candidates), the plan at tau* (one CTA,
// from the view it built in an earlier Q_SEARCH call), or both with a ticket
// between them (the last CTA to finish builds).
enum QPhase : int { Q_SEARCH = 1, Q_BUILD = 2, Q_ALL = 3 };

__device__ void q_search_build(const int32_t* __restrict__ loads, const int32_t* __restrict__ excl, int tpr, int E,
                               int R, int B, int64_t P, uint32_t* hdr, int32_t* __restrict__ plan,
                               const EpQuotaLayout& L, int32_t* sm, int phase) {
  const int cap = L.cap;
  int32_t* s_T = sm;                // [E]
  int32_t* s_sT = s_T + E;          // [E] each rank's loads, heaviest first
  int32_t* s_ord = s_sT + E;        // [E] the matching expert ids
  int32_t* s_rfirst = s_ord + E;    // [E] (build)
  int32_t* s_rcnt = s_rfirst + E;   // [E] (build)
  int32_t* s_hq = s_rcnt + E;       // [E] (build)
  int32_t* s_H = s_hq + E;          // [R]
  int32_t* s_oH = s_H + R;          // [R] possibly overloaded ranks: H
  int32_t* s_oOff = s_oH + R;       // [R]   and r * E/R
  int32_t* s_mH = s_oOff + R;       // [R] possible rooms: H
  int32_t* s_mR = s_mH + R;         // [R]   and rank
  int32_t* s_rnrep = s_mR + R;      // [R] (build)
  int32_t* s_rrf = s_rnrep + R;     // [R] (build)
  int32_t* s_rl = s_rrf + R;        // [R] (build)
  int32_t* s_re = s_rl + R;         // [cap]
  int32_t* s_rr = s_re + cap;       // [cap]
  int32_t* s_rc = s_rr + cap;       // [cap]
  int32_t* s_loc = s_rc + cap;      // [E + cap]
  int32_t* s_chE = s_loc + E + cap; // [E] chunks at tau*: expert
  int32_t* s_chB = s_chE + E;       // [E]   first position in the excess sequence
  int32_t* s_chN = s_chB + E;       // [E]   size
  int32_t* s_wS = s_chN + E;        // [R] room windows at tau*: start
  int32_t* s_wE = s_wS + R;         // [R]   end
  int32_t* s_wR = s_wE + R;         // [R]   rank
  int32_t* s_wP = s_wR + R;         // [R]   first piece
  __shared__ int s_last, s_nrep, s_novr, s_nroom, s_maxH, s_nwin;
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t s_total, s_local;
  const int ER = E / R;
  const int64_t lo = (P + R - 1) / R;
  if (phase & Q_SEARCH) {
    // every CTA derives the rank loads, each rank's order and the range itself
    if (threadIdx.x == 0) {
      s_total = 0;
      s_maxH = 0;
    }
    for (int r = threadIdx.x; r < R; r += blockDim.x) s_H[r] = 0;
    __syncthreads();
    {
      int32_t part = 0;  // loads count valid pairs only, so every sum stays below 2^31
      for (int x = threadIdx.x; x < E; x += blockDim.x) {
        const int32_t v = __ldcg(loads + x);  // (written by atomics in the one-launch route)
        s_T[x] = v;
        part += v;
        atomicAdd(&s_H[x / ER], v);
      }
      for (int d = 16; d > 0; d >>= 1) part += __shfl_down_sync(0xffffffffu, part, d);
      if ((threadIdx.x & 31) == 0) atomicAdd(&s_total, part);
    }
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += blockDim.x) {  // heaviest first, ties to the lower id
      const int r = x / ER;
      if (s_H[r] <= lo) {  // never sheds: the order is not needed
        s_sT[x] = s_T[x];
        s_ord[x] = x;
        continue;
      }
      const int32_t v = s_T[x];
      int k = 0;
      for (int y = r * ER; y < (r + 1) * ER; ++y) {
        const int32_t w = s_T[y];
        k += (w > v) || (w == v && y < x);
      }
      s_sT[r * ER + k] = v;
      s_ord[r * ER + k] = x;
    }
    for (int r = threadIdx.x; r < R; r += blockDim.x) atomicMax(&s_maxH, s_H[r]);
    __syncthreads();
  }
  const bool valid = (int64_t)s_total == P;
  const int64_t hi = (int64_t)s_maxH > lo ? (int64_t)s_maxH : lo;
  const int64_t tmin = lo + (int64_t)blockIdx.x * blockDim.x;  // this CTA's smallest candidate
  if (phase & Q_SEARCH) {
    if (threadIdx.x == 0) {
      if (valid && blockIdx.x == 0) atomicMin(hdr + QH_BEST, (uint32_t)hi);
      int no = 0, nm = 0;
      for (int r = 0; r < R; ++r) {
        if (s_H[r] > tmin) {
          s_oH[no] = s_H[r];
          s_oOff[no++] = r * ER;
        }
        if (s_H[r] < hi) {
          s_mH[nm] = s_H[r];
          s_mR[nm++] = r;
        }
      }
      s_novr = no;
      s_nroom = nm;
    }
    __syncthreads();
    if (valid) {
      const int64_t N = (int64_t)gridDim.x * blockDim.x;
      volatile uint32_t* best = hdr + QH_BEST;
      const int novr = s_novr, nroom = s_nroom;
      for (int64_t tau = tmin + threadIdx.x; tau < hi; tau += N) {
        if (tau >= (int64_t)*best) break;
        if (q_feasible((int32_t)tau, s_sT, s_oH, s_oOff, novr, s_mH, nroom, ER, B)) {
          atomicMin(hdr + QH_BEST, (uint32_t)tau);
          break;
        }
      }
    }
  }
  if (!(phase & Q_BUILD)) return;
  if (phase & Q_SEARCH) {  // both: the last CTA to finish its candidates builds
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&hdr[QH_TICKET_SEARCH], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
  }

  // ---- the plan at tau*, by the last CTA, from shared memory
  const int32_t tau = valid ? (int32_t)atomicAdd(hdr + QH_BEST, 0u) : -1;
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
  // chunks at tau*: each rank sheds H_r - tau* from its heaviest experts
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    const int32_t X = valid ? s_H[r] - tau : 0;
    int m = 0;
    for (int32_t acc = 0; m < ER && acc < X && s_sT[r * ER + m] > 0; ++m) acc += s_sT[r * ER + m];
    s_rl[r] = m;  // (s_rl is free until the rank loads)
  }
  __syncthreads();
  const int nch = block_scan_array(s_rl, R, warp_sums);
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    const int32_t X = valid ? s_H[r] - tau : 0;
    const int m = (r + 1 < R ? s_rl[r + 1] : nch) - s_rl[r];
    int32_t acc = 0;
    for (int i = 0; i < m; ++i) {
      const int32_t v = s_sT[r * ER + i];
      s_chE[s_rl[r] + i] = s_ord[r * ER + i];
      s_chN[s_rl[r] + i] = min(v, X - acc);
      acc += v;
    }
  }
  __syncthreads();
  for (int k = threadIdx.x; k < nch; k += blockDim.x) s_chB[k] = s_chN[k];
  __syncthreads();
  const int32_t Xtot = block_scan_array(s_chB, nch, warp_sums);  // chunk starts
  // room windows: room j takes [x, min(x + room, end of the B-th chunk from x));
  // one thread runs the recurrence, with a forward pointer over the chunks
  if (threadIdx.x == 0) {
    int nw = 0, k = 0;
    int32_t x = 0;
    for (int j = 0; j < s_nroom && x < Xtot && B > 0; ++j) {
      if (s_mH[j] >= tau) continue;
      int32_t e = x + (tau - s_mH[j]);
      if (k + B - 1 < nch) e = min(e, s_chB[k + B - 1] + s_chN[k + B - 1]);
      e = min(e, Xtot);
      s_wS[nw] = x;
      s_wE[nw] = e;
      s_wR[nw] = s_mR[j];
      ++nw;
      x = e;
      while (k < nch && s_chB[k] + s_chN[k] <= x) ++k;
    }
    s_nwin = nw;
  }
  __syncthreads();
  const int nw = s_nwin;
  // pieces per window: the chunks it overlaps (binary searches over chunk starts)
  for (int w = threadIdx.x; w < nw; w += blockDim.x) {
    int a = 0, b = nch - 1;  // chunk holding position s_wS[w]: last start <= it
    while (a < b) {
      const int mid = (a + b + 1) >> 1;
      if (s_chB[mid] <= s_wS[w]) a = mid; else b = mid - 1;
    }
    int c = a, d = nch - 1;  // chunk holding position s_wE[w] - 1
    while (c < d) {
      const int mid = (c + d + 1) >> 1;
      if (s_chB[mid] <= s_wE[w] - 1) c = mid; else d = mid - 1;
    }
    s_wP[w] = c - a + 1;
    s_rnrep[s_wR[w]] = c - a + 1;
  }
  __syncthreads();
  const int n_pieces = block_scan_array(s_wP, nw, warp_sums);
  // emit in match order: window by window, chunk by chunk
  for (int w = threadIdx.x; w < nw; w += blockDim.x) {
    int a = 0, b = nch - 1;
    while (a < b) {
      const int mid = (a + b + 1) >> 1;
      if (s_chB[mid] <= s_wS[w]) a = mid; else b = mid - 1;
    }
    const int np = (w + 1 < nw ? s_wP[w + 1] : n_pieces) - s_wP[w];
    for (int q = 0; q < np && s_wP[w] + q < cap; ++q) {
      const int k = a + q, m = s_wP[w] + q;
      const int32_t cb = s_chB[k], ce = cb + s_chN[k];
      const int e = s_chE[k];
      s_re[m] = e;
      s_rr[m] = s_wR[w];
      s_rc[m] = min(ce, s_wE[w]) - max(cb, s_wS[w]);
      if (cb >= s_wS[w]) s_rfirst[e] = m;  // the chunk starts in this window
      atomicAdd(&s_rcnt[e], 1);
    }
  }
  for (int k = threadIdx.x; k < E; k += blockDim.x) plan[L.rep_experts + k] = k < nch ? s_chE[k] : -1;
  if (threadIdx.x == 0) {
    s_nrep = min(n_pieces, cap);
    plan[L.n_chunks] = nch;
  }
  __syncthreads();
  const int n_rep = s_nrep;
  for (int m = threadIdx.x; m < cap; m += blockDim.x) {
    const bool v = m < n_rep;
    plan[L.rep_expert + m] = v ? s_re[m] : -1;
    plan[L.rep_rank + m] = v ? s_rr[m] : -1;
    plan[L.rep_count + m] = v ? s_rc[m] : 0;
  }
  for (int x = threadIdx.x; x < E; x += blockDim.x) {  // home quotas
    int32_t q = valid ? s_T[x] : 0;
    for (int k = 0; k < s_rcnt[x]; ++k) q -= s_rc[s_rfirst[x] + k];
    s_hq[x] = q;
    plan[L.home_quota + x] = q;
    plan[L.rep_first + x] = s_rfirst[x];
    plan[L.rep_cnt + x] = s_rcnt[x];
  }
  for (int r = threadIdx.x; r < R; r += blockDim.x) s_rrf[r] = s_rnrep[r];
  __syncthreads();
  block_scan_array(s_rrf, R, warp_sums);  // replicas received by lower ranks
  // local pairs of every instance: min(quota, pairs of e from the instance's
  // rank); the prefix loads are independent, so they go out together
  for (int i = threadIdx.x; i < E + n_rep; i += blockDim.x) {
    const int e = i < E ? i : s_re[i - E];
    const int r = i < E ? i / ER : s_rr[i - E];
    const int32_t q = i < E ? s_hq[i] : s_rc[i - E];
    const int32_t lpre = __ldcg(excl + (int64_t)r * tpr * E + e);
    const int32_t lsrc = __ldcg(excl + (int64_t)(r + 1) * tpr * E + e) - lpre;
    const int32_t loc = valid ? min(q, lsrc) : 0;
    s_loc[i] = loc;
    plan[L.inst_local + i] = loc;
    plan[L.inst_lpre + i] = lpre;
  }
  __syncthreads();
  // cumulative looked-up ranges in instance order (home, then replicas), and
  // the running local count over e's replicas (match order = ascending rank)
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int32_t cum = s_hq[x] - s_loc[x], inc = 0;
    plan[L.inst_cum + x] = 0;
    for (int k = 0; k < s_rcnt[x]; ++k) {
      const int m = s_rfirst[x] + k;
      plan[L.inst_cum + E + m] = cum;
      cum += s_rc[m] - s_loc[E + m];
      inc += s_loc[E + m];
      plan[L.rep_local_incl + m] = inc;
    }
    atomicAdd(&s_local, s_loc[x] + inc);
  }
  for (int r = threadIdx.x; r < R; r += blockDim.x) {  // rank loads
    int32_t l = 0;
    for (int x = r * ER; x < (r + 1) * ER; ++x) l += s_hq[x];
    for (int k = 0; k < s_rnrep[r]; ++k) l += s_rc[s_rrf[r] + k];
    s_rl[r] = l;
    plan[L.rank_load + r] = l;
    plan[L.rank_nrep + r] = s_rnrep[r];
    plan[L.rank_rep_first + r] = s_rrf[r];
  }
  __syncthreads();
  block_scan_array(s_rl, R, warp_sums);  // first row of each rank
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
      row += s_rc[m];
      plan[L.cu_seqlens + slot + 1] = row;
    }
  }
  for (int slot = E + n_rep + threadIdx.x; slot < E + cap; slot += blockDim.x) {
    plan[L.slot_order + slot] = -1;
    plan[L.cu_seqlens + slot + 1] = valid ? (int32_t)P : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    plan[L.cu_seqlens] = 0;
    plan[L.tau] = tau;
    plan[L.n_rep] = n_rep;
    plan[L.n_local] = s_local;
    if (phase & Q_SEARCH) hdr[QH_TICKET_SEARCH] = 0;
  }
}

__global__ void __launch_bounds__(Q_SEARCH_THREADS)
    k_q_search(const int32_t* __restrict__ loads, const int32_t* __restrict__ excl, int tpr, int E, int R, int B,
               int64_t P, uint32_t* hdr, int32_t* __restrict__ plan, EpQuotaLayout L) {
  extern __shared__ int32_t sm[];
  q_search_build(loads, excl, tpr, E, R, B, P, hdr, plan, L, sm, Q_ALL);
}

// ----------------------------------------------------------------- 4. layout

// base_counts == NULL: the pairs of all R source ranks, rank-aligned tiles,
// excl the global per-tile prefixes.  Otherwise (rank-local form) the pairs of
// source rank base_rank only: excl holds the per-tile prefixes of those pairs
// alone (tpr = its tile count), base_counts [R, E] is the gathered load matrix
// that gives the pairs of each expert on lower source ranks, pos is indexed by
// the rank's own pairs and src may be NULL.
// Tile t of the layout; sm: the layout's shared memory (q_layout_smem).  The
// plan and the prefixes are read past L1 (in the one-launch route other CTAs
// of the same launch wrote them).  stage & 1: load the tile's ids and its
// per-warp first ranks (needs only the prefixes); stage & 2: read the plan and
// place every pair (needs the plan, and stage 1 done on the same sm).
__device__ void q_layout_tile(const int32_t* __restrict__ topk, int64_t SK, int E, int R, int tile, int tpr,
                              const int32_t* __restrict__ excl, const int32_t* __restrict__ base_counts,
                              int base_rank, const int32_t* __restrict__ plan, const EpQuotaLayout& L,
                              int32_t* __restrict__ pos, int32_t* __restrict__ src, int32_t* dev_status, int64_t t,
                              int32_t* sm, int stage) {
  int32_t* s_ids = sm;                  // [tile]
  int32_t* s_whist = s_ids + tile;      // [SCAT_WARPS * E]
  int32_t* s_lpre = s_whist + SCAT_WARPS * E;  // [E] pairs of e from source ranks below this tile's
  int32_t* s_oloc = s_lpre + E;         // [E] local pairs of e's instance on this rank (0: none)
  int32_t* s_obase = s_oloc + E;        // [E] its first row
  int32_t* s_locb = s_obase + E;        // [E] local pairs of e's instances on ranks <= this one
  int32_t* s_rf = s_locb + E;           // [E]
  int32_t* s_rc = s_rf + E;             // [E]
  int32_t* s_rrank = s_rc + E;          // [cap] rep_rank
  int32_t* s_icum = s_rrank + L.cap;    // [E + cap] cumulative start of instance i's looked-up range
  int32_t* s_istart = s_icum + E + L.cap;  // [E + cap] its first looked-up row
  int32_t* s_ispan = s_istart + E + L.cap; // [E + cap] its looked-up rows
  int32_t* s_excl = s_ispan + E + L.cap;   // [E] this tile's list offsets
  __shared__ int s_flags;
  const bool local = base_counts != nullptr;
  const int rs = local ? base_rank : (int)(t / tpr);
  const int64_t lt = local ? t : t % tpr;
  const int64_t p0 = (local ? 0 : (int64_t)rs * SK) + lt * tile;
  const int n = (int)min((int64_t)tile, SK - lt * tile);
  const int ER = E / R;
  const int64_t P = (int64_t)R * SK;
  if (stage & 1) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int32_t b = 0;
      if (local)
        for (int r = 0; r < rs; ++r) b += base_counts[(int64_t)r * E + e];
      s_excl[e] = __ldcg(excl + t * E + e) + b;
    }
    // (tile_ranks_prepare reads s_excl after its own barriers)
    tile_ranks_prepare(topk, E, tile, p0, n, s_excl, s_ids, s_whist);
  }
  if (!(stage & 2)) return;
  const int32_t tau = __ldcg(plan + L.tau);
  if (threadIdx.x == 0) s_flags = 0;
  if (tau < 0) {  // no plan (bad input): nothing is placed
    for (int i = threadIdx.x; i < n; i += blockDim.x) pos[p0 + i] = -1;
    return;
  }
  const int n_rep = min(max(__ldcg(plan + L.n_rep), 0), L.cap);
  for (int i = threadIdx.x; i < E + n_rep; i += blockDim.x) {
    const int32_t q = i < E ? __ldcg(plan + L.home_quota + i) : __ldcg(plan + L.rep_count + i - E);
    const int32_t loc = __ldcg(plan + L.inst_local + i);
    s_icum[i] = __ldcg(plan + L.inst_cum + i);
    s_istart[i] = __ldcg(plan + L.inst_base + i) + loc;
    s_ispan[i] = q - loc;
    if (i >= E) s_rrank[i - E] = __ldcg(plan + L.rep_rank + i - E);
  }
  __syncthreads();
  // per-expert view from this tile's source rank (e's replicas sit on
  // ascending ranks, so each lookup is a binary search)
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int rf = __ldcg(plan + L.rep_first + e), rc = __ldcg(plan + L.rep_cnt + e);
    s_rf[e] = rf;
    s_rc[e] = rc;
    if (local) {
      int32_t b = 0;
      for (int r = 0; r < rs; ++r) b += base_counts[(int64_t)r * E + e];
      s_lpre[e] = b;
    } else {
      s_lpre[e] = __ldcg(excl + (int64_t)rs * tpr * E + e);
    }
    int a = 0, b = rc;  // replicas of e on ranks < rs: the first a
    while (a < b) {
      const int mid = (a + b) >> 1;
      if (s_rrank[rf + mid] < rs)
        a = mid + 1;
      else
        b = mid;
    }
    int own = -1, below = a;
    if (e / ER == rs) {
      own = e;
    } else if (a < rc && s_rrank[rf + a] == rs) {
      own = E + rf + a;
      below = a + 1;
    }
    s_oloc[e] = own >= 0 ? __ldcg(plan + L.inst_local + own) : 0;
    s_obase[e] = own >= 0 ? __ldcg(plan + L.inst_base + own) : 0;
    s_locb[e] = (e / ER <= rs ? __ldcg(plan + L.inst_local + e) : 0) +
               (below > 0 ? __ldcg(plan + L.rep_local_incl + rf + below - 1) : 0);
  }
  __syncthreads();
  auto emit = [&](int64_t p, int e, int32_t g) {
    const int32_t ls = g - s_lpre[e];
    int32_t row = -1;
    if (ls < s_oloc[e]) {
      row = s_obase[e] + ls;
    } else {
      // rank among e's pairs not placed locally, then the last instance
      // (home, replicas in match order) whose cumulative start is <= it
      const int32_t j = g - s_locb[e];
      const int rf = s_rf[e];
      int a = 0, b = s_rc[e];
      while (a < b) {
        const int mid = (a + b + 1) >> 1;
        if (s_icum[E + rf + mid - 1] <= j)
          a = mid;
        else
          b = mid - 1;
      }
      const int i = a == 0 ? e : E + rf + a - 1;
      const int32_t off = j - s_icum[i];
      if (off >= 0 && off < s_ispan[i]) row = s_istart[i] + off;
    }
    if (row < 0 || row >= P) {
      atomicOr(&s_flags, EP_DEV_BAD_ROW);
      pos[p] = -1;
      return;
    }
    pos[p] = row;
    if (src) src[row] = (int32_t)p;
  };
  auto bad = [&](int64_t p) {
    atomicOr(&s_flags, EP_DEV_BAD_EXPERT_ID);
    pos[p] = -1;
  };
  tile_ranks_walk(E, tile, p0, n, s_ids, s_whist, emit, bad);
  __syncthreads();
  if (threadIdx.x == 0 && s_flags) flag(dev_status, s_flags);
}

inline size_t q_layout_smem(int tile, int E, int cap) {
  return sizeof(int32_t) *
         ((size_t)tile + (size_t)SCAT_WARPS * E + 7 * (size_t)E + (size_t)cap + 3 * ((size_t)E + cap));
}

__global__ void __launch_bounds__(SCAT_THREADS)
    k_q_layout(const int32_t* __restrict__ topk, int64_t SK, int E, int R, int tile, int tpr,
               const int32_t* __restrict__ excl, const int32_t* __restrict__ base_counts, int base_rank,
               const int32_t* __restrict__ plan, EpQuotaLayout L, int32_t* __restrict__ pos,
               int32_t* __restrict__ src, int32_t* dev_status) {
  extern __shared__ int32_t sm[];
  q_layout_tile(topk, SK, E, R, tile, tpr, excl, base_counts, base_rank, plan, L, pos, src, dev_status, blockIdx.x,
                sm, 3);
}

// ------------------------------------------------------- the one-launch route

// The four steps in one cooperative launch (all CTAs co-resident), every CTA
// owning one rank-aligned tile:
//   1. tile counts, added into T_e by integer atomics;  -- grid barrier --
//   2. every CTA tests its threshold candidates from T_e (its own view of the
//      loads, as k_q_search) while the CTAs scan the tile columns into the
//      exclusive prefixes;  -- grid barrier --
//   3. CTA 0 builds the plan at tau* from its view and raises a flag, while
//      the others load their tiles and count them per warp;
//   4. every CTA places its tile's pairs once the flag is up.
// Same outputs as the four launches, bit for bit; every wait is bounded.
struct QFusedArgs {
  const int32_t* topk;
  int64_t SK, P;
  int E, R, B, tile, tpr, ntiles;
  uint32_t* hdr;
  int32_t* tot;
  int32_t* cnt;
  int32_t* excl;
  int32_t* loads;
  int32_t* plan;
  EpQuotaLayout L;
  int32_t* pos;
  int32_t* src;
  int32_t* dev_status;
};

__global__ void __launch_bounds__(SCAT_THREADS) k_q_fused(QFusedArgs a) {
  extern __shared__ int32_t sm[];
  __shared__ int32_t warp_sums[32];
  const int G = gridDim.x, t = blockIdx.x, tid = threadIdx.x, E = a.E;
  if (t == 0 && tid == 0) a.hdr[QH_BEST] = 0xffffffffu;  // read by no CTA before the first barrier
  q_count_tile(a.topk, a.SK, E, a.tile, a.tpr, t, a.cnt, a.tot, sm, a.dev_status);
  grid_barrier(a.hdr + QH_BARRIER, (uint32_t)G, a.dev_status);

  q_search_build(a.tot, a.excl, a.tpr, E, a.R, a.B, a.P, a.hdr, a.plan, a.L, sm, Q_SEARCH);
  for (int e = t; e < E; e += G) {  // column e over the G tiles (G <= blockDim)
    const int32_t v = tid < G ? __ldcg(a.cnt + (int64_t)tid * E + e) : 0;
    int32_t total;
    const int32_t ex = block_exclusive_scan(v, warp_sums, &total);
    if (tid < G) a.excl[(int64_t)tid * E + e] = ex;
    if (tid == 0) {
      a.excl[(int64_t)G * E + e] = total;
      a.loads[e] = total;
    }
  }
  grid_barrier(a.hdr + QH_BARRIER, 2u * G, a.dev_status);

  if (t == 0) {
    q_search_build(a.tot, a.excl, a.tpr, E, a.R, a.B, a.P, a.hdr, a.plan, a.L, sm, Q_BUILD);
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      st_release_u32(a.hdr + QH_FLAG, 1u);
    }
  }
  // the plan-free half of the layout while CTA 0 builds (its search state is
  // dead once the build is done), then the rest once the plan is out
  q_layout_tile(a.topk, a.SK, E, a.R, a.tile, a.tpr, a.excl, nullptr, 0, a.plan, a.L, a.pos, a.src, a.dev_status,
                t, sm, 1);
  wait_at_least(a.hdr + QH_FLAG, 1u, a.dev_status);
  q_layout_tile(a.topk, a.SK, E, a.R, a.tile, a.tpr, a.excl, nullptr, 0, a.plan, a.L, a.pos, a.src, a.dev_status,
                t, sm, 2);
}

// Launches the one-launch route when its grid can be co-resident within the
// workspace's tile regions; returns false (nothing launched) otherwise.
static bool q_fused_launch(const int32_t* topk, int64_t SK, int E, int R, int B, int32_t* loads, int32_t* plan,
                           const EpQuotaLayout& L, int32_t* pos, int32_t* src, char* ws, const QWs& w,
                           int64_t ws_tiles, int32_t* dev_status, cudaStream_t stream, int* rc) {
  *rc = EP_OK;
  if (SK <= 0) return false;
  const size_t base = std::max(q_search_smem(E, R), sizeof(int32_t) * (size_t)E);
  for (int per_sm = 2; per_sm >= 1; --per_sm) {
    const int64_t resident = (int64_t)num_sms() * per_sm;
    if (R > resident) continue;
    const int64_t tpr0 = std::min<int64_t>(resident / R, SCAT_THREADS / R > 0 ? SCAT_THREADS / R : 1);
    if (tpr0 < 1) continue;
    int64_t tile = ((SK + tpr0 - 1) / tpr0 + 511) / 512 * 512;
    const int64_t tpr = (SK + tile - 1) / tile;
    const int64_t nt = (int64_t)R * tpr;
    if (nt > resident || nt > SCAT_THREADS || nt > ws_tiles || tile > (1 << 20)) continue;
    const size_t smem = std::max(base, q_layout_smem((int)tile, E, L.cap));
    if (smem > 227 * 1024) continue;
    if (smem > 48 * 1024 &&
        !raise_smem_limit((const void*)k_q_fused, smem))
      continue;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_q_fused, SCAT_THREADS, smem) != cudaSuccess ||
        occ < per_sm)
      continue;
    if (cudaMemsetAsync(ws, 0, w.cnt, stream) != cudaSuccess) {  // header words and T_e
      *rc = EP_ERR_CUDA;
      return true;
    }
    QFusedArgs args;
    args.topk = topk;
    args.SK = SK;
    args.P = (int64_t)R * SK;
    args.E = E;
    args.R = R;
    args.B = B;
    args.tile = (int)tile;
    args.tpr = (int)tpr;
    args.ntiles = (int)nt;
    args.hdr = reinterpret_cast<uint32_t*>(ws + w.hdr);
    args.tot = reinterpret_cast<int32_t*>(ws + w.tot);
    args.cnt = reinterpret_cast<int32_t*>(ws + w.cnt);
    args.excl = reinterpret_cast<int32_t*>(ws + w.excl);
    args.loads = loads;
    args.plan = plan;
    args.L = L;
    args.pos = pos;
    args.src = src;
    args.dev_status = dev_status;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nt);
    cfg.blockDim = dim3(SCAT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    *rc = cudaLaunchKernelEx(&cfg, k_q_fused, args) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
    if (*rc == EP_OK) count_launch();
    return true;
  }
  return false;
}

struct QCountsWs {
  size_t hdr, pre, bytes;
};
inline QCountsWs q_counts_ws(int E, int R) {
  QCountsWs w;
  w.hdr = 0;
  w.pre = 256;
  w.bytes = (w.pre + sizeof(int32_t) * (size_t)E * (size_t)(R + 1) + 255) & ~(size_t)255;
  return w;
}

static int run_q_layout(const int32_t* topk, int64_t SK, int E, int R, int tile, int tpr, int64_t ntiles,
                        const int32_t* excl, const int32_t* base_counts, int base_rank, const int32_t* plan,
                        const EpQuotaLayout& L, int32_t* pos, int32_t* src, int32_t* dev_status,
                        cudaStream_t stream) {
  const size_t smem = q_layout_smem(tile, E, L.cap);
  if (smem > 48 * 1024 &&
      !raise_smem_limit((const void*)k_q_layout, smem))
    return EP_ERR_CUDA;
  k_q_layout<<<(unsigned)ntiles, SCAT_THREADS, smem, stream>>>(topk, SK, E, R, tile, tpr, excl, base_counts,
                                                               base_rank, plan, L, pos, src, dev_status);
  count_launch();
  return launch_status();
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
  int frc = EP_OK;
  if (q_fused_launch(topk_ids, SK, E, R, B, loads, plan, L, pos, src, base, w, q.ntiles, dev_status, stream, &frc))
    return frc == EP_OK ? launch_status() : frc;
  uint32_t* hdr = reinterpret_cast<uint32_t*>(base + w.hdr);
  int32_t* cnt = reinterpret_cast<int32_t*>(base + w.cnt);
  int32_t* excl = reinterpret_cast<int32_t*>(base + w.excl);
  k_q_count<<<(unsigned)std::max<int64_t>(q.ntiles, 1), SCAT_THREADS, sizeof(int32_t) * E, stream>>>(
      topk_ids, SK, E, q.tile, q.tpr, q.ntiles, cnt, hdr, dev_status);
  k_q_scan<<<(E + Q_SCAN_EXPERTS - 1) / Q_SCAN_EXPERTS, Q_SCAN_THREADS, 0, stream>>>(cnt, q.ntiles, E, excl, loads);
  const size_t search_smem = q_search_smem(E, R);
  if (search_smem > 48 * 1024 &&
      !raise_smem_limit((const void*)k_q_search, search_smem))
    return EP_ERR_CUDA;
  k_q_search<<<2 * num_sms(), Q_SEARCH_THREADS, search_smem, stream>>>(loads, excl, q.tpr, E, R, B, P, hdr, plan, L);
  count_launch(3);
  if (q.ntiles > 0) {
    const int rc = run_q_layout(topk_ids, SK, E, R, q.tile, q.tpr, q.ntiles, excl, nullptr, 0, plan, L, pos, src,
                                dev_status, stream);
    if (rc != EP_OK) return rc;
  }
  return launch_status();
}

extern "C" int ep_quota_counts_workspace_size(int E, int R, size_t* bytes) {
  if (!bytes || E < 1 || E > EP_MAX_EXPERTS || R < 1 || R > EP_MAX_RANKS || E % R) return EP_ERR_ARG;
  *bytes = q_counts_ws(E, R).bytes;
  return EP_OK;
}

extern "C" int ep_quota_plan_from_counts(const int32_t* counts, int R, int64_t S, int K, int E, int B, int32_t* loads,
                                         int32_t* plan, size_t plan_words, void* ws, size_t ws_bytes,
                                         int32_t* dev_status, cudaStream_t stream) {
  if (!counts || !loads || !plan || !ws || R < 1 || R > EP_MAX_RANKS || E < 1 || E > EP_MAX_EXPERTS || E % R ||
      K < 1 || K > E || S < 0 || B < 0)
    return EP_ERR_ARG;
  if ((int64_t)R * S * K >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  EpQuotaLayout L;
  quota_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  const QCountsWs w = q_counts_ws(E, R);
  if (ws_bytes < w.bytes) return EP_ERR_CAPACITY;
  char* base = static_cast<char*>(ws);
  uint32_t* hdr = reinterpret_cast<uint32_t*>(base + w.hdr);
  int32_t* pre = reinterpret_cast<int32_t*>(base + w.pre);
  k_q_counts_prefix<<<(E + 255) / 256, 256, 0, stream>>>(counts, R, E, pre, loads, hdr);
  const size_t search_smem = q_search_smem(E, R);
  if (search_smem > 48 * 1024 &&
      !raise_smem_limit((const void*)k_q_search, search_smem))
    return EP_ERR_CUDA;
  const int64_t P = (int64_t)R * S * K;
  k_q_search<<<2 * num_sms(), Q_SEARCH_THREADS, search_smem, stream>>>(loads, pre, 1, E, R, B, P, hdr, plan, L);
  count_launch(2);
  (void)dev_status;  // invalid counts show as tau = -1 in the plan
  return launch_status();
}

extern "C" int ep_quota_layout_rank(const int32_t* topk_local, int64_t S, int K, int E, int R, int rank,
                                    const int32_t* counts, const int32_t* plan, size_t plan_words, const void* ws,
                                    size_t ws_bytes, int32_t* pos_local, int32_t* dev_status, cudaStream_t stream) {
  if (!valid_tke(S, K, E) || R < 1 || R > EP_MAX_RANKS || E % R || rank < 0 || rank >= R) return EP_ERR_ARG;
  if ((int64_t)R * S * K >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  if (!plan || !ws || !counts) return EP_ERR_ARG;
  const int64_t SK = S * K;
  if (SK > 0 && (!topk_local || !pos_local)) return EP_ERR_ARG;
  EpQuotaLayout L;
  quota_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  const WsLayout wl = ws_layout(SK, E);  // the scratch ep_route_stats filled for topk_local
  if (ws_bytes < wl.bytes) return EP_ERR_CAPACITY;
  if (SK == 0) return EP_OK;
  const int tile = tile_pairs_for(SK);
  const int64_t nt = num_tiles(SK, tile);
  const int32_t* excl = reinterpret_cast<const int32_t*>(static_cast<const char*>(ws) + wl.excl_off);
  return run_q_layout(topk_local, SK, E, R, tile, (int)nt, nt, excl, counts, rank, plan, L, pos_local, nullptr,
                      dev_status, stream);
}
