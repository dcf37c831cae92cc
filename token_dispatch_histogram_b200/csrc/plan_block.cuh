// Block-level replica planner, shared by the one-CTA ep_plan kernel and the
// fused route kernel.  Works for any blockDim.x (a multiple of 32, <= 1024) and
// any R <= EP_MAX_RANKS, E <= EP_MAX_EXPERTS.
//
// [GR] "Η βασική υπόσχεση του MoonEP: σταθερό φορτίο S × K" (twodots.gr MoonEP
// article): every rank ends with exactly S*K pairs through a few temporary
// expert copies planned online on the GPU.  Rule (this library's deterministic
// reading): rank load L_r; an overloaded rank's excess L_r - S*K is cut into
// chunks from its home experts in descending id (chunk = min(T_e, excess left));
// underloaded ranks' deficits are taken in ascending rank; the two prefix-sum
// sequences are merged and every piece between consecutive breakpoints is one
// replica (expert, receiving rank, count), numbered in merge ("match") order.
//
// Parallel form: per-rank walks (<= E/R steps each) strided over threads, four
// rank-length prefix sums in one block scan, then a merge-path: each breakpoint
// finds its merged position by binary search in the other list, so all replicas
// are emitted independently.
#pragma once

#include "common.cuh"

namespace ep {

__device__ __forceinline__ int lower_bound_i32(const int32_t* a, int n, int32_t v) {
  int lo = 0, hi = n;  // first i with a[i] >= v
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < v)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

__device__ __forceinline__ int upper_bound_i32(const int32_t* a, int n, int32_t v) {
  int lo = 0, hi = n;  // first i with a[i] > v
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] <= v)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

// Exclusive scan of four int32 per thread at once; totals in *total.
__device__ __forceinline__ int4 block_exclusive_scan4(int4 v, int4* warp_sums, int4* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int4 x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int4 y = make_int4(__shfl_up_sync(~0u, x.x, d), __shfl_up_sync(~0u, x.y, d), __shfl_up_sync(~0u, x.z, d),
                             __shfl_up_sync(~0u, x.w, d));
    if (lane >= d) {
      x.x += y.x;
      x.y += y.y;
      x.z += y.z;
      x.w += y.w;
    }
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int4 s = lane < nwarps ? warp_sums[lane] : make_int4(0, 0, 0, 0);
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int4 y = make_int4(__shfl_up_sync(~0u, s.x, d), __shfl_up_sync(~0u, s.y, d),
                               __shfl_up_sync(~0u, s.z, d), __shfl_up_sync(~0u, s.w, d));
      if (lane >= d) {
        s.x += y.x;
        s.y += y.y;
        s.z += y.z;
        s.w += y.w;
      }
    }
    if (lane < nwarps) warp_sums[lane] = s;
  }
  __syncthreads();
  const int4 base = warp > 0 ? warp_sums[warp - 1] : make_int4(0, 0, 0, 0);
  *total = warp_sums[nwarps - 1];
  __syncthreads();
  return make_int4(base.x + x.x - v.x, base.y + x.y - v.y, base.z + x.z - v.z, base.w + x.w - v.w);
}

// Exclusive scan of a[0..n) in place (shared or global memory); returns the
// total.  Each thread scans one contiguous segment.
__device__ __forceinline__ int32_t block_scan_inplace(int32_t* a, int n, int32_t* warp_sums) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b = min(n, (int)threadIdx.x * per), e = min(n, b + per);
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

// Words of shared scratch plan_block needs.
__host__ __device__ __forceinline__ int plan_work_words(int E, int R) { return 9 * R + 5 * E + 16; }

// Writes the whole plan buffer from loads in shared memory.  Every thread of
// the block must call it.  Returns n_rep (or 0 when the loads are invalid, in
// which case EP_DEV_BAD_LOADS is reported and an empty plan is written).
static __device__ int plan_block(const int32_t* s_loads, int R, int32_t SK, int E, int32_t* __restrict__ plan,
                          const EpPlanLayout& L, int32_t* work, int32_t* dev_status) {
  __shared__ int4 warp_sums4[32];
  __shared__ int32_t warp_sums[32];
  __shared__ int s_bad;
  const int ER = E / R;
  const int tid = threadIdx.x, nt = blockDim.x;
  int32_t* r_L = work;                  // [R]
  int32_t* r_X = r_L + R;               // [R + 1] excess, then its exclusive prefix
  int32_t* r_D = r_X + R + 1;           // [R + 1] deficit, then prefix
  int32_t* r_nch = r_D + R + 1;         // [R + 1] chunk count, then prefix
  int32_t* r_def = r_nch + R + 1;       // [R + 1] is-underloaded, then prefix
  int32_t* ch_e = r_def + R + 1;        // [E]
  int32_t* ch_start = ch_e + E;         // [E + 1]
  int32_t* ch_first = ch_start + E + 1; // [E + 1]
  int32_t* chunk_of = ch_first + E + 1; // [E]
  int32_t* home = chunk_of + E;         // [E]
  int32_t* df_rank = home + E;          // [R]
  int32_t* df_start = df_rank + R;      // [R + 1]
  int32_t* df_first = df_start + R + 1; // [R + 1]
  int32_t* df_coinc = df_first + R + 1; // [R + 1]

  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int e = tid; e < E; e += nt) {
    chunk_of[e] = -1;
    if (s_loads[e] < 0) s_bad = 1;
  }
  // per-rank quantities, then their prefix sums in one pass (segments per thread)
  const int per = (R + nt - 1) / nt;
  const int rb = min(R, tid * per), re = min(R, rb + per);
  int4 seg = make_int4(0, 0, 0, 0);
  for (int r = rb; r < re; ++r) {
    int32_t Lr = 0;
    for (int e = r * ER; e < (r + 1) * ER; ++e) Lr += s_loads[e];
    const int32_t X = Lr > SK ? Lr - SK : 0, D = Lr < SK ? SK - Lr : 0;
    int32_t rem = X, nch = 0;
    for (int e = (r + 1) * ER - 1; e >= r * ER && rem > 0; --e) {
      const int32_t take = min(s_loads[e], rem);
      if (take > 0) {
        ++nch;
        rem -= take;
      }
    }
    r_L[r] = Lr;
    r_X[r] = X;
    r_D[r] = D;
    r_nch[r] = nch;
    r_def[r] = D > 0;
    seg.x += X;
    seg.y += D;
    seg.z += nch;
    seg.w += D > 0;
  }
  int4 tot;
  int4 run = block_exclusive_scan4(seg, warp_sums4, &tot);
  for (int r = rb; r < re; ++r) {
    const int4 v = make_int4(r_X[r], r_D[r], r_nch[r], r_def[r]);
    r_X[r] = run.x;
    r_D[r] = run.y;
    r_nch[r] = run.z;
    r_def[r] = run.w;
    run.x += v.x;
    run.y += v.y;
    run.z += v.z;
    run.w += v.w;
  }
  if (tid == 0) {
    r_X[R] = tot.x;
    r_D[R] = tot.y;
    r_nch[R] = tot.z;
    r_def[R] = tot.w;
    if (tot.x != tot.y) s_bad = 1;  // sum_r (L_r - S*K) != 0: loads do not add up to R*S*K
  }
  __syncthreads();
  const bool bad = s_bad != 0;
  const int nC = bad ? 0 : r_nch[R], nD = bad ? 0 : r_def[R];
  const int32_t Xtot = r_X[R];

  // chunks (descending id per overloaded rank), home counts, deficits
  for (int r = tid; r < R; r += nt) {
    for (int e = r * ER; e < (r + 1) * ER; ++e) home[e] = bad ? 0 : s_loads[e];
    if (bad) continue;
    const int32_t Lr = r_L[r];
    int32_t rem = Lr > SK ? Lr - SK : 0, start = r_X[r];
    int c = r_nch[r];
    for (int e = (r + 1) * ER - 1; e >= r * ER && rem > 0; --e) {
      const int32_t take = min(s_loads[e], rem);
      if (take > 0) {
        ch_e[c] = e;
        ch_start[c] = start;
        chunk_of[e] = c;
        home[e] = s_loads[e] - take;
        start += take;
        rem -= take;
        ++c;
      }
    }
    if (Lr < SK) {
      df_rank[r_def[r]] = r;
      df_start[r_def[r]] = r_D[r];
    }
  }
  if (tid == 0) {
    ch_start[nC] = Xtot;
    df_start[nD] = Xtot;
    if (bad) flag(dev_status, EP_DEV_BAD_LOADS);
  }
  __syncthreads();
  // deficit starts that coincide with a chunk start share one breakpoint
  for (int d = tid; d < nD; d += nt) {
    const int32_t v = df_start[d];
    const int i = lower_bound_i32(ch_start, nC, v);
    df_coinc[d] = (i < nC && ch_start[i] == v) ? 1 : 0;
  }
  __syncthreads();
  const int32_t ncoinc = block_scan_inplace(df_coinc, nD, warp_sums);
  if (tid == 0) df_coinc[nD] = ncoinc;
  __syncthreads();
  const int n_rep = nC + nD - ncoinc;

  int32_t* rep_expert = plan + L.rep_expert;
  int32_t* rep_rank = plan + L.rep_rank;
  int32_t* rep_count = plan + L.rep_count;
  int32_t* rep_begin = plan + L.rep_begin;
  int32_t* rep_base = plan + L.rep_base;
  auto emit = [&](int m, int c, int d, int32_t v) {
    const int32_t end = min(ch_start[c + 1], df_start[d + 1]);
    const int e = ch_e[c];
    const int rr = df_rank[d];
    rep_expert[m] = e;
    rep_rank[m] = rr;
    rep_count[m] = end - v;
    rep_begin[m] = home[e] + (v - ch_start[c]);
    rep_base[m] = rr * SK + r_L[rr] + (v - df_start[d]);  // the receiver is underloaded: its home rows = L_r
  };
  for (int c = tid; c < nC; c += nt) {
    const int32_t v = ch_start[c];
    const int dl = lower_bound_i32(df_start, nD, v);
    const int m = c + dl - df_coinc[dl];
    const int d = upper_bound_i32(df_start, nD, v) - 1;
    ch_first[c] = m;
    if (df_start[d] == v) df_first[d] = m;
    emit(m, c, d, v);
  }
  for (int d = tid; d < nD; d += nt) {
    const int32_t v = df_start[d];
    const int cl = lower_bound_i32(ch_start, nC, v);
    if (cl < nC && ch_start[cl] == v) continue;
    const int m = cl + d - df_coinc[d];
    df_first[d] = m;
    emit(m, cl - 1, d, v);
  }
  if (tid == 0) {
    ch_first[nC] = n_rep;
    df_first[nD] = n_rep;
  }
  __syncthreads();

  for (int e = tid; e < E; e += nt) {
    const int c = chunk_of[e];
    plan[L.home_count + e] = home[e];
    plan[L.copy_first + e] = c >= 0 ? ch_first[c] : 0;
    plan[L.copy_cnt + e] = c >= 0 ? ch_first[c + 1] - ch_first[c] : 0;
    plan[L.rep_experts + e] = e < nC ? ch_e[e] : -1;
  }
  for (int r = tid; r < R; r += nt) {
    const int32_t Lr = bad ? 0 : r_L[r];
    const int di = bad ? 0 : r_def[r];
    const int32_t first = bad ? 0 : df_first[di];
    const int32_t nrecv = (bad || Lr >= SK) ? 0 : df_first[di + 1] - df_first[di];
    plan[L.rank_load + r] = Lr;
    plan[L.rank_rep_first + r] = first;
    plan[L.rank_nrep + r] = nrecv;
    int32_t row = r * SK;
    const int sbase = r * ER + first;
    for (int i = 0; i < ER; ++i) {
      const int e = r * ER + i;
      plan[L.home_base + e] = row;
      plan[L.slot_order + sbase + i] = e;
      plan[L.cu_seqlens + sbase + i] = row;
      row += home[e];
    }
    for (int j = 0; j < nrecv; ++j) {
      const int m = first + j;
      plan[L.slot_order + sbase + ER + j] = E + m;
      plan[L.cu_seqlens + sbase + ER + j] = rep_base[m];
    }
  }
  for (int i = E + n_rep + tid; i <= E + L.cap; i += nt) {
    plan[L.cu_seqlens + i] = R * SK;
    if (i < E + L.cap) plan[L.slot_order + i] = -1;
  }
  for (int m = n_rep + tid; m < L.cap; m += nt) {
    rep_expert[m] = -1;
    rep_rank[m] = -1;
    rep_count[m] = 0;
    rep_begin[m] = 0;
    rep_base[m] = 0;
  }
  if (tid == 0) {
    plan[L.n_rep] = n_rep;
    plan[L.n_chunks] = nC;
  }
  return n_rep;
}

}  // namespace ep
