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
// Parallel form: closed-form chunks from a prefix sum of the loads, rank
// prefix sums in one block scan, then a merge-path: each breakpoint finds its
// merged position by binary search in the other list, so all replicas are
// emitted independently.
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
__host__ __device__ __forceinline__ int plan_work_words(int E, int R) { return 7 * E + 7 * R + 24; }

// Writes the whole plan buffer from loads in shared memory.  Every thread of
// the block must call it.  Returns n_rep (or 0 when the loads are invalid, in
// which case EP_DEV_BAD_LOADS is reported and an empty plan is written).
//
// No thread walks a rank serially: with pre[] the prefix sum of T_e in expert
// order, rank r's load is L_r = pre[(r+1)E_R] - pre[r E_R] and the pairs its
// home experts with a higher id hold are above(e) = pre[(r+1)E_R] - pre[e+1].
// Since the excess X_r is cut from the highest id down, expert e gives
//   take_e = clamp(X_r - above(e), 0, T_e),
// its chunk starts at X_prefix[r] + min(X_r, above(e)) in the excess sequence,
// and its home copy begins min(X_r, above(e) + T_e) - X_r + (pre[e] - pre[r E_R])
// rows after rank r's first row.  Chunk numbers come from one scan of the chunk
// flags in chunk order (ranks ascending, ids descending within a rank).
static __device__ int plan_block(const int32_t* s_loads, int R, int32_t SK, int E, int32_t* __restrict__ plan,
                                 const EpPlanLayout& L, int32_t* work, int32_t* dev_status) {
  __shared__ int4 warp_sums4[32];
  __shared__ int32_t warp_sums[32];
  __shared__ int s_bad;
  const int ER = E / R;
  const int tid = threadIdx.x, nt = blockDim.x;
  int32_t* pre = work;                   // [E + 1] exclusive prefix of T_e, expert order
  int32_t* qf = pre + E + 1;             // [E + 1] chunk flags in chunk order, then their prefix
  int32_t* ch_e = qf + E + 1;            // [E] expert of chunk c
  int32_t* ch_start = ch_e + E;          // [E + 1] chunk start in the excess sequence
  int32_t* ch_first = ch_start + E + 1;  // [E + 1] first match index of chunk c
  int32_t* home = ch_first + E + 1;      // [E] home_count
  int32_t* chunk_of = home + E;          // [E] chunk of expert e or -1
  int32_t* r_X = chunk_of + E;           // [R + 1] exclusive prefix of the excess X_r
  int32_t* r_D = r_X + R + 1;            // [R + 1] exclusive prefix of the deficit D_r
  int32_t* r_di = r_D + R + 1;           // [R + 1] exclusive count of underloaded ranks
  int32_t* df_rank = r_di + R + 1;       // [R] rank of deficit d
  int32_t* df_start = df_rank + R;       // [R + 1] deficit start
  int32_t* df_first = df_start + R + 1;  // [R + 1] first match index of deficit d
  int32_t* df_coinc = df_first + R + 1;  // [R + 1] exclusive count of deficit starts that are chunk starts

  // 1. prefix of the loads
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int e = tid; e < E; e += nt) {
    const int32_t v = s_loads[e];
    pre[e] = v;
    if (v < 0) s_bad = 1;
  }
  __syncthreads();
  const int32_t total = block_scan_inplace(pre, E, warp_sums);
  if (tid == 0) {
    pre[E] = total;
    if (total != R * SK) s_bad = 1;
  }
  __syncthreads();
  const bool bad = s_bad != 0;

  // 2. per-rank excess, deficit, underloaded flag, and their prefixes (one scan)
  const int per = (R + nt - 1) / nt;
  const int rb = min(R, tid * per), re = min(R, rb + per);
  int4 seg = make_int4(0, 0, 0, 0);
  for (int r = rb; r < re; ++r) {
    const int32_t Lr = bad ? SK : pre[(r + 1) * ER] - pre[r * ER];
    const int32_t X = Lr > SK ? Lr - SK : 0, D = Lr < SK ? SK - Lr : 0;
    r_X[r] = X;
    r_D[r] = D;
    r_di[r] = D > 0;
    seg.x += X;
    seg.y += D;
    seg.z += D > 0;
  }
  int4 tot;
  int4 run = block_exclusive_scan4(seg, warp_sums4, &tot);
  for (int r = rb; r < re; ++r) {
    const int3 v = make_int3(r_X[r], r_D[r], r_di[r]);
    r_X[r] = run.x;
    r_D[r] = run.y;
    r_di[r] = run.z;
    run.x += v.x;
    run.y += v.y;
    run.z += v.z;
  }
  if (tid == 0) {
    r_X[R] = tot.x;
    r_D[R] = tot.y;
    r_di[R] = tot.z;
  }
  __syncthreads();
  const int nD = r_di[R];
  const int32_t Xtot = r_X[R];

  // 3. what each expert gives up, and the chunk flags in chunk order
  for (int e = tid; e < E; e += nt) {
    const int r = e / ER, i = e - r * ER;
    const int32_t T_e = bad ? 0 : s_loads[e];
    const int32_t Lr = bad ? SK : pre[(r + 1) * ER] - pre[r * ER];
    const int32_t X = Lr > SK ? Lr - SK : 0;
    const int32_t above = pre[(r + 1) * ER] - pre[e + 1];
    const int32_t take = bad ? 0 : min(max(X - above, 0), T_e);
    home[e] = T_e - take;
    chunk_of[e] = -1;
    qf[r * ER + (ER - 1 - i)] = take > 0;
  }
  __syncthreads();
  const int nC = block_scan_inplace(qf, E, warp_sums);
  for (int e = tid; e < E; e += nt) {
    const int r = e / ER, i = e - r * ER;
    const int32_t T_e = bad ? 0 : s_loads[e];
    const int32_t Lr = bad ? SK : pre[(r + 1) * ER] - pre[r * ER];
    const int32_t X = Lr > SK ? Lr - SK : 0;
    const int32_t above = pre[(r + 1) * ER] - pre[e + 1];
    if (!bad && min(max(X - above, 0), T_e) > 0) {
      const int c = qf[r * ER + (ER - 1 - i)];
      ch_e[c] = e;
      ch_start[c] = r_X[r] + min(X, above);
      chunk_of[e] = c;
    }
  }
  for (int r = tid; r < R; r += nt) {
    const int32_t Lr = bad ? SK : pre[(r + 1) * ER] - pre[r * ER];
    if (Lr < SK) {
      df_rank[r_di[r]] = r;
      df_start[r_di[r]] = r_D[r];
    }
  }
  if (tid == 0) {
    ch_start[nC] = Xtot;
    df_start[nD] = Xtot;
    if (bad) flag(dev_status, EP_DEV_BAD_LOADS);
  }
  __syncthreads();

  // 4. deficit starts that coincide with a chunk start share one breakpoint
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

  // 5. merge-path: one replica per breakpoint, with its slot in buffer order
  int32_t* rep_expert = plan + L.rep_expert;
  int32_t* rep_rank = plan + L.rep_rank;
  int32_t* rep_count = plan + L.rep_count;
  int32_t* rep_begin = plan + L.rep_begin;
  int32_t* rep_base = plan + L.rep_base;
  auto emit = [&](int m, int c, int d, int32_t v) {
    const int32_t end = min(ch_start[c + 1], df_start[d + 1]);
    const int e = ch_e[c];
    const int rr = df_rank[d];
    const int32_t Lrr = pre[(rr + 1) * ER] - pre[rr * ER];
    const int32_t base = rr * SK + Lrr + (v - df_start[d]);  // the receiver is underloaded: its home rows = L_r
    rep_expert[m] = e;
    rep_rank[m] = rr;
    rep_count[m] = end - v;
    rep_begin[m] = home[e] + (v - ch_start[c]);
    rep_base[m] = base;
    plan[L.slot_order + (rr + 1) * ER + m] = E + m;  // after the receiver's home slots and earlier replicas
    plan[L.cu_seqlens + (rr + 1) * ER + m] = base;
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

  // 6. per-expert and per-rank tables, home slots, tails
  for (int e = tid; e < E; e += nt) {
    const int r = e / ER;
    const int c = chunk_of[e];
    plan[L.home_count + e] = home[e];
    plan[L.copy_first + e] = c >= 0 ? ch_first[c] : 0;
    plan[L.copy_cnt + e] = c >= 0 ? ch_first[c + 1] - ch_first[c] : 0;
    plan[L.rep_experts + e] = e < nC ? ch_e[e] : -1;
    int32_t hb = r * SK;
    if (!bad) {
      const int32_t Lr = pre[(r + 1) * ER] - pre[r * ER];
      const int32_t X = Lr > SK ? Lr - SK : 0;
      const int32_t from_e = pre[(r + 1) * ER] - pre[e];  // pairs of ids >= e on rank r
      hb += (pre[e] - pre[r * ER]) - (X - min(X, from_e));
    }
    const int slot = e + df_first[r_di[r]];  // home slots of rank r follow the replicas of ranks < r
    plan[L.home_base + e] = hb;
    plan[L.slot_order + slot] = e;
    plan[L.cu_seqlens + slot] = hb;
  }
  for (int r = tid; r < R; r += nt) {
    const int32_t Lr = bad ? 0 : pre[(r + 1) * ER] - pre[r * ER];
    const int di = r_di[r];
    plan[L.rank_load + r] = Lr;
    plan[L.rank_rep_first + r] = df_first[di];
    plan[L.rank_nrep + r] = (!bad && Lr < SK) ? df_first[di + 1] - df_first[di] : 0;
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
