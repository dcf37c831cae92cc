// a2. Replica plan: every rank ends with exactly S*K routed pairs.
//
// [GR] "Η βασική υπόσχεση του MoonEP: σταθερό φορτίο S × K" (twodots.gr MoonEP
// article): each rank receives exactly S*K pairs however skewed the router, by
// a handful of temporary expert copies planned online from the current router
// output, on the GPU ([GR] "Online planning, zero copy και στατικά σχήματα").
// [JA] "その仕組みは高速なエキスパート複製に依存する" (remio.ai UltraEP
// article): one decision gives which hot experts get copies, where they run and
// how many tokens each instance takes, computed entirely on the GPU.
//
// Rule (this library's deterministic reading; the pages do not print one):
//  - expert e is homed on rank floor(e / E_R); rank load L_r;
//  - an overloaded rank's excess X_r = L_r - S*K is cut into chunks from its
//    home experts in descending id, chunk = min(T_e, excess left);
//  - underloaded ranks' deficits D_r = S*K - L_r are taken in ascending rank;
//  - the chunks' prefix sums and the deficits' prefix sums (both over the same
//    total) are merged: every interval between consecutive breakpoints of the
//    union is one replica (expert of the chunk covering it, rank of the deficit
//    covering it, interval length).  Replicas are numbered in breakpoint order,
//    the "match order".
//
// One CTA of 1024 threads: one thread per rank for the per-rank walks (at most
// E_R steps each), block scans for the prefix sums, and a merge-path over the
// two sorted breakpoint lists: each breakpoint finds its merged position by
// binary search in the other list, so every replica is emitted independently.
#include "common.cuh"

namespace ep {

constexpr int PLAN_THREADS = 1024;

__device__ __forceinline__ int lower_bound_i32(const int32_t* a, int n, int32_t v) {
  int lo = 0, hi = n;  // first i with a[i] >= v
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
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
    int mid = (lo + hi) >> 1;
    if (a[mid] <= v)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(PLAN_THREADS)
    k_plan(const int32_t* __restrict__ loads, int R, int32_t SK, int E, int32_t* __restrict__ plan, EpPlanLayout L,
           int32_t* dev_status) {
  extern __shared__ int32_t sm[];
  const int ER = E / R;
  // shared arrays
  int32_t* s_loads = sm;                  // [E]
  int32_t* s_chunk_of = s_loads + E;      // [E] chunk index of e or -1
  int32_t* s_home = s_chunk_of + E;       // [E] home_count
  int32_t* ch_e = s_home + E;             // [E] chunk expert
  int32_t* ch_start = ch_e + E;           // [E + 1] chunk start in the excess sequence
  int32_t* ch_first = ch_start + E + 1;   // [E + 1] first match index of the chunk
  int32_t* df_rank = ch_first + E + 1;    // [R]
  int32_t* df_start = df_rank + R;        // [R + 1]
  int32_t* df_first = df_start + R + 1;   // [R + 1]
  int32_t* df_coinc = df_first + R + 1;   // [R + 1] exclusive count of deficit starts that are chunk starts
  int32_t* r_load = df_coinc + R + 1;     // [R]
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t s_nC, s_nD, s_ncoinc;
  __shared__ unsigned long long s_sum;
  __shared__ int s_bad;

  const int tid = threadIdx.x;
  if (tid == 0) {
    s_sum = 0;
    s_bad = 0;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int32_t v = loads[e];
    s_loads[e] = v;
    s_chunk_of[e] = -1;
    if (v < 0) s_bad = 1;
    atomicAdd(&s_sum, (unsigned long long)(int64_t)v);
  }
  __syncthreads();
  const bool bad = s_bad || (int64_t)s_sum != (int64_t)R * SK;

  // per-rank loads, excess/deficit, chunk counts (thread r owns rank r; R <= 1024)
  const int r = tid;
  int32_t Lr = 0, Xr = 0, Dr = 0, nch = 0;
  if (r < R && !bad) {
    for (int e = r * ER; e < (r + 1) * ER; ++e) Lr += s_loads[e];
    Xr = Lr > SK ? Lr - SK : 0;
    Dr = Lr < SK ? SK - Lr : 0;
    int32_t rem = Xr;
    for (int e = (r + 1) * ER - 1; e >= r * ER && rem > 0; --e) {
      const int32_t take = min(s_loads[e], rem);
      if (take > 0) {
        ++nch;
        rem -= take;
      }
    }
    r_load[r] = Lr;
  }
  int32_t Xtot, Dtot, nC, nD;
  const int32_t X_pref = block_exclusive_scan(Xr, warp_sums, &Xtot);
  const int32_t D_pref = block_exclusive_scan(Dr, warp_sums, &Dtot);
  const int32_t ch_off = block_exclusive_scan(nch, warp_sums, &nC);
  const int32_t df_off = block_exclusive_scan(Dr > 0 ? 1 : 0, warp_sums, &nD);

  // chunks of rank r (descending id), deficits, home counts
  if (r < R && !bad) {
    for (int e = r * ER; e < (r + 1) * ER; ++e) s_home[e] = s_loads[e];
    int32_t rem = Xr, start = X_pref, c = ch_off;
    for (int e = (r + 1) * ER - 1; e >= r * ER && rem > 0; --e) {
      const int32_t take = min(s_loads[e], rem);
      if (take > 0) {
        ch_e[c] = e;
        ch_start[c] = start;
        s_chunk_of[e] = c;
        s_home[e] = s_loads[e] - take;
        start += take;
        rem -= take;
        ++c;
      }
    }
    if (Dr > 0) {
      df_rank[df_off] = r;
      df_start[df_off] = D_pref;
    }
  }
  if (tid == 0) {
    s_nC = bad ? 0 : nC;
    s_nD = bad ? 0 : nD;
    ch_start[bad ? 0 : nC] = Xtot;
    df_start[bad ? 0 : nD] = Xtot;
    if (bad) flag(dev_status, EP_DEV_BAD_LOADS);
  }
  __syncthreads();
  nC = s_nC;
  nD = s_nD;

  // which deficit starts coincide with a chunk start (they share one breakpoint)
  int32_t coinc = 0;
  if (tid < nD) {
    const int32_t v = df_start[tid];
    const int i = lower_bound_i32(ch_start, nC, v);
    coinc = (i < nC && ch_start[i] == v) ? 1 : 0;
  }
  int32_t ncoinc;
  const int32_t coinc_pref = block_exclusive_scan(coinc, warp_sums, &ncoinc);
  if (tid < nD) df_coinc[tid] = coinc_pref;
  if (tid == 0) {
    df_coinc[nD] = ncoinc;
    s_ncoinc = ncoinc;
  }
  __syncthreads();
  const int32_t n_rep = nC + nD - s_ncoinc;

  int32_t* rep_expert = plan + L.rep_expert;
  int32_t* rep_rank = plan + L.rep_rank;
  int32_t* rep_count = plan + L.rep_count;
  int32_t* rep_begin = plan + L.rep_begin;
  int32_t* rep_base = plan + L.rep_base;

  // emit one replica for the interval [v, end) covered by chunk c and deficit d
  auto emit = [&](int m, int c, int d, int32_t v) {
    const int32_t end = min(ch_start[c + 1], df_start[d + 1]);
    const int e = ch_e[c];
    const int rr = df_rank[d];
    rep_expert[m] = e;
    rep_rank[m] = rr;
    rep_count[m] = end - v;
    rep_begin[m] = s_home[e] + (v - ch_start[c]);
    rep_base[m] = rr * SK + r_load[rr] + (v - df_start[d]);  // receiver is underloaded: its home rows = L_r
  };
  // chunk breakpoints: merged index = chunks before + distinct deficit starts before
  for (int c = tid; c < nC; c += blockDim.x) {
    const int32_t v = ch_start[c];
    const int dl = lower_bound_i32(df_start, nD, v);
    const int m = c + dl - df_coinc[dl];
    const int d = upper_bound_i32(df_start, nD, v) - 1;
    ch_first[c] = m;
    if (df_start[d] == v) df_first[d] = m;
    emit(m, c, d, v);
  }
  // deficit breakpoints that are not also chunk breakpoints
  for (int d = tid; d < nD; d += blockDim.x) {
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

  // per-expert tables
  for (int e = tid; e < E; e += blockDim.x) {
    const int c = s_chunk_of[e];
    plan[L.home_count + e] = bad ? 0 : s_home[e];
    plan[L.copy_first + e] = c >= 0 ? ch_first[c] : 0;
    plan[L.copy_cnt + e] = c >= 0 ? ch_first[c + 1] - ch_first[c] : 0;
    plan[L.rep_experts + e] = e < nC ? ch_e[e] : -1;
  }
  // per-rank tables, home rows, slot order and cu_seqlens
  if (r < R) {
    const int32_t first = bad ? 0 : df_first[df_off];
    const int32_t nrecv = (bad || Dr == 0) ? 0 : df_first[df_off + 1] - df_first[df_off];
    plan[L.rank_load + r] = bad ? 0 : Lr;
    plan[L.rank_rep_first + r] = first;
    plan[L.rank_nrep + r] = nrecv;
    int32_t row = r * SK;
    const int sbase = r * ER + first;
    for (int i = 0; i < ER; ++i) {
      const int e = r * ER + i;
      plan[L.home_base + e] = row;
      plan[L.slot_order + sbase + i] = e;
      plan[L.cu_seqlens + sbase + i] = row;
      row += bad ? 0 : s_home[e];
    }
    for (int j = 0; j < nrecv; ++j) {
      const int m = first + j;
      plan[L.slot_order + sbase + ER + j] = E + m;
      plan[L.cu_seqlens + sbase + ER + j] = rep_base[m];
    }
  }
  // tails
  for (int i = E + n_rep + tid; i <= E + L.cap; i += blockDim.x) {
    plan[L.cu_seqlens + i] = R * SK;
    if (i < E + L.cap) plan[L.slot_order + i] = -1;
  }
  for (int m = n_rep + tid; m < L.cap; m += blockDim.x) {
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
}

void plan_layout(int E, int R, EpPlanLayout* L) {
  const int cap = E + R - 1;
  int32_t o = 0;
  auto take = [&](int32_t n) {
    const int32_t at = o;
    o += (n + 7) & ~7;  // keep every array 32-byte aligned
    return at;
  };
  L->cap = cap;
  L->n_rep = take(1);
  L->n_chunks = take(1);
  L->rank_load = take(R);
  L->rank_nrep = take(R);
  L->rank_rep_first = take(R);
  L->home_count = take(E);
  L->home_base = take(E);
  L->copy_first = take(E);
  L->copy_cnt = take(E);
  L->rep_expert = take(cap);
  L->rep_rank = take(cap);
  L->rep_count = take(cap);
  L->rep_begin = take(cap);
  L->rep_base = take(cap);
  L->rep_experts = take(E);
  L->slot_order = take(E + cap);
  L->cu_seqlens = take(E + cap + 1);
  L->words = o;
}

size_t plan_smem_bytes(int E, int R) { return sizeof(int32_t) * (size_t)(6 * E + 2 + 5 * R + 3); }

}  // namespace ep

using namespace ep;

extern "C" int ep_plan_layout(int E, int R, EpPlanLayout* layout) {
  if (!layout || E < 1 || R < 1 || E > EP_MAX_EXPERTS || R > EP_MAX_RANKS || E % R) return EP_ERR_ARG;
  plan_layout(E, R, layout);
  return EP_OK;
}

extern "C" int ep_plan(const int32_t* loads, int R, int64_t S, int K, int E, int32_t* plan, size_t plan_words,
                       int32_t* dev_status, cudaStream_t stream) {
  if (!loads || !plan || R < 1 || R > EP_MAX_RANKS || E < 1 || E > EP_MAX_EXPERTS || E % R || K < 1 || S < 0)
    return EP_ERR_ARG;
  if ((int64_t)R * S * K >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  const size_t smem = plan_smem_bytes(E, R);  // <= 45 KB at the limits: no opt-in needed
  k_plan<<<1, PLAN_THREADS, smem, stream>>>(loads, R, (int32_t)(S * K), E, plan, L, dev_status);
  count_launch();
  return launch_status();
}
