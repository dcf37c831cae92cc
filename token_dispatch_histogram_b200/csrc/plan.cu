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
// One CTA of 1024 threads runs the block-level planner of plan_block.cuh
// (per-rank walks, one four-way block scan, a merge-path over the two sorted
// breakpoint lists); the fused route kernel runs the same planner.
#include "plan_block.cuh"

namespace ep {

constexpr int PLAN_THREADS = 1024;

__global__ void __launch_bounds__(PLAN_THREADS)
    k_plan(const int32_t* __restrict__ loads, int R, int32_t SK, int E, int32_t* __restrict__ plan, EpPlanLayout L,
           int32_t* dev_status) {
  extern __shared__ int32_t sm[];
  int32_t* s_loads = sm;       // [E]
  int32_t* work = sm + E;      // plan_work_words(E, R)
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_loads[e] = loads[e];
  __syncthreads();
  plan_block(s_loads, R, SK, E, plan, L, work, dev_status);
}

// The plan from the gathered [R, E] load matrix (rank-local form): the column
// sums are the loads, then the same block planner.  A column sum outside int32
// range becomes -1, which the planner rejects as invalid loads.
__global__ void __launch_bounds__(PLAN_THREADS)
    k_plan_counts(const int32_t* __restrict__ counts, int R, int32_t SK, int E, int32_t* __restrict__ loads,
                  int32_t* __restrict__ plan, EpPlanLayout L, int32_t* dev_status) {
  extern __shared__ int32_t sm[];
  int32_t* s_loads = sm;       // [E]
  int32_t* work = sm + E;      // plan_work_words(E, R)
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int64_t t = 0;
    bool ok = true;
    for (int r = 0; r < R; ++r) {
      const int32_t c = counts[(int64_t)r * E + e];
      ok = ok && c >= 0;
      t += c;
    }
    const int32_t v = (ok && t <= INT32_MAX) ? (int32_t)t : -1;
    s_loads[e] = v;
    if (loads) loads[e] = v;
  }
  __syncthreads();
  plan_block(s_loads, R, SK, E, plan, L, work, dev_status);
}

// Prefetch slots under a per-rank budget B: replica m is the j-th replica its
// rank receives, j = m - rank_rep_first[rank] (replicas of a rank are
// consecutive in match order); it gets weight row E + j while j < B, else -1
// (its weights are read from the home rank).  With load_capped, also the rank
// loads when a slotless replica's pairs stay with the expert's home rank:
// integer atomics in shared memory, so the sums do not depend on their order.
// One CTA: cap = E + R - 1 < 2048.
__global__ void __launch_bounds__(1024)
    k_prefetch_slots(const int32_t* __restrict__ plan, EpPlanLayout L, int E, int R, int64_t SK, int B,
                     int32_t* __restrict__ slot, int32_t* __restrict__ n_remote, int64_t* __restrict__ load_capped) {
  __shared__ unsigned long long s_load[EP_MAX_RANKS];
  const int ER = E / R;
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    s_load[r] = (unsigned long long)SK;
    n_remote[r] = max(0, plan[L.rank_nrep + r] - B);
  }
  __syncthreads();
  const int n_rep = min(max(plan[L.n_rep], 0), L.cap);
  for (int m = threadIdx.x; m < L.cap; m += blockDim.x) {
    int32_t s = -1;
    if (m < n_rep) {
      const int r = plan[L.rep_rank + m];
      const int e = plan[L.rep_expert + m];
      if (r >= 0 && r < R && e >= 0 && e < E) {
        const int j = m - plan[L.rank_rep_first + r];
        if (j >= 0 && j < B) {
          s = E + j;
        } else if (load_capped) {
          const unsigned long long c = (unsigned long long)(int64_t)plan[L.rep_count + m];
          atomicAdd(&s_load[r], 0ull - c);
          atomicAdd(&s_load[e / ER], c);
        }
      }
    }
    slot[m] = s;
  }
  if (!load_capped) return;
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x) load_capped[r] = (int64_t)s_load[r];
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

size_t plan_smem_bytes(int E, int R) { return sizeof(int32_t) * (size_t)(E + plan_work_words(E, R)); }

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
  const size_t smem = plan_smem_bytes(E, R);  // <= 61 KB at the limits
  if (smem > 48 * 1024 &&
      !raise_smem_limit((const void*)k_plan, smem))
    return EP_ERR_CUDA;
  k_plan<<<1, PLAN_THREADS, smem, stream>>>(loads, R, (int32_t)(S * K), E, plan, L, dev_status);
  count_launch();
  return launch_status();
}

extern "C" int ep_plan_from_counts(const int32_t* counts, int R, int64_t S, int K, int E, int32_t* loads,
                                   int32_t* plan, size_t plan_words, int32_t* dev_status, cudaStream_t stream) {
  if (!counts || !plan || R < 1 || R > EP_MAX_RANKS || E < 1 || E > EP_MAX_EXPERTS || E % R || K < 1 || S < 0)
    return EP_ERR_ARG;
  if ((int64_t)R * S * K >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  const size_t smem = plan_smem_bytes(E, R);
  if (smem > 48 * 1024 &&
      !raise_smem_limit((const void*)k_plan_counts, smem))
    return EP_ERR_CUDA;
  k_plan_counts<<<1, PLAN_THREADS, smem, stream>>>(counts, R, (int32_t)(S * K), E, loads, plan, L, dev_status);
  count_launch();
  return launch_status();
}

extern "C" int ep_prefetch_slots(const int32_t* plan, size_t plan_words, int E, int R, int64_t SK, int B,
                                 int32_t* slot, int32_t* n_remote, int64_t* load_capped, cudaStream_t stream) {
  if (!plan || !slot || !n_remote || R < 1 || R > EP_MAX_RANKS || E < 1 || E > EP_MAX_EXPERTS || E % R || B < 0 ||
      SK < 0)
    return EP_ERR_ARG;
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  k_prefetch_slots<<<1, 1024, 0, stream>>>(plan, L, E, R, SK, B, slot, n_remote, load_capped);
  count_launch();
  return launch_status();
}
