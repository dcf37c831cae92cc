// a7. Replica gradient reduction into the home expert.
//
// [GR] "Τι συμβαίνει στους gradients κατά την εκπαίδευση" (twodots.gr MoonEP
// article): gradients are fp32; the prefetched (replica) slots write into a
// separate reduce buffer, and reduce_grad adds the slots of a rank's own experts
// into its local parameter gradient, then clears the used slots before the next
// micro-batch.  Per element, home first and then the replicas in match order,
// one fp32 add each:  g_home[e] = ((g_home[e] + g_rep[m1]) + g_rep[m2]) + ...
//
// Work = (replicated expert, 4096-element unit) items; the replicated experts
// and each one's replica range come from the plan on the device (no host sync),
// read into shared memory once per CTA (one-buffer form) or once per unit
// (rank-local form, which also stages the unit's replica row addresses).  Each thread owns two 8-element
// vectors of a unit and loads up to four replica vectors before adding them in
// match order, so several 32-byte loads are in flight per thread.
#include <algorithm>

#include "common.cuh"

namespace ep {

constexpr int GRAD_THREADS = 256;
constexpr int GRAD_VECS = 2;                                   // 8-element vectors per thread per unit
constexpr int64_t GRAD_UNIT = (int64_t)GRAD_THREADS * 8 * GRAD_VECS;  // elements per work unit
constexpr int GRAD_BATCH = 4;                                  // replica rows loaded before adding

__device__ __forceinline__ void add_f32x8(float (&a)[8], uint4 lo, uint4 hi) {
  a[0] = __fadd_rn(a[0], __uint_as_float(lo.x));
  a[1] = __fadd_rn(a[1], __uint_as_float(lo.y));
  a[2] = __fadd_rn(a[2], __uint_as_float(lo.z));
  a[3] = __fadd_rn(a[3], __uint_as_float(lo.w));
  a[4] = __fadd_rn(a[4], __uint_as_float(hi.x));
  a[5] = __fadd_rn(a[5], __uint_as_float(hi.y));
  a[6] = __fadd_rn(a[6], __uint_as_float(hi.z));
  a[7] = __fadd_rn(a[7], __uint_as_float(hi.w));
}

__device__ __forceinline__ void add_bf16x8(float (&a)[8], uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    a[2 * q] = __fadd_rn(a[2 * q], bf16_bits_to_f32(w[q] & 0xFFFFu));
    a[2 * q + 1] = __fadd_rn(a[2 * q + 1], bf16_bits_to_f32(w[q] >> 16));
  }
}

// One 8-element vector of one replicated expert: home + replicas m0..m0+mc-1
// in match order.  Up to GRAD_BATCH replica vectors are loaded before any add,
// so their loads overlap; the adds still go in match order.
// rowp(m): base address of replica m's gradient row.
template <bool BF16, bool CLEAR, class RowP>
__device__ __forceinline__ void reduce_vec8(float* __restrict__ home, const RowP& rowp, int64_t j, int m0, int mc) {
  float a[8];
  const float4 h0 = *reinterpret_cast<const float4*>(home + j);
  const float4 h1 = *reinterpret_cast<const float4*>(home + j + 4);
  a[0] = h0.x; a[1] = h0.y; a[2] = h0.z; a[3] = h0.w;
  a[4] = h1.x; a[5] = h1.y; a[6] = h1.z; a[7] = h1.w;
  for (int mb = m0; mb < m0 + mc; mb += GRAD_BATCH) {
    uint4 r[GRAD_BATCH][BF16 ? 1 : 2];
#pragma unroll
    for (int q = 0; q < GRAD_BATCH; ++q) {
      if (mb + q < m0 + mc) {
        if (BF16) {
          r[q][0] = ld_stream_v4(reinterpret_cast<const uint16_t*>(rowp(mb + q)) + j);
        } else {
          const float* rp = reinterpret_cast<const float*>(rowp(mb + q)) + j;
          r[q][0] = ld_stream_v4(rp);
          r[q][BF16 ? 0 : 1] = ld_stream_v4(rp + 4);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < GRAD_BATCH; ++q) {
      if (mb + q < m0 + mc) {
        if (BF16)
          add_bf16x8(a, r[q][0]);
        else
          add_f32x8(a, r[q][0], r[q][BF16 ? 0 : 1]);
        if (CLEAR) {
          if (BF16) {
            st_v4(reinterpret_cast<uint16_t*>(rowp(mb + q)) + j, make_uint4(0, 0, 0, 0));
          } else {
            float* rp = reinterpret_cast<float*>(rowp(mb + q)) + j;
            st_v4(rp, make_uint4(0, 0, 0, 0));
            st_v4(rp + 4, make_uint4(0, 0, 0, 0));
          }
        }
      }
    }
  }
  *reinterpret_cast<float4*>(home + j) = make_float4(a[0], a[1], a[2], a[3]);
  *reinterpret_cast<float4*>(home + j + 4) = make_float4(a[4], a[5], a[6], a[7]);
}

// One unit (GRAD_UNIT elements from j0) of one replicated expert: home row
// `home`, replicas m0 .. m0+mc-1 (rowp(m): replica m's row), in match order.
template <bool BF16, bool CLEAR, class RowP>
__device__ __forceinline__ void reduce_unit(float* __restrict__ home, const RowP& rowp, int64_t n, int64_t j0, int m0,
                                            int mc, bool vec) {
  if (vec) {
#pragma unroll
    for (int vv = 0; vv < GRAD_VECS; ++vv) {
      const int64_t j = j0 + ((int64_t)vv * GRAD_THREADS + threadIdx.x) * 8;
      if (j >= n) break;
      reduce_vec8<BF16, CLEAR>(home, rowp, j, m0, mc);
    }
    return;
  }
  for (int64_t j = j0 + threadIdx.x; j < min(n, j0 + GRAD_UNIT); j += blockDim.x) {
    float a = home[j];
    for (int m = m0; m < m0 + mc; ++m) {
      if (!BF16) {
        float* r = reinterpret_cast<float*>(rowp(m)) + j;
        a = __fadd_rn(a, *r);
        if (CLEAR) *r = 0.0f;
      } else {
        uint16_t* r = reinterpret_cast<uint16_t*>(rowp(m)) + j;
        a = __fadd_rn(a, bf16_bits_to_f32(*r));
        if (CLEAR) *r = 0;
      }
    }
    home[j] = a;
  }
}

// PEER (rank-local form): only the experts homed on `rank` are reduced, into
// g_home [E/R, n]; replica m's row is row m - rank_rep_first[d] of the buffer
// at peers[d], d = rep_rank[m] (a rank's replicas are consecutive in match
// order).  The unit's replica row addresses are staged in shared memory.
template <bool BF16, bool CLEAR, bool PEER>
__global__ void __launch_bounds__(GRAD_THREADS, 4)
    k_grad_reduce(float* __restrict__ g_home, void* __restrict__ g_rep, int64_t n, const int32_t* __restrict__ plan,
                  EpPlanLayout L, int E, const uint64_t* __restrict__ peers, int R, int rank, int64_t rep_rows,
                  int32_t* dev_status) {
  __shared__ int s_e, s_m0, s_mc;
  __shared__ char* s_rows[PEER ? EP_MAX_RANKS : 1];
  wait_for_predecessor();
  const int ER = E / R;
  const int nC = min(max(plan[L.n_chunks], 0), E);
  const int64_t units_per_expert = (n + GRAD_UNIT - 1) / GRAD_UNIT;
  const int64_t total = (int64_t)nC * units_per_expert;
  const bool vec = (n % 8) == 0;
  if (!PEER && vec) {
    // one-buffer form, rows of 8-element vectors: every replicated expert's
    // (e, first replica, replica count) read once into shared memory, so a
    // unit starts without a dependent plan lookup or a block barrier (on B200:
    // 1% faster with fp32 replica rows, 4% with bf16 ones, than looking them
    // up per unit)
    __shared__ int s_tab[PEER ? 1 : 3 * EP_MAX_EXPERTS];
    for (int c = threadIdx.x; c < nC; c += blockDim.x) {
      const int e = plan[L.rep_experts + c];
      int m0 = 0, mc = 0;
      if (e >= 0 && e < E) {
        m0 = plan[L.copy_first + e];
        mc = plan[L.copy_cnt + e];
      }
      const bool bad = e < 0 || e >= E || m0 < 0 || mc < 0 || m0 + mc > L.cap;
      if (bad) flag(dev_status, EP_DEV_BAD_ROW);
      s_tab[3 * c] = bad ? -1 : e;
      s_tab[3 * c + 1] = m0;
      s_tab[3 * c + 2] = mc;
    }
    __syncthreads();
    const int64_t esz = BF16 ? 2 : 4;
    auto rowp = [&](int m) -> char* { return static_cast<char*>(g_rep) + (int64_t)m * n * esz; };
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
      const int c = (int)(u / units_per_expert);
      const int64_t j0 = (u - (int64_t)c * units_per_expert) * GRAD_UNIT;
      const int e = s_tab[3 * c];
      if (e < 0) continue;
      float* home = g_home + (int64_t)e * n;
      const int m0 = s_tab[3 * c + 1], mc = s_tab[3 * c + 2];
#pragma unroll
      for (int vv = 0; vv < GRAD_VECS; ++vv) {
        const int64_t j = j0 + ((int64_t)vv * GRAD_THREADS + threadIdx.x) * 8;
        if (j >= n) break;
        reduce_vec8<BF16, CLEAR>(home, rowp, j, m0, mc);
      }
    }
  } else {
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
      const int c = (int)(u / units_per_expert);
      const int64_t j0 = (u - (int64_t)c * units_per_expert) * GRAD_UNIT;
      __syncthreads();  // the previous unit is done with s_e, s_m0, s_mc
      if (threadIdx.x == 0) {
        const int e = plan[L.rep_experts + c];
        int m0 = 0, mc = 0;
        if (e >= 0 && e < E) {
          m0 = plan[L.copy_first + e];
          mc = plan[L.copy_cnt + e];
        }
        if (e < 0 || e >= E || m0 < 0 || mc < 0 || m0 + mc > L.cap || (PEER && mc > EP_MAX_RANKS)) {
          flag(dev_status, EP_DEV_BAD_ROW);
          s_e = -1;
        } else if (PEER && e / ER != rank) {
          s_e = -1;  // another rank's expert
        } else {
          s_e = e;
          s_m0 = m0;
          s_mc = mc;
        }
      }
      __syncthreads();
      const int e = s_e;
      if (e < 0) continue;
      const int m0 = s_m0, mc = s_mc;
      const int64_t esz = BF16 ? 2 : 4;
      if (PEER) {
        for (int q = threadIdx.x; q < mc; q += blockDim.x) {
          const int m = m0 + q;
          const int d = plan[L.rep_rank + m];
          char* base = nullptr;
          if (d >= 0 && d < R) {
            const int64_t j = m - plan[L.rank_rep_first + d];
            const uint64_t pb = __ldg(peers + d);
            if (pb && !(pb & 15u) && j >= 0 && j < rep_rows) base = reinterpret_cast<char*>(pb) + j * n * esz;
          }
          if (!base) flag(dev_status, EP_DEV_BAD_ROW);
          s_rows[PEER ? q : 0] = base;
        }
        __syncthreads();
        bool ok = true;
        for (int q = 0; q < mc; ++q) ok = ok && s_rows[PEER ? q : 0] != nullptr;
        if (!ok) continue;  // every thread saw the same table: skip the unit together
      }
      auto rowp = [&](int m) -> char* {
        return PEER ? s_rows[PEER ? m - m0 : 0] : static_cast<char*>(g_rep) + (int64_t)m * n * esz;
      };
      reduce_unit<BF16, CLEAR>(g_home + (int64_t)(PEER ? e - rank * ER : e) * n, rowp, n, j0, m0, mc, vec);
    }
  }
}

int occupancy_grid(const void* fn, int threads, size_t smem, int64_t work_items, int cap_per_sm);

}  // namespace ep

using namespace ep;

namespace ep {
void quota_layout(int E, int R, EpQuotaLayout* L);

// The plan fields the reduction reads: replicated experts in match order, and
// each expert's first replica and replica count.
template <bool PEER>
static const void* grad_fn(int rep_dtype, int clear) {
  if (rep_dtype == EP_DTYPE_F32)
    return clear ? (const void*)k_grad_reduce<false, true, PEER> : (const void*)k_grad_reduce<false, false, PEER>;
  return clear ? (const void*)k_grad_reduce<true, true, PEER> : (const void*)k_grad_reduce<true, false, PEER>;
}

// The fields of a quota plan the reduction reads, under the names of the
// exact-S*K plan's layout.
static EpPlanLayout grad_view(const EpQuotaLayout& Q) {
  EpPlanLayout L{};
  L.words = Q.words;
  L.cap = Q.cap;
  L.n_chunks = Q.n_chunks;
  L.rep_experts = Q.rep_experts;
  L.copy_first = Q.rep_first;
  L.copy_cnt = Q.rep_cnt;
  L.rep_rank = Q.rep_rank;
  L.rank_rep_first = Q.rank_rep_first;
  return L;
}

// peers == NULL: g_home [E, n], g_rep [cap, n] (row m = replica m).  Else the
// rank-local form for `rank` (g_home [E/R, n], replica rows behind peers).
static int run_grad_reduce(float* g_home, const void* g_rep, int rep_dtype, int64_t n, int E, const int32_t* plan,
                           EpPlanLayout L, int clear_replicas, const uint64_t* peers, int R, int rank,
                           int64_t rep_rows, int32_t* dev_status, cudaStream_t stream) {
  if (n == 0) return EP_OK;
  if (!g_home || !aligned16(g_home)) return EP_ERR_ARG;
  if (!peers && (!g_rep || !aligned16(g_rep))) return EP_ERR_ARG;
  const int64_t units = (int64_t)E * ((n + GRAD_UNIT - 1) / GRAD_UNIT);  // upper bound (n_chunks <= E)
  // 4 CTAs per SM measured best
  const void* fn = peers ? grad_fn<true>(rep_dtype, clear_replicas) : grad_fn<false>(rep_dtype, clear_replicas);
  const int grid = occupancy_grid(fn, GRAD_THREADS, 0, units, 4);
  void* gr = const_cast<void*>(g_rep);
  void* args[] = {(void*)&g_home, (void*)&gr,    (void*)&n, (void*)&plan, (void*)&L,         (void*)&E,
                  (void*)&peers,  (void*)&R,     (void*)&rank, (void*)&rep_rows, (void*)&dev_status};
  if (launch_pdl(fn, dim3(grid), dim3(GRAD_THREADS), args, 0, stream) != cudaSuccess) return EP_ERR_CUDA;
  count_launch();
  return launch_status();
}
}  // namespace ep

extern "C" int ep_replica_grad_reduce(float* g_home, const void* g_rep, int rep_dtype, int64_t n, int E, int R,
                                      const int32_t* plan, size_t plan_words, int clear_replicas,
                                      int32_t* dev_status, cudaStream_t stream) {
  if (n < 0 || E < 1 || E > EP_MAX_EXPERTS || R < 1 || R > EP_MAX_RANKS || E % R) return EP_ERR_ARG;
  if (rep_dtype != EP_DTYPE_F32 && rep_dtype != EP_DTYPE_BF16) return EP_ERR_ARG;
  if (!plan) return EP_ERR_ARG;
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  return run_grad_reduce(g_home, g_rep, rep_dtype, n, E, plan, L, clear_replicas, nullptr, R, 0, 0, dev_status, stream);
}

extern "C" int ep_replica_grad_reduce_peer(float* g_home_local, const uint64_t* peer_g_rep, int64_t rep_rows,
                                           int rep_dtype, int64_t n, int E, int R, int rank, const int32_t* plan,
                                           size_t plan_words, int clear_replicas, int32_t* dev_status,
                                           cudaStream_t stream) {
  if (n < 0 || E < 1 || E > EP_MAX_EXPERTS || R < 1 || R > EP_MAX_RANKS || E % R || rank < 0 || rank >= R ||
      rep_rows < 0)
    return EP_ERR_ARG;
  if (rep_dtype != EP_DTYPE_F32 && rep_dtype != EP_DTYPE_BF16) return EP_ERR_ARG;
  if (!plan || !peer_g_rep) return EP_ERR_ARG;
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  return run_grad_reduce(g_home_local, nullptr, rep_dtype, n, E, plan, L, clear_replicas, peer_g_rep, R, rank,
                         rep_rows, dev_status, stream);
}

extern "C" int ep_quota_replica_grad_reduce_peer(float* g_home_local, const uint64_t* peer_g_rep, int64_t rep_rows,
                                                 int rep_dtype, int64_t n, int E, int R, int rank, const int32_t* plan,
                                                 size_t plan_words, int clear_replicas, int32_t* dev_status,
                                                 cudaStream_t stream) {
  if (n < 0 || E < 1 || E > EP_MAX_EXPERTS || R < 1 || R > EP_MAX_RANKS || E % R || rank < 0 || rank >= R ||
      rep_rows < 0)
    return EP_ERR_ARG;
  if (rep_dtype != EP_DTYPE_F32 && rep_dtype != EP_DTYPE_BF16) return EP_ERR_ARG;
  if (!plan || !peer_g_rep) return EP_ERR_ARG;
  EpQuotaLayout Q;
  quota_layout(E, R, &Q);
  if ((int64_t)plan_words < Q.words) return EP_ERR_CAPACITY;
  const EpPlanLayout L = grad_view(Q);
  return run_grad_reduce(g_home_local, nullptr, rep_dtype, n, E, plan, L, clear_replicas, peer_g_rep, R, rank,
                         rep_rows, dev_status, stream);
}

extern "C" int ep_quota_replica_grad_reduce(float* g_home, const void* g_rep, int rep_dtype, int64_t n, int E, int R,
                                            const int32_t* plan, size_t plan_words, int clear_replicas,
                                            int32_t* dev_status, cudaStream_t stream) {
  if (n < 0 || E < 1 || E > EP_MAX_EXPERTS || R < 1 || R > EP_MAX_RANKS || E % R) return EP_ERR_ARG;
  if (rep_dtype != EP_DTYPE_F32 && rep_dtype != EP_DTYPE_BF16) return EP_ERR_ARG;
  if (!plan) return EP_ERR_ARG;
  EpQuotaLayout Q;
  quota_layout(E, R, &Q);
  if ((int64_t)plan_words < Q.words) return EP_ERR_CAPACITY;
  const EpPlanLayout L = grad_view(Q);
  return run_grad_reduce(g_home, g_rep, rep_dtype, n, E, plan, L, clear_replicas, nullptr, R, 0, 0, dev_status, stream);
}
