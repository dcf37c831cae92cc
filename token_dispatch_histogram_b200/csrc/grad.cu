// a7. Replica gradient reduction into the home expert.
//
// [GR] "Τι συμβαίνει στους gradients κατά την εκπαίδευση" (twodots.gr MoonEP
// article): gradients are fp32; the prefetched (replica) slots write into a
// separate reduce buffer, and reduce_grad adds the slots of a rank's own experts
// into its local parameter gradient, then clears the used slots before the next
// micro-batch.  Per element, home first and then the replicas in match order,
// one fp32 add each:  g_home[e] = ((g_home[e] + g_rep[m1]) + g_rep[m2]) + ...
//
// Work = (replicated expert, 8-element vector) items; the replicated experts and
// each one's replica range come from the plan on the device (no host sync).
// A persistent grid walks the items in units of 2048 elements; each thread keeps
// two 32-byte groups of loads in flight per replica step.
#include <algorithm>

#include "common.cuh"

namespace ep {

constexpr int GRAD_THREADS = 256;
constexpr int64_t GRAD_UNIT = GRAD_THREADS * 8;  // elements per work unit

__device__ __forceinline__ void add_bf16x8(float (&a)[8], uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    a[2 * q] = __fadd_rn(a[2 * q], bf16_bits_to_f32(w[q] & 0xFFFFu));
    a[2 * q + 1] = __fadd_rn(a[2 * q + 1], bf16_bits_to_f32(w[q] >> 16));
  }
}

__global__ void __launch_bounds__(GRAD_THREADS)
    k_grad_reduce(float* __restrict__ g_home, void* __restrict__ g_rep, int rep_dtype, int64_t n,
                  const int32_t* __restrict__ plan, EpPlanLayout L, int E, int clear, int32_t* dev_status) {
  const int nC = min(max(plan[L.n_chunks], 0), E);
  const int64_t units_per_expert = (n + GRAD_UNIT - 1) / GRAD_UNIT;
  const int64_t total = (int64_t)nC * units_per_expert;
  const bool vec = (n % 8) == 0;
  for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
    const int c = (int)(u / units_per_expert);
    const int64_t j0 = (u - (int64_t)c * units_per_expert) * GRAD_UNIT;
    const int e = plan[L.rep_experts + c];
    if (e < 0 || e >= E) {
      if (threadIdx.x == 0) flag(dev_status, EP_DEV_BAD_ROW);
      continue;
    }
    const int m0 = plan[L.copy_first + e], mc = plan[L.copy_cnt + e];
    if (m0 < 0 || mc < 0 || m0 + mc > L.cap) {
      if (threadIdx.x == 0) flag(dev_status, EP_DEV_BAD_ROW);
      continue;
    }
    float* home = g_home + (int64_t)e * n;
    if (vec) {
      const int64_t j = j0 + (int64_t)threadIdx.x * 8;
      if (j >= n) continue;
      float a[8];
      const float4 h0 = *reinterpret_cast<const float4*>(home + j);
      const float4 h1 = *reinterpret_cast<const float4*>(home + j + 4);
      a[0] = h0.x; a[1] = h0.y; a[2] = h0.z; a[3] = h0.w;
      a[4] = h1.x; a[5] = h1.y; a[6] = h1.z; a[7] = h1.w;
      for (int m = m0; m < m0 + mc; ++m) {
        if (rep_dtype == EP_DTYPE_F32) {
          const float* r = static_cast<const float*>(g_rep) + (int64_t)m * n + j;
          const uint4 r0 = ld_stream_v4(r), r1 = ld_stream_v4(r + 4);
          a[0] = __fadd_rn(a[0], __uint_as_float(r0.x));
          a[1] = __fadd_rn(a[1], __uint_as_float(r0.y));
          a[2] = __fadd_rn(a[2], __uint_as_float(r0.z));
          a[3] = __fadd_rn(a[3], __uint_as_float(r0.w));
          a[4] = __fadd_rn(a[4], __uint_as_float(r1.x));
          a[5] = __fadd_rn(a[5], __uint_as_float(r1.y));
          a[6] = __fadd_rn(a[6], __uint_as_float(r1.z));
          a[7] = __fadd_rn(a[7], __uint_as_float(r1.w));
          if (clear) {
            st_v4((void*)r, make_uint4(0, 0, 0, 0));
            st_v4((void*)(r + 4), make_uint4(0, 0, 0, 0));
          }
        } else {
          const uint16_t* r = static_cast<const uint16_t*>(g_rep) + (int64_t)m * n + j;
          add_bf16x8(a, ld_stream_v4(r));
          if (clear) st_v4((void*)r, make_uint4(0, 0, 0, 0));
        }
      }
      *reinterpret_cast<float4*>(home + j) = make_float4(a[0], a[1], a[2], a[3]);
      *reinterpret_cast<float4*>(home + j + 4) = make_float4(a[4], a[5], a[6], a[7]);
    } else {
      for (int64_t j = j0 + threadIdx.x; j < min(n, j0 + GRAD_UNIT); j += blockDim.x) {
        float a = home[j];
        for (int m = m0; m < m0 + mc; ++m) {
          if (rep_dtype == EP_DTYPE_F32) {
            float* r = static_cast<float*>(g_rep) + (int64_t)m * n + j;
            a = __fadd_rn(a, *r);
            if (clear) *r = 0.0f;
          } else {
            uint16_t* r = static_cast<uint16_t*>(g_rep) + (int64_t)m * n + j;
            a = __fadd_rn(a, bf16_bits_to_f32(*r));
            if (clear) *r = 0;
          }
        }
        home[j] = a;
      }
    }
  }
}

int occupancy_grid(const void* fn, int threads, size_t smem, int64_t work_items, int cap_per_sm);

}  // namespace ep

using namespace ep;

extern "C" int ep_replica_grad_reduce(float* g_home, const void* g_rep, int rep_dtype, int64_t n, int E, int R,
                                      const int32_t* plan, size_t plan_words, int clear_replicas,
                                      int32_t* dev_status, cudaStream_t stream) {
  if (n < 0 || E < 1 || E > EP_MAX_EXPERTS || R < 1 || R > EP_MAX_RANKS || E % R) return EP_ERR_ARG;
  if (rep_dtype != EP_DTYPE_F32 && rep_dtype != EP_DTYPE_BF16) return EP_ERR_ARG;
  if (!plan) return EP_ERR_ARG;
  EpPlanLayout L;
  plan_layout(E, R, &L);
  if ((int64_t)plan_words < L.words) return EP_ERR_CAPACITY;
  if (n == 0) return EP_OK;
  if (!g_home || !g_rep || !aligned16(g_home) || !aligned16(g_rep)) return EP_ERR_ARG;
  const int64_t units = (int64_t)E * ((n + GRAD_UNIT - 1) / GRAD_UNIT);  // upper bound (n_chunks <= E)
  const int grid = occupancy_grid((const void*)k_grad_reduce, GRAD_THREADS, 0, units, 8);
  k_grad_reduce<<<grid, GRAD_THREADS, 0, stream>>>(g_home, const_cast<void*>(g_rep), rep_dtype, n, plan, L, E,
                                                   clear_replicas, dev_status);
  count_launch();
  return launch_status();
}
