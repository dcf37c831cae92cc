// a5. Dispatch and a6. Combine: the HBM-bound row movers.
//
// Dispatch ([GR] "Online planning, zero copy και στατικά σχήματα", twodots.gr
// MoonEP article): each token's hidden row is written straight into the K rows
// the layout gave its pairs, in the static expert-grouped buffer.
// buf[pos[t*K + k]] = x[t] for k < K.  Minimal traffic: each x row is read once
// (T*H*2 bytes) and each buffer row written once (P*H*2 bytes).
//
// B200 design: one-warp CTAs, each owning DISPATCH_TOKENS_PER_CTA consecutive
// tokens, with a ring of shared-memory stages.  Lane 0 brings a whole row in
// with one TMA bulk copy (cp.async.bulk global->shared, completion on an
// mbarrier); once it lands, lanes 0..K-1 each issue one bulk store
// (shared->global) of that row to one destination.  The grid has one CTA per
// pair of tokens (not a persistent grid), and each CTA reserves enough shared
// memory that only as many fit an SM as keep about 32 KB of row loads in flight
// per SM, which measured fastest.  Measured on B200 against a persistent
// grid-stride grid of the same residency: 5-14% faster alone (the block
// scheduler keeps the tokens in flight close together and balances the tail),
// and it shares the GPU gracefully: next to an unrelated kernel on another
// stream, the persistent grid took 2-4x its time (its late-starting CTAs still
// owned a full share of tokens), this one the sum of the two.  The stores carry
// an L2 evict-first policy: each buffer row is written once (1-2% faster for
// 15-17 GB dispatch buffers, the same for a 0.8 GB one).
//
// Rank-local form (PEER = true): the R ranks' buffers are separate allocations,
// possibly on other GPUs, reached through a device table of R base pointers;
// global row `row` lives at peers[row / rows_per_rank] + (row % rows_per_rank)
// rows.  Dispatch then writes each row straight into the receiving rank's
// buffer and combine reads it back from there; nothing else changes.
//
// Combine: out[t] = bf16_rn(sum_k w[t,k] * float(y[pos[t*K+k]])), fp32 in k
// order, separate multiply and add roundings (no FMA).  One thread owns 8
// consecutive bf16 of one output row (one 16-byte vector); it issues all K
// 16-byte row loads before using any, so K loads are in flight per thread,
// with the token's row indices and weights already staged in shared memory.
#include <algorithm>

#include "common.cuh"

namespace ep {

constexpr int DISPATCH_MAX_STAGES = 8;
constexpr int DISPATCH_TOKENS_PER_CTA = 2;  // 1, 4 and 8 measured slower on B200
constexpr int COMBINE_ITERS = 4;  // token iterations per combine CTA (1-3 measured slower at 0.9 GB)

template <bool PEER>
__global__ void __launch_bounds__(32)
    k_dispatch(const uint8_t* __restrict__ x, int64_t T, int K, uint32_t row_bytes, const int32_t* __restrict__ pos,
               int64_t buf_rows, uint8_t* __restrict__ buf, const uint64_t* __restrict__ peers,
               const int32_t* __restrict__ rank_first, int R, int64_t rows_per_rank, int stages,
               int32_t* dev_status) {
  extern __shared__ __align__(128) uint8_t smem[];
  wait_for_predecessor();
  const uint32_t stride_b = (row_bytes + 127u) & ~127u;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)stages * stride_b);
  int32_t* ring = reinterpret_cast<int32_t*>(bars + DISPATCH_MAX_STAGES);  // [stages][K] destination rows
  const int lane = threadIdx.x;
  const uint64_t evict_first = l2_evict_first_policy();  // each buffer row is written once
  if (lane == 0)
    for (int s = 0; s < stages; ++s) mbar_init(&bars[s], 1);
  fence_mbar_init();
  __syncwarp();

  const int64_t first = (int64_t)blockIdx.x * DISPATCH_TOKENS_PER_CTA;
  const int64_t njobs = first < T ? min((int64_t)DISPATCH_TOKENS_PER_CTA, T - first) : 0;
  auto issue = [&](int64_t j) {
    const int s = (int)(j % stages);
    const int64_t t = first + j;
    if (lane < K) ring[s * K + lane] = __ldg(pos + t * K + lane);
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[s], row_bytes);
      bulk_load(smem + (size_t)s * stride_b, x + t * (int64_t)row_bytes, row_bytes, &bars[s]);
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
      if (row >= 0 && row < buf_rows) {
        uint8_t* dst;
        if (PEER) {  // a missing or misaligned rank buffer, or a row past it, is reported, never written
          dst = reinterpret_cast<uint8_t*>(peer_row(peers, rank_first, R, rows_per_rank, row, row_bytes));
        } else {
          dst = buf + (int64_t)row * row_bytes;
        }
        if (dst)
          bulk_store_hint(dst, smem + (size_t)s * stride_b, row_bytes, evict_first);
        else
          bad = EP_DEV_BAD_ROW;
      } else
        bad = EP_DEV_BAD_ROW;
    }
    bulk_commit();
    // refill the previous job's stage once its stores have read shared memory
    if (j >= 1 && issued < njobs) {
      bulk_wait_read<1>();
      __syncwarp();
      issue(issued);
      ++issued;
    }
  }
  if (!ok) {
    // a copy did not land in time: report, then give every load still in
    // flight a bounded chance to land before the CTA (and its smem) goes away
    if (lane == 0) flag(dev_status, EP_DEV_COPY_TIMEOUT);
    for (int64_t q = j; q < issued; ++q) {
      const int s = (int)(q % stages);
      const uint32_t parity = (uint32_t)((q / stages) & 1);
      mbar_wait_bounded(&bars[s], parity);
    }
  }
  bulk_wait_all();
  if (bad) flag(dev_status, bad);
}

// y[i] = bf16_rn(float(buf[i]) * scale[topk[src[i]]])  (stand-in expert)
__global__ void __launch_bounds__(256)
    k_expert_scale(const uint16_t* __restrict__ buf, int64_t rows, int64_t H, const int32_t* __restrict__ src,
                   const int32_t* __restrict__ topk, int64_t P, const float* __restrict__ scale, int E,
                   uint16_t* __restrict__ y, int32_t* dev_status) {
  const int64_t nvec = H / 8;
  const int tpr = (int)(nvec >= 256 ? 256 : (nvec + 31) / 32 * 32);  // threads per row
  const int rows_per_cta = 256 / tpr;
  const int sub = threadIdx.x / tpr, v0 = threadIdx.x % tpr;
  int32_t bad = 0;
  for (int64_t r = (int64_t)blockIdx.x * rows_per_cta + sub; r < rows; r += (int64_t)gridDim.x * rows_per_cta) {
    if (sub >= rows_per_cta) break;
    const int32_t p = __ldg(src + r);
    int e = (p >= 0 && p < P) ? __ldg(topk + p) : -1;
    if (e < 0 || e >= E) {
      bad = EP_DEV_BAD_ROW;
      continue;
    }
    const float s = __ldg(scale + e);
    for (int64_t v = v0; v < nvec; v += tpr) {
      const uint4 in = ld_stream_v4(buf + r * H + v * 8);
      const uint32_t w[4] = {in.x, in.y, in.z, in.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        o[q] = f32x2_to_bf16x2(__fmul_rn(bf16_bits_to_f32(w[q] & 0xFFFFu), s),
                               __fmul_rn(bf16_bits_to_f32(w[q] >> 16), s));
      }
      st_v4(y + r * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
  if (bad) flag(dev_status, bad);
}

// Combine with the indices and gate weights of a CTA's tokens staged in shared
// memory one iteration ahead (double buffer), so each thread's K 16-byte row
// loads issue back to back without waiting on index loads, and registers stay
// within 64 (four 256-thread CTAs per SM).  Each CTA owns COMBINE_ITERS
// iterations of consecutive tokens (not a persistent grid): on B200 the same
// time as a persistent grid-stride grid at 0.9 GB, 4-6% faster at 17-19 GB
// (the block scheduler keeps the tokens in flight close together).
template <int K, bool PEER>
__global__ void __launch_bounds__(256, 4)
    k_combine(const uint16_t* __restrict__ y, int64_t y_rows, const float* __restrict__ w,
              const int32_t* __restrict__ pos, int64_t T, int64_t H, uint16_t* __restrict__ out,
              const uint64_t* __restrict__ peers, const int32_t* __restrict__ rank_first, int R,
              int64_t rows_per_rank, int32_t* dev_status) {
  wait_for_predecessor();
  constexpr int MAXT = 8;  // tokens per CTA iteration (rows narrower than 256 vectors)
  __shared__ int32_t s_rows[2][MAXT][K];
  __shared__ float s_w[2][MAXT][K];
  __shared__ const uint16_t* s_ptr[PEER ? 2 : 1][PEER ? MAXT : 1][PEER ? K : 1];  // row bases (PEER)
  __shared__ int s_bad;
  const int64_t nvec = H / 8;
  const int tpr = (int)(nvec >= 256 ? 256 : (nvec + 31) / 32 * 32);  // threads per token
  const int tpc = 256 / tpr <= MAXT ? 256 / tpr : MAXT;                // tokens per CTA iteration
  const int sub = threadIdx.x / tpr, v0 = threadIdx.x % tpr;
  const int64_t step = tpc;
  const int64_t t_begin = (int64_t)blockIdx.x * tpc * COMBINE_ITERS;
  const int64_t t_end = min(T, t_begin + (int64_t)tpc * COMBINE_ITERS);
  if (threadIdx.x == 0) s_bad = 0;
  auto stage = [&](int b, int64_t tb) {
    if (threadIdx.x < tpc * K) {
      const int s = threadIdx.x / K, k = threadIdx.x - s * K;
      const int64_t t = tb + s;
      int32_t r = -1;
      float wk = 0.0f;
      if (t < T) {
        r = __ldg(pos + t * K + k);
        wk = w ? __ldg(w + t * K + k) : 1.0f;  // no weights: the unpermute (x 1.0f is exact)
        if (r < 0 || r >= y_rows) {
          r = -1;
          s_bad = 1;
        }
      }
      s_rows[b][s][k] = r;
      s_w[b][s][k] = wk;
      if constexpr (PEER) {
        const uint16_t* base = nullptr;
        if (r >= 0) {
          base = reinterpret_cast<const uint16_t*>(peer_row(peers, rank_first, R, rows_per_rank, r, H * 2));
          if (!base) {  // a missing or misaligned rank buffer, or a row past it, is reported, never read
            s_rows[b][s][k] = -1;
            s_bad = 1;
          }
        }
        s_ptr[PEER ? b : 0][PEER ? s : 0][PEER ? k : 0] = base;
      }
    }
  };
  int64_t tb = t_begin;
  stage(0, tb);
  __syncthreads();
  for (int b = 0; tb < t_end; tb += step, b ^= 1) {
    if (tb + step < t_end) stage(b ^ 1, tb + step);
    const int64_t t = tb + sub;
    if (sub < tpc && t < T) {
      for (int64_t v = v0; v < nvec; v += tpr) {
        uint4 in[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
          const int32_t r = s_rows[b][sub][k];
          if constexpr (PEER)
            in[k] = r >= 0 ? ld_stream_v4(s_ptr[PEER ? b : 0][PEER ? sub : 0][PEER ? k : 0] + v * 8)
                           : make_uint4(0, 0, 0, 0);
          else
            in[k] = r >= 0 ? ld_stream_v4(y + (int64_t)r * H + v * 8) : make_uint4(0, 0, 0, 0);
        }
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll
        for (int k = 0; k < K; ++k) {
          if (s_rows[b][sub][k] < 0) continue;  // an invalid row contributes nothing
          const float wk = s_w[b][sub][k];
          const uint32_t wd[4] = {in[k].x, in[k].y, in[k].z, in[k].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[2 * q] = __fadd_rn(acc[2 * q], __fmul_rn(wk, bf16_bits_to_f32(wd[q] & 0xFFFFu)));
            acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __fmul_rn(wk, bf16_bits_to_f32(wd[q] >> 16)));
          }
        }
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] = f32x2_to_bf16x2(acc[2 * q], acc[2 * q + 1]);
        st_v4(out + t * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0 && s_bad) flag(dev_status, EP_DEV_BAD_ROW);
}

// Any K up to 32, one row at a time (no K-wide register arrays).
__global__ void __launch_bounds__(256)
    k_combine_any(const uint16_t* __restrict__ y, int64_t y_rows, const float* __restrict__ w,
                  const int32_t* __restrict__ pos, int64_t T, int K, int64_t H, uint16_t* __restrict__ out,
                  int32_t* dev_status) {
  const int64_t nvec = H / 8;
  int32_t bad = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < T * nvec; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / nvec, v = i - t * nvec;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
    for (int k = 0; k < K; ++k) {
      const int32_t r = __ldg(pos + t * K + k);
      if (r < 0 || r >= y_rows) {
        bad = EP_DEV_BAD_ROW;
        continue;
      }
      const float wk = w ? __ldg(w + t * K + k) : 1.0f;
      const uint4 in = ld_stream_v4(y + (int64_t)r * H + v * 8);
      const uint32_t wd[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] = __fadd_rn(acc[2 * q], __fmul_rn(wk, bf16_bits_to_f32(wd[q] & 0xFFFFu)));
        acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __fmul_rn(wk, bf16_bits_to_f32(wd[q] >> 16)));
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = f32x2_to_bf16x2(acc[2 * q], acc[2 * q + 1]);
    st_v4(out + t * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
  }
  if (bad) flag(dev_status, bad);
}

// Backward of combine.  For every pair (t, k) with row r = pos[t*K+k]:
//   dy[r]    = bf16_rn(w[t,k] * float(dout[t]))          (one fp32 multiply per element)
//   dw[t,k]  = sum_h float(dout[t,h]) * float(y[r,h])     (fp32; any summation order)
// One group of G lanes owns one token (G = 32 for rows of 256+ elements, else
// the power of two covering the row's 16-byte vectors, so a warp carries
// 32 / G tokens), and each warp owns exactly one such group of tokens: the
// grid is one warp per token group, four warps per CTA (not persistent).  The
// group's rows and weights are read into shared memory once.  A lane walks
// every G-th 16-byte vector of its token's row ("jobs"); the dout vector and
// the K y vectors of each job are copied into a per-warp shared-memory ring of
// CB_STAGES slots with cp.async, CB_STAGES - 1 jobs ahead of the one being
// computed, so the loads in flight hold no registers.  From its slot a lane
// writes the K scaled dy vectors and adds to K partial dot products, which a
// butterfly of shuffles inside the group sums at the end.  A lane only ever
// reads what it copied itself, so the warp needs no barrier around the ring.
// Measured on B200 (fraction of the measured copy bandwidth, graph of one
// launch, L2 flushed): 0.92 -> 0.98 on the moderate EP8 workload and 0.96 ->
// 1.01 on the 17-19 GB ones, against the earlier register-staged loop (116-128
// registers, 16 warps per SM); outputs bit for bit the same.
constexpr int CB_THREADS = 128;
constexpr int CB_STAGES = 4;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__host__ __device__ __forceinline__ int combine_bwd_group(int64_t nvec) {
  return nvec >= 32 ? 32 : nvec > 8 ? (nvec > 16 ? 32 : 16) : (nvec > 4 ? 8 : nvec > 2 ? 4 : (int)nvec);
}

// Shared memory per warp: the ring [CB_STAGES][K + 1][32] of 16-byte vectors,
// then the group's rows [gpw][K] and weights [gpw][K]; rounded up to 16 bytes
// so that every warp's ring starts where cp.async can write 16 bytes.
__host__ __device__ __forceinline__ size_t combine_bwd_warp_bytes(int K, int gpw) {
  return ((size_t)CB_STAGES * (K + 1) * 512 + (size_t)2 * gpw * K * 4 + 15) & ~(size_t)15;
}

template <int K>
__global__ void __launch_bounds__(CB_THREADS, 4)
    k_combine_bwd(const uint16_t* __restrict__ dout, const float* __restrict__ w, const uint16_t* __restrict__ y,
                  int64_t y_rows, const int32_t* __restrict__ pos, int64_t T, int64_t H, uint16_t* __restrict__ dy,
                  float* __restrict__ dw, int32_t* dev_status) {
  extern __shared__ __align__(16) unsigned char cb_smem[];
  const int64_t nvec = H / 8;
  const int G = combine_bwd_group(nvec);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gpw = 32 / G;
  const int sub = lane / G, gl = lane % G;
  unsigned char* mine = cb_smem + warp * combine_bwd_warp_bytes(K, gpw);
  uint4* ring = reinterpret_cast<uint4*>(mine);  // [CB_STAGES][K + 1][32]
  int32_t* s_r = reinterpret_cast<int32_t*>(mine + (size_t)CB_STAGES * (K + 1) * 512);
  float* s_w = reinterpret_cast<float*>(s_r + gpw * K);
  const int64_t t0 = (((int64_t)blockIdx.x * CB_THREADS + threadIdx.x) >> 5) * gpw;  // the warp's first token
  if (t0 >= T) return;                                                             // warp-uniform
  int32_t bad = 0;
  for (int i = lane; i < gpw * K; i += 32) {
    const int64_t t = t0 + i / K;
    int32_t r = -1;
    float wk = 0.0f;
    if (t < T) {
      r = __ldg(pos + t * K + i % K);
      wk = __ldg(w + t * K + i % K);
      if (r < 0 || r >= y_rows) {  // reported, never read or written
        r = -1;
        bad = EP_DEV_BAD_ROW;
      }
    }
    s_r[i] = r;
    s_w[i] = wk;
  }
  __syncwarp();
  const int64_t t = t0 + sub;
  const int32_t* rr = s_r + sub * K;
  const float* ww = s_w + sub * K;
  const int nj = (int)((nvec + G - 1) / G);
  auto issue = [&](int j) {
    const int64_t v = gl + (int64_t)j * G;
    if (j < nj && t < T && v < nvec) {
      uint4* dst = ring + (size_t)(j % CB_STAGES) * (K + 1) * 32 + lane;
      cp_async16(dst, dout + t * H + v * 8);
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (rr[k] >= 0) cp_async16(dst + (k + 1) * 32, y + (int64_t)rr[k] * H + v * 8);
    }
    cp_async_commit();  // one group per job, empty or not, so the wait counts stay uniform
  };
#pragma unroll
  for (int j = 0; j < CB_STAGES - 1; ++j) issue(j);
  float part[K];
#pragma unroll
  for (int k = 0; k < K; ++k) part[k] = 0.0f;
  for (int j = 0; j < nj; ++j) {
    issue(j + CB_STAGES - 1);  // into the slot job j - 1 used (computed last iteration)
    cp_async_wait<CB_STAGES - 1>();
    const int64_t v = gl + (int64_t)j * G;
    if (t < T && v < nvec) {
      const uint4* src = ring + (size_t)(j % CB_STAGES) * (K + 1) * 32 + lane;
      const uint4 g = src[0];
      const uint32_t gd[4] = {g.x, g.y, g.z, g.w};
      float gf[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        gf[2 * q] = bf16_bits_to_f32(gd[q] & 0xFFFFu);
        gf[2 * q + 1] = bf16_bits_to_f32(gd[q] >> 16);
      }
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int32_t r = rr[k];
        if (r < 0) continue;
        const float wk = ww[k];
        const uint4 yk = src[(k + 1) * 32];
        const uint32_t yd[4] = {yk.x, yk.y, yk.z, yk.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          o[q] = f32x2_to_bf16x2(__fmul_rn(wk, gf[2 * q]), __fmul_rn(wk, gf[2 * q + 1]));
          part[k] = fmaf(gf[2 * q], bf16_bits_to_f32(yd[q] & 0xFFFFu), part[k]);
          part[k] = fmaf(gf[2 * q + 1], bf16_bits_to_f32(yd[q] >> 16), part[k]);
        }
        st_v4(dy + (int64_t)r * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
      }
    }
  }
  cp_async_wait<0>();
  // add the group's partial products (every lane of the warp takes part)
#pragma unroll
  for (int k = 0; k < K; ++k)
    for (int d = G >> 1; d; d >>= 1) part[k] += __shfl_xor_sync(0xffffffffu, part[k], d);
  if (t < T && gl == 0) {
#pragma unroll
    for (int k = 0; k < K; ++k) dw[t * K + k] = rr[k] >= 0 ? part[k] : 0.0f;
  }
  if (bad) flag(dev_status, bad);
}

// Combine for large problems (at least COMBINE_RING_MIN row elements): the same
// arithmetic as k_combine, bit for bit, with the ring structure of
// k_combine_bwd -- one warp per token group, the K y vectors of each 16-byte
// job copied into a per-warp four-slot shared-memory ring with cp.async three
// jobs ahead, so no register holds a load in flight.  Measured on B200 (graph
// of one launch, L2 flushed, fraction of the measured copy bandwidth): 1.04 ->
// 1.10 on the fine-grained and adversarial workloads; slower at 0.9 GB (0.95 ->
// 0.93), where k_combine stays.
constexpr int64_t COMBINE_RING_MIN = (int64_t)1 << 28;

// per warp: the ring [CB_STAGES][K][32], the group's rows and weights; rounded
// up to 16 bytes (every warp's ring starts on a cp.async boundary)
__host__ __device__ __forceinline__ size_t combine_ring_warp_bytes(int K, int gpw) {
  return ((size_t)CB_STAGES * K * 512 + (size_t)2 * gpw * K * 4 + 15) & ~(size_t)15;
}

template <int K>
__global__ void __launch_bounds__(CB_THREADS, 4)
    k_combine_ring(const uint16_t* __restrict__ y, int64_t y_rows, const float* __restrict__ w,
                   const int32_t* __restrict__ pos, int64_t T, int64_t H, uint16_t* __restrict__ out,
                   int32_t* dev_status) {
  wait_for_predecessor();
  extern __shared__ __align__(16) unsigned char cr_smem[];
  const int64_t nvec = H / 8;
  const int G = combine_bwd_group(nvec);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gpw = 32 / G;
  const int sub = lane / G, gl = lane % G;
  unsigned char* mine = cr_smem + warp * combine_ring_warp_bytes(K, gpw);
  uint4* ring = reinterpret_cast<uint4*>(mine);  // [CB_STAGES][K][32]
  int32_t* s_r = reinterpret_cast<int32_t*>(mine + (size_t)CB_STAGES * K * 512);
  float* s_w = reinterpret_cast<float*>(s_r + gpw * K);
  const int64_t t0 = (((int64_t)blockIdx.x * CB_THREADS + threadIdx.x) >> 5) * gpw;
  if (t0 >= T) return;  // warp-uniform
  int32_t bad = 0;
  for (int i = lane; i < gpw * K; i += 32) {
    const int64_t t = t0 + i / K;
    int32_t r = -1;
    float wk = 0.0f;
    if (t < T) {
      r = __ldg(pos + t * K + i % K);
      wk = w ? __ldg(w + t * K + i % K) : 1.0f;  // no weights: the unpermute (x 1.0f is exact)
      if (r < 0 || r >= y_rows) {  // reported, never read; contributes nothing
        r = -1;
        bad = EP_DEV_BAD_ROW;
      }
    }
    s_r[i] = r;
    s_w[i] = wk;
  }
  __syncwarp();
  const int64_t t = t0 + sub;
  const int32_t* rr = s_r + sub * K;
  const float* ww = s_w + sub * K;
  const int nj = (int)((nvec + G - 1) / G);
  auto issue = [&](int j) {
    const int64_t v = gl + (int64_t)j * G;
    if (j < nj && t < T && v < nvec) {
      uint4* dst = ring + (size_t)(j % CB_STAGES) * K * 32 + lane;
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (rr[k] >= 0) cp_async16(dst + k * 32, y + (int64_t)rr[k] * H + v * 8);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int j = 0; j < CB_STAGES - 1; ++j) issue(j);
  for (int j = 0; j < nj; ++j) {
    issue(j + CB_STAGES - 1);
    cp_async_wait<CB_STAGES - 1>();
    const int64_t v = gl + (int64_t)j * G;
    if (t < T && v < nvec) {
      const uint4* src = ring + (size_t)(j % CB_STAGES) * K * 32 + lane;
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if (rr[k] < 0) continue;  // an invalid row contributes nothing
        const float wk = ww[k];
        const uint4 yk = src[k * 32];
        const uint32_t wd[4] = {yk.x, yk.y, yk.z, yk.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] = __fadd_rn(acc[2 * q], __fmul_rn(wk, bf16_bits_to_f32(wd[q] & 0xFFFFu)));
          acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __fmul_rn(wk, bf16_bits_to_f32(wd[q] >> 16)));
        }
      }
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) o[q] = f32x2_to_bf16x2(acc[2 * q], acc[2 * q + 1]);
      st_v4(out + t * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
  cp_async_wait<0>();
  if (bad) flag(dev_status, bad);
}

static const void* combine_ring_fn(int K) {
  switch (K) {
    case 1: return (const void*)k_combine_ring<1>;
    case 2: return (const void*)k_combine_ring<2>;
    case 3: return (const void*)k_combine_ring<3>;
    case 4: return (const void*)k_combine_ring<4>;
    case 5: return (const void*)k_combine_ring<5>;
    case 6: return (const void*)k_combine_ring<6>;
    case 7: return (const void*)k_combine_ring<7>;
    case 8: return (const void*)k_combine_ring<8>;
    default: return nullptr;
  }
}

// Grid of k_combine<K, *> for T tokens of H values: one CTA per
// COMBINE_ITERS iterations of its tokens-per-iteration (the kernel's tpc).
static int combine_grid(int64_t T, int64_t H) {
  const int64_t nvec = H / 8;
  const int tpr = (int)(nvec >= 256 ? 256 : (nvec + 31) / 32 * 32);
  const int tpc = 256 / tpr <= 8 ? 256 / tpr : 8;
  const int64_t per_cta = (int64_t)tpc * COMBINE_ITERS;
  return (int)std::min<int64_t>((T + per_cta - 1) / per_cta, 0x7fffffff);
}

int occupancy_grid(const void* fn, int threads, size_t smem, int64_t work_items, int cap_per_sm) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  per_sm = std::min(per_sm, cap_per_sm);
  int64_t g = (int64_t)num_sms() * per_sm;
  g = std::min<int64_t>(g, std::max<int64_t>(1, work_items));
  return (int)g;
}

}  // namespace ep

using namespace ep;

namespace ep {

// Shared-memory stages of one dispatch CTA for rows of H bf16 values (the
// launch below): 4 stages for rows up to 1 KB, else 2.
static size_t dispatch_smem(int64_t H, int K) {
  const uint32_t stride_b = ((uint32_t)(H * 2) + 127u) & ~127u;
  const int stages = stride_b * 2u * 16u <= 32u * 1024u ? 4 : 2;
  return (size_t)stages * stride_b + DISPATCH_MAX_STAGES * 8 + (size_t)stages * K * 4;
}

// Whether ep_dispatch accepts rows of H values at top-K = K (its stages fit).
bool dispatch_shape_ok(int64_t H, int K) {
  return K >= 1 && K <= 32 && H >= 8 && H % 8 == 0 && H * 2 <= (1 << 20) && dispatch_smem(H, K) <= 200 * 1024;
}

// Dispatch launch shared by the one-buffer and the rank-local (peer) entry
// points.  peers == NULL: rows go to buf[row]; else to the rank buffers.
static int run_dispatch(const uint16_t* x, int64_t T, int K, int64_t H, const int32_t* pos, uint16_t* buf,
                        int64_t buf_rows, const uint64_t* peers, const int32_t* rank_first, int R,
                        int64_t rows_per_rank, int32_t* dev_status, cudaStream_t stream) {
  const uint32_t row_bytes = (uint32_t)(H * 2);
  const uint32_t stride_b = (row_bytes + 127u) & ~127u;
  // Measured on B200: the scatter runs fastest with about 32 KB of row loads
  // in flight per SM (e.g. 2 stages x 4 CTAs of 4 KB rows: 6.0 TB/s, against
  // 5.5 TB/s with 48 KB per CTA and 6 CTAs); more concurrency only adds
  // read/write contention at the memory.  Small rows use 4 stages so the
  // per-SM target is reached within 32 CTAs.
  const uint32_t target = 32u * 1024u;
  const int stages = stride_b * 2u * 16u <= target ? 4 : 2;
  const int per_sm = (int)std::min<uint32_t>(32, std::max<uint32_t>(1, (target + stages * stride_b - 1) / (stages * stride_b)));
  const size_t need = dispatch_smem(H, K);
  if (need > 200 * 1024) return EP_ERR_ARG;
  // the same rows in flight per SM as per_sm CTAs of `stages` rows each: a CTA
  // holds DISPATCH_TOKENS_PER_CTA rows, so per_sm * stages / that many CTAs
  // may be resident; the shared memory each reserves caps them (228 KB per SM,
  // 1 KB of it per CTA; at most 32 CTAs)
  static_assert(DISPATCH_TOKENS_PER_CTA <= 2, "stages (2 or 4) must cover a CTA's tokens");
  const int resident = std::min(32, per_sm * stages / DISPATCH_TOKENS_PER_CTA);
  const size_t smem = std::max(need, (size_t)(220 * 1024) / resident);
  const void* fn = peers ? (const void*)k_dispatch<true> : (const void*)k_dispatch<false>;
  if (smem > 48 * 1024 && !raise_smem_limit(fn, smem))
    return EP_ERR_CUDA;
  const int64_t blocks = (T + DISPATCH_TOKENS_PER_CTA - 1) / DISPATCH_TOKENS_PER_CTA;
  if (blocks > 0x7fffffff) return EP_ERR_ARG;
  const int grid = (int)blocks;
  const uint8_t* xb = reinterpret_cast<const uint8_t*>(x);
  uint8_t* bb = reinterpret_cast<uint8_t*>(buf);
  void* args[] = {(void*)&xb,    (void*)&T,          (void*)&K, (void*)&row_bytes,     (void*)&pos,
                  (void*)&buf_rows, (void*)&bb,      (void*)&peers, (void*)&rank_first, (void*)&R,
                  (void*)&rows_per_rank, (void*)&stages, (void*)&dev_status};
  if (launch_pdl(fn, dim3(grid), dim3(32), args, smem, stream) != cudaSuccess) return EP_ERR_CUDA;
  count_launch();
  return launch_status();
}

}  // namespace ep

extern "C" int ep_dispatch(const uint16_t* x, int64_t T, int K, int64_t H, const int32_t* pos, uint16_t* buf,
                           int64_t buf_rows, int32_t* dev_status, cudaStream_t stream) {
  if (T < 0 || K < 1 || K > 32 || H < 8 || H % 8 || buf_rows < 0) return EP_ERR_ARG;
  if (H * 2 > (1 << 20)) return EP_ERR_ARG;  // one row per bulk copy, at most 1 MiB
  if (T * (int64_t)K >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  if (T == 0) return EP_OK;
  if (!x || !pos || !buf || !aligned16(x) || !aligned16(buf)) return EP_ERR_ARG;
  return run_dispatch(x, T, K, H, pos, buf, buf_rows, nullptr, nullptr, 1, 0, dev_status, stream);
}

extern "C" int ep_dispatch_peer(const uint16_t* x_local, int64_t S, int K, int64_t H, const int32_t* pos_local,
                                const uint64_t* peer_bufs, const int32_t* rank_first_row, int R,
                                int64_t rows_per_rank, int64_t total_rows, int32_t* dev_status,
                                cudaStream_t stream) {
  if (S < 0 || K < 1 || K > 32 || H < 8 || H % 8 || R < 1 || R > EP_MAX_RANKS || rows_per_rank < 1 || total_rows < 0)
    return EP_ERR_ARG;
  if (H * 2 > (1 << 20)) return EP_ERR_ARG;
  if (S * (int64_t)K >= ((int64_t)1 << 31) || total_rows >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  if (S == 0) return EP_OK;
  if (!x_local || !pos_local || !peer_bufs || !aligned16(x_local)) return EP_ERR_ARG;
  return run_dispatch(x_local, S, K, H, pos_local, nullptr, total_rows, peer_bufs, rank_first_row, R, rows_per_rank,
                      dev_status, stream);
}

extern "C" int ep_expert_scale(const uint16_t* buf, int64_t rows, int64_t H, const int32_t* src,
                               const int32_t* topk_ids, int64_t P, const float* scale, int E, uint16_t* y,
                               int32_t* dev_status, cudaStream_t stream) {
  if (rows < 0 || H < 8 || H % 8 || E < 1 || P < 0) return EP_ERR_ARG;
  if (rows == 0) return EP_OK;
  if (!buf || !src || !topk_ids || !scale || !y || !aligned16(buf) || !aligned16(y)) return EP_ERR_ARG;
  const int grid = occupancy_grid((const void*)k_expert_scale, 256, 0, rows, 8);
  k_expert_scale<<<grid, 256, 0, stream>>>(buf, rows, H, src, topk_ids, P, scale, E, y, dev_status);
  count_launch();
  return launch_status();
}

namespace ep {

template <bool PEER>
static const void* combine_fn(int K) {
  switch (K) {
    case 1: return (const void*)k_combine<1, PEER>;
    case 2: return (const void*)k_combine<2, PEER>;
    case 3: return (const void*)k_combine<3, PEER>;
    case 4: return (const void*)k_combine<4, PEER>;
    case 5: return (const void*)k_combine<5, PEER>;
    case 6: return (const void*)k_combine<6, PEER>;
    case 7: return (const void*)k_combine<7, PEER>;
    case 8: return (const void*)k_combine<8, PEER>;
    default: return nullptr;
  }
}

}  // namespace ep

extern "C" int ep_combine(const uint16_t* y, int64_t y_rows, const float* w, const int32_t* pos, int64_t T, int K,
                          int64_t H, uint16_t* out, int32_t* dev_status, cudaStream_t stream) {
  if (T < 0 || K < 1 || K > 32 || H < 8 || H % 8 || y_rows < 0) return EP_ERR_ARG;
  if (T * (int64_t)K >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  if (T == 0) return EP_OK;
  if (!y || !pos || !out || !aligned16(y) || !aligned16(out)) return EP_ERR_ARG;  // w == NULL: unit weights
  const void* ring_fn = T * H >= COMBINE_RING_MIN ? combine_ring_fn(K) : nullptr;
  const void* fn = combine_fn<false>(K);
  if (ring_fn) {  // large problems: one warp per token group, loads through a shared-memory ring
    const int gpw = 32 / combine_bwd_group(H / 8);
    const int64_t groups = (T + gpw - 1) / gpw;
    const int64_t ctas = (groups + CB_THREADS / 32 - 1) / (CB_THREADS / 32);
    if (ctas > 0x7fffffff) return EP_ERR_ARG;
    const size_t smem = (size_t)(CB_THREADS / 32) * combine_ring_warp_bytes(K, gpw);
    if (smem > 48 * 1024 && !raise_smem_limit(ring_fn, smem)) return EP_ERR_CUDA;
    void* args[] = {(void*)&y, (void*)&y_rows, (void*)&w, (void*)&pos, (void*)&T, (void*)&H, (void*)&out,
                    (void*)&dev_status};
    if (launch_pdl(ring_fn, dim3((unsigned)ctas), dim3(CB_THREADS), args, smem, stream) != cudaSuccess)
      return EP_ERR_CUDA;
  } else if (fn) {
    const int grid = combine_grid(T, H);
    const uint64_t* peers = nullptr;
    const int32_t* rank_first = nullptr;
    int R = 1;
    int64_t rpr = 0;
    void* args[] = {(void*)&y,     (void*)&y_rows,     (void*)&w, (void*)&pos, (void*)&T,          (void*)&H,
                    (void*)&out,   (void*)&peers, (void*)&rank_first, (void*)&R, (void*)&rpr, (void*)&dev_status};
    if (launch_pdl(fn, dim3(grid), dim3(256), args, 0, stream) != cudaSuccess) return EP_ERR_CUDA;
  } else {
    const int grid = occupancy_grid((const void*)k_combine_any, 256, 0, T * (H / 8) / 256 + 1, 8);
    k_combine_any<<<grid, 256, 0, stream>>>(y, y_rows, w, pos, T, K, H, out, dev_status);
  }
  count_launch();
  return launch_status();
}

extern "C" int ep_combine_peer(const uint64_t* peer_bufs, const int32_t* rank_first_row, int R,
                               int64_t rows_per_rank, int64_t total_rows, const float* w_local,
                               const int32_t* pos_local, int64_t S, int K, int64_t H, uint16_t* out_local,
                               int32_t* dev_status, cudaStream_t stream) {
  if (S < 0 || K < 1 || K > 8 || H < 8 || H % 8 || R < 1 || R > EP_MAX_RANKS || rows_per_rank < 1 || total_rows < 0)
    return EP_ERR_ARG;
  if (S * (int64_t)K >= ((int64_t)1 << 31) || total_rows >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  if (S == 0) return EP_OK;
  if (!peer_bufs || !pos_local || !out_local || !aligned16(out_local)) return EP_ERR_ARG;  // w NULL: unit weights
  const void* fn = combine_fn<true>(K);
  const int grid = combine_grid(S, H);
  const uint16_t* y = nullptr;
  void* args[] = {(void*)&y,          (void*)&total_rows, (void*)&w_local,        (void*)&pos_local,
                  (void*)&S,          (void*)&H,          (void*)&out_local,      (void*)&peer_bufs,
                  (void*)&rank_first_row, (void*)&R,      (void*)&rows_per_rank,  (void*)&dev_status};
  if (launch_pdl(fn, dim3(grid), dim3(256), args, 0, stream) != cudaSuccess) return EP_ERR_CUDA;
  count_launch();
  return launch_status();
}

extern "C" int ep_dispatch_backward(const uint16_t* dbuf, int64_t buf_rows, const int32_t* pos, int64_t T, int K,
                                    int64_t H, uint16_t* dx, int32_t* dev_status, cudaStream_t stream) {
  // dx[t] = sum_k dbuf[pos[t*K+k]]: the combine kernel with unit weights
  return ep_combine(dbuf, buf_rows, nullptr, pos, T, K, H, dx, dev_status, stream);
}

extern "C" int ep_combine_backward(const uint16_t* dout, const float* w, const uint16_t* y, int64_t y_rows,
                                   const int32_t* pos, int64_t T, int K, int64_t H, uint16_t* dy, float* dw,
                                   int32_t* dev_status, cudaStream_t stream) {
  if (T < 0 || K < 1 || K > 8 || H < 8 || H % 8 || y_rows < 0) return EP_ERR_ARG;
  if (T * (int64_t)K >= ((int64_t)1 << 31)) return EP_ERR_ARG;
  if (T == 0) return EP_OK;
  if (!dout || !w || !y || !pos || !dy || !dw || !aligned16(dout) || !aligned16(y) || !aligned16(dy)) return EP_ERR_ARG;
  const void* fn = nullptr;
  switch (K) {
    case 1: fn = (const void*)k_combine_bwd<1>; break;
    case 2: fn = (const void*)k_combine_bwd<2>; break;
    case 3: fn = (const void*)k_combine_bwd<3>; break;
    case 4: fn = (const void*)k_combine_bwd<4>; break;
    case 5: fn = (const void*)k_combine_bwd<5>; break;
    case 6: fn = (const void*)k_combine_bwd<6>; break;
    case 7: fn = (const void*)k_combine_bwd<7>; break;
    default: fn = (const void*)k_combine_bwd<8>; break;
  }
  // one warp per token group (32 / G tokens), four warps per CTA
  const int64_t nvec = H / 8;
  const int G = combine_bwd_group(nvec);
  const int gpw = 32 / G;
  const int64_t groups = (T + gpw - 1) / gpw;
  const int64_t ctas = (groups + CB_THREADS / 32 - 1) / (CB_THREADS / 32);
  if (ctas > 0x7fffffff) return EP_ERR_ARG;
  const size_t smem = (size_t)(CB_THREADS / 32) * combine_bwd_warp_bytes(K, gpw);
  if (smem > 48 * 1024 && !raise_smem_limit(fn, smem)) return EP_ERR_CUDA;
  const int grid = (int)ctas;
  void* args[] = {(void*)&dout, (void*)&w, (void*)&y, (void*)&y_rows, (void*)&pos, (void*)&T, (void*)&H, (void*)&dy,
                  (void*)&dw, (void*)&dev_status};
  if (cudaLaunchKernel(fn, dim3(grid), dim3(CB_THREADS), args, smem, stream) != cudaSuccess) return EP_ERR_CUDA;
  count_launch();
  return launch_status();
}
