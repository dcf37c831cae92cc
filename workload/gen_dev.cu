// Device twin of gen.c's normal12 generator, for inputs too large to build on
// the host (hidden rows and replica gradients at the large workloads).
//
// Same definition as the host side: Philox4x32-10 (Salmon et al., SC'11) with
// key = (seed low word, stream) and counter = (block low, block high, seed high
// word, 0); element i sums the top 20 bits of the twelve words of blocks 3i,
// 3i+1, 3i+2, converts the integer sum (< 2^24) to fp32 exactly, scales by
// 2^-20 and subtracts 6 -- all exact, so host and device agree bit for bit.
// bf16 outputs are the round-to-nearest-even of that fp32 value.
//
// This file generates inputs only; it contains none of the method under test.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = 0xD2511F53u * c[0];
    const uint32_t hi0 = __umulhi(0xD2511F53u, c[0]);
    const uint32_t lo1 = 0xCD9E8D57u * c[2];
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c[2]);
    const uint32_t n0 = hi1 ^ c[1] ^ k0;
    const uint32_t n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

__device__ __forceinline__ float normal12_at(uint64_t seed, uint32_t stream, uint64_t i) {
  uint32_t sum = 0;
#pragma unroll
  for (int b = 0; b < 3; ++b) {
    const uint64_t blk = 3ull * i + (uint64_t)b;
    uint32_t w[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), (uint32_t)(seed >> 32), 0u};
    philox4x32_10(w, (uint32_t)seed, stream);
    sum += (w[0] >> 12) + (w[1] >> 12) + (w[2] >> 12) + (w[3] >> 12);
  }
  const float s = __uint2float_rn(sum);         // exact, sum < 2^24
  return __fsub_rn(__fmul_rn(s, 0x1p-20f), 6.0f); // both steps exact
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__global__ void fill_f32_kernel(uint64_t seed, uint32_t stream, uint64_t offset, int64_t n, float* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = normal12_at(seed, stream, offset + (uint64_t)i);
}

__global__ void fill_bf16_kernel(uint64_t seed, uint32_t stream, uint64_t offset, int64_t n, uint16_t* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = f32_to_bf16_rne(normal12_at(seed, stream, offset + (uint64_t)i));
}

int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" int gen_dev_fill_normal_f32(uint64_t seed, uint32_t stream, uint64_t offset, int64_t n, float* out,
                                       cudaStream_t st) {
  if (n <= 0) return 0;
  if (!out) return -1;
  fill_f32_kernel<<<grid_for(n), 256, 0, st>>>(seed, stream, offset, n, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

extern "C" int gen_dev_fill_normal_bf16(uint64_t seed, uint32_t stream, uint64_t offset, int64_t n, uint16_t* out,
                                        cudaStream_t st) {
  if (n <= 0) return 0;
  if (!out) return -1;
  fill_bf16_kernel<<<grid_for(n), 256, 0, st>>>(seed, stream, offset, n, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
