// Covariance-aware routing statistic: M_j = || S1_j - Hbar ||_F per key block.
//
// PISA explainer ("PISA: Piecewise Sparse Attention Is Wiser for Efficient
// Diffusion Transformers"), technical summary section 2, "Covariance-aware
// routing": besides attention relevance, the selection score of a block carries
// the norm of its first-order matrix's deviation from the global statistic
// Hbar, so that blocks a shared first-order term describes badly go to the
// exact path. The norm is the Frobenius norm; S1 is read as stored (bf16) and
// Hbar is the mean of the stored S1 over the head's blocks.
//
// Both kernels stream the per-block S1 of a head once: grid (slice, block chunk,
// head), where a slice is 2048 consecutive elements of the d x d matrix (8 per
// thread, one 16-byte load per block) and a chunk kRouteChunk consecutive blocks.
//   routing_hbar_kernel: Hbar += (1/nB) sum over the chunk (fp32 atomics; Hbar
//                        zeroed by the caller);
//   routing_norm_kernel: M2_j += sum over the slice of (S1_j - Hbar)^2 (fp32,
//                        CTA reduction, one atomic per block and slice; M2
//                        zeroed by the caller);
//   routing_sqrt_kernel: M_j = sqrt(M2_j).
#pragma once

#include "common.cuh"

namespace pisa {

constexpr int kRouteThreads = 256;
constexpr int kRouteSlice = kRouteThreads * 8;  // matrix elements per CTA
constexpr int kRouteChunk = 64;                 // key blocks per CTA

__global__ void __launch_bounds__(kRouteThreads)
routing_hbar_kernel(const bf16* __restrict__ S1, int nB, int dd, float* __restrict__ Hbar) {
  const int e0 = blockIdx.x * kRouteSlice + threadIdx.x * 8;  // first element of this thread
  const int j0 = blockIdx.y * kRouteChunk;
  const int j1 = min(nB, j0 + kRouteChunk);
  const size_t bh = blockIdx.z;
  const bf16* src = S1 + (bh * size_t(nB)) * dd + e0;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 8
  for (int j = j0; j < j1; ++j) {
    const uint4 w = ldg_stream_v4(src + size_t(j) * dd);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += bf16_lo(ww[e]);
      acc[2 * e + 1] += bf16_hi(ww[e]);
    }
  }
  const float inv = 1.f / float(nB);
  float* dst = Hbar + bh * size_t(dd) + e0;
  atomicAdd(reinterpret_cast<float4*>(dst), make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv));
  atomicAdd(reinterpret_cast<float4*>(dst + 4), make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv));
}

__global__ void __launch_bounds__(kRouteThreads)
routing_norm_kernel(const bf16* __restrict__ S1, const float* __restrict__ Hbar, int nB, int dd,
                    float* __restrict__ M2) {
  __shared__ float part[kRouteThreads / 32][kRouteChunk];
  const int e0 = blockIdx.x * kRouteSlice + threadIdx.x * 8;
  const int j0 = blockIdx.y * kRouteChunk;
  const int j1 = min(nB, j0 + kRouteChunk);
  const size_t bh = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float4 h0 = *reinterpret_cast<const float4*>(Hbar + bh * size_t(dd) + e0);
  const float4 h1 = *reinterpret_cast<const float4*>(Hbar + bh * size_t(dd) + e0 + 4);
  const float h[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  const bf16* src = S1 + (bh * size_t(nB)) * dd + e0;
#pragma unroll 8
  for (int j = j0; j < j1; ++j) {
    const uint4 w = ldg_stream_v4(src + size_t(j) * dd);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = bf16_lo(ww[e]) - h[2 * e], b = bf16_hi(ww[e]) - h[2 * e + 1];
      s = fmaf(a, a, s);
      s = fmaf(b, b, s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) part[warp][j - j0] = s;
  }
  __syncthreads();
  for (int jj = threadIdx.x; jj < j1 - j0; jj += kRouteThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kRouteThreads / 32; ++w) s += part[w][jj];
    atomicAdd(M2 + bh * size_t(nB) + j0 + jj, s);
  }
}

__global__ void routing_sqrt_kernel(float* __restrict__ M, size_t n) {
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) M[i] = sqrtf(M[i]);
}

}  // namespace pisa
