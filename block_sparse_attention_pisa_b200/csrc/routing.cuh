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
// Both kernels stream the per-block S1 of a head once, and every sum runs in a fixed
// order (no atomics), so Hbar and M are the same bit for bit on every call:
//   routing_hbar_kernel: grid (slice, head); a slice is 1024 consecutive elements of the
//                        d x d matrix, 8 per thread (one 16-byte load per block, 16 blocks
//                        in flight); each thread sums its elements over all blocks
//                        j = 0 .. nB - 1 in turn, then Hbar = sum / nB;
//   routing_norm_kernel: grid (chunk of kRouteChunk blocks, head); per block, each
//                        thread sums (S1_j - Hbar)^2 over its D*D/256 elements, the
//                        warps reduce by shuffles, and after one CTA barrier thread jj
//                        adds block jj's eight warp sums in warp order: M_j = sqrt(sum).
#pragma once

#include "common.cuh"

namespace pisa {

constexpr int kRouteThreads = 256;              // norm kernel
constexpr int kRouteSlice = kRouteThreads * 8;  // matrix elements per norm-kernel pass
constexpr int kRouteChunk = 16;                 // key blocks per norm CTA
constexpr int kHbarThreads = 128;               // Hbar kernel
constexpr int kHbarSlice = kHbarThreads * 8;    // matrix elements per Hbar CTA

__global__ void __launch_bounds__(kHbarThreads)
routing_hbar_kernel(const bf16* __restrict__ S1, int nB, int dd, float* __restrict__ Hbar) {
  const int e0 = blockIdx.x * kHbarSlice + threadIdx.x * 8;  // first element of this thread
  const size_t bh = blockIdx.y;
  const bf16* src = S1 + (bh * size_t(nB)) * dd + e0;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  auto add = [&](const uint4& w) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += bf16_lo(ww[e]);
      acc[2 * e + 1] += bf16_hi(ww[e]);
    }
  };
  // 16 blocks' loads in flight, then their sums in block order
  int j = 0;
  for (; j + 16 <= nB; j += 16) {
    uint4 w[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) w[u] = __ldg(reinterpret_cast<const uint4*>(src + size_t(j + u) * dd));
#pragma unroll
    for (int u = 0; u < 16; ++u) add(w[u]);
  }
  for (; j < nB; ++j) add(ldg_stream_v4(src + size_t(j) * dd));
  const float inv = 1.f / float(nB);
  float4* dst = reinterpret_cast<float4*>(Hbar + bh * size_t(dd) + e0);
  dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
}

template <int D>
__global__ void __launch_bounds__(kRouteThreads)
routing_norm_kernel(const bf16* __restrict__ S1, const float* __restrict__ Hbar, int nB, float* __restrict__ M) {
  constexpr int DD = D * D;
  constexpr int NV = DD / (kRouteThreads * 8);  // 16-byte loads per thread and block
  static_assert(NV * kRouteThreads * 8 == DD, "slices");
  __shared__ float part[kRouteThreads / 32][kRouteChunk];
  const int j0 = blockIdx.x * kRouteChunk;
  const int j1 = min(nB, j0 + kRouteChunk);
  const size_t bh = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // this thread's elements: v * 2048 + 8 * threadIdx.x + e
  float h[NV][8];
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const float* hp = Hbar + bh * size_t(DD) + v * kRouteSlice + threadIdx.x * 8;
    const float4 h0 = *reinterpret_cast<const float4*>(hp);
    const float4 h1 = *reinterpret_cast<const float4*>(hp + 4);
    h[v][0] = h0.x; h[v][1] = h0.y; h[v][2] = h0.z; h[v][3] = h0.w;
    h[v][4] = h1.x; h[v][5] = h1.y; h[v][6] = h1.z; h[v][7] = h1.w;
  }
  const bf16* src = S1 + (bh * size_t(nB)) * DD + threadIdx.x * 8;
#pragma unroll 2
  for (int j = j0; j < j1; ++j) {
    uint4 w[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) w[v] = ldg_stream_v4(src + size_t(j) * DD + v * kRouteSlice);
    float s = 0.f;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const uint32_t ww[4] = {w[v].x, w[v].y, w[v].z, w[v].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16_lo(ww[e]) - h[v][2 * e], b = bf16_hi(ww[e]) - h[v][2 * e + 1];
        s = fmaf(a, a, s);
        s = fmaf(b, b, s);
      }
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
    M[bh * size_t(nB) + j0 + jj] = sqrtf(s);
  }
}

}  // namespace pisa
