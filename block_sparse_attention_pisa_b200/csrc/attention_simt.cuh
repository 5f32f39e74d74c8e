// Plain CUDA-core PISA attention (cross-check kernel, not tuned).
//
// Same definition as the fused tensor-core kernel (PISA explainer, technical
// summary section 2, "Core algorithm": exact sparse term over the critical
// blocks, zeroth-order term alpha_{t,j} S0_j with alpha = exp(x.kbar_j), and
// the first-order term alpha_{t,j} S1_j^T x_t; one online-softmax accumulator),
// with the same order codes: -1 keep-or-drop, 0, 1 per-block first order,
// 2 hybrid order with the global correction (x_t Hbar) sum_U alpha_{t,j}.
// One CTA per (query block, head), one thread per query row; blocks are visited
// in ascending order and the accumulator is rescaled whenever the running row
// maximum grows. It is reached only through its own entry point
// (pisa_attention_simt): an independent GPU cross-check of the fused kernel on
// sizes where the CPU oracle is slow. pisa_attention never routes to it.
#pragma once

#include "common.cuh"

namespace pisa {

template <int D>
struct SimtCfg {
  static constexpr int kMaxRows = 128;
  static size_t smem_bytes() {
    return size_t(D) * kMaxRows * sizeof(float)                 // xT
           + size_t(2) * kMaxRows * D * sizeof(bf16)              // K, V tile (S1 tile overlays)
           + size_t(2) * D * sizeof(float)                        // kbar_j, S0_j
           + size_t(PISA_MAX_BLOCKS_DEV / 32) * sizeof(uint32_t);  // critical-block bitmask
  }
  static constexpr int PISA_MAX_BLOCKS_DEV = 2048;
  static_assert(2 * kMaxRows * D >= D * D, "S1 tile must fit in the K/V tile");
};

template <int D>
__global__ void __launch_bounds__(128)
attention_simt_kernel(const bf16* __restrict__ Q, const bf16* __restrict__ K,
                      const bf16* __restrict__ V, const float* __restrict__ kbar,
                      const float* __restrict__ S0, const bf16* __restrict__ S1,
                      const float* __restrict__ hbar, const int32_t* __restrict__ idx, int N, int nB, int block, int topk,
                      int order, float scale, bf16* __restrict__ O) {
  using C = SimtCfg<D>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* xT = reinterpret_cast<float*>(smem_raw);         // [D][kMaxRows]
  bf16* sK = reinterpret_cast<bf16*>(xT + D * C::kMaxRows);  // [block][D]
  bf16* sV = sK + C::kMaxRows * D;                          // [block][D]
  bf16* sS1 = sK;                                           // [D][D] overlay
  float* sKb = reinterpret_cast<float*>(sV + C::kMaxRows * D);
  float* sS0 = sKb + D;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sS0 + D);

  const int i = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int t = threadIdx.x;
  const int nthr = blockDim.x;
  const int row = i * block + t;
  const bool valid = t < block && row < N;

  for (int w = t; w < (nB + 31) / 32; w += nthr) sMask[w] = 0u;
  __syncthreads();
  const int32_t* myidx = idx + (bh * size_t(nB) + i) * topk;
  for (int e = t; e < topk; e += nthr) {
    const int j = myidx[e];
    if (j >= 0 && j < nB) atomicOr(&sMask[j >> 5], 1u << (j & 31));
    else flag_error(kErrBadIndex);
  }
  const bf16* qrow = Q + (bh * size_t(N) + (valid ? row : 0)) * D;
  for (int a = 0; a < D; ++a) xT[a * C::kMaxRows + t] = valid ? scale * __bfloat162float(qrow[a]) : 0.f;
  __syncthreads();

  float acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f, s_alpha = 0.f;

  for (int j = 0; j < nB; ++j) {
    const int s = j * block;
    const int n = min(block, N - s);
    const bool critical = (sMask[j >> 5] >> (j & 31)) & 1u;
    __syncthreads();  // previous tile fully consumed
    if (critical) {
      const bf16* gK = K + (bh * size_t(N) + s) * D;
      const bf16* gV = V + (bh * size_t(N) + s) * D;
      for (int e = t; e < n * D / 8; e += nthr) {
        reinterpret_cast<uint4*>(sK)[e] = reinterpret_cast<const uint4*>(gK)[e];
        reinterpret_cast<uint4*>(sV)[e] = reinterpret_cast<const uint4*>(gV)[e];
      }
      __syncthreads();
      for (int r = 0; r < n; ++r) {
        float z = 0.f;
#pragma unroll 8
        for (int a = 0; a < D; ++a) z = fmaf(xT[a * C::kMaxRows + t], __bfloat162float(sK[r * D + a]), z);
        if (z > m) {
          const float corr = __expf(m - z);
          l *= corr;
          s_alpha *= corr;
#pragma unroll
          for (int c = 0; c < D; ++c) acc[c] *= corr;
          m = z;
        }
        const float p = __expf(z - m);
        l += p;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = fmaf(p, __bfloat162float(sV[r * D + c]), acc[c]);
      }
    } else if (order >= 0) {
      const float* gkb = kbar + (bh * size_t(nB) + j) * D;
      const float* gs0 = S0 + (bh * size_t(nB) + j) * D;
      for (int e = t; e < D; e += nthr) {
        sKb[e] = gkb[e];
        sS0[e] = gs0[e];
      }
      if (order == 1) {
        const bf16* g1 = S1 + (bh * size_t(nB) + j) * size_t(D) * D;
        for (int e = t; e < D * D / 8; e += nthr)
          reinterpret_cast<uint4*>(sS1)[e] = reinterpret_cast<const uint4*>(g1)[e];
      }
      __syncthreads();
      float z = 0.f;
#pragma unroll 8
      for (int a = 0; a < D; ++a) z = fmaf(xT[a * C::kMaxRows + t], sKb[a], z);
      if (z > m) {
        const float corr = __expf(m - z);
        l *= corr;
        s_alpha *= corr;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] *= corr;
        m = z;
      }
      const float w = __expf(z - m);
      l += float(n) * w;
      s_alpha += w;
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = fmaf(w, sS0[c], acc[c]);
      if (order == 1) {
        for (int a = 0; a < D; ++a) {
          const float wx = w * xT[a * C::kMaxRows + t];
#pragma unroll
          for (int c = 0; c < D; ++c) acc[c] = fmaf(wx, __bfloat162float(sS1[a * D + c]), acc[c]);
        }
      }
    }
  }
  if (order == 2) {
    const float* gh = hbar + bh * size_t(D) * D;
    for (int a = 0; a < D; ++a) {
      const float sx = s_alpha * xT[a * C::kMaxRows + t];
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = fmaf(sx, __ldg(gh + a * D + c), acc[c]);
    }
  }
  if (valid) {
    const float inv = 1.f / l;
    bf16* orow = O + (bh * size_t(N) + row) * D;
#pragma unroll
    for (int c = 0; c < D; c += 2)
      *reinterpret_cast<uint32_t*>(orow + c) = pack_bf16x2(acc[c] * inv, acc[c + 1] * inv);
  }
}

}  // namespace pisa
