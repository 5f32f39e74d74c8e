// Critical-block selection: pooled-score rows and a per-row warp top-k.
//
// PISA explainer, technical summary section 2, "Covariance-aware routing": the
// blocks most relevant by attention score are routed to the exact path. The
// relevance of key block j to query block i is the pooled score
// qbar_i . kbar_j, with qbar_i the mean of the query block's real rows (fp32
// throughout, so that the ranking matches an exact evaluation except at
// near-ties).
//
// One CTA handles kQB consecutive query blocks of one head:
//   1. pool: stream the kQB query blocks once (16-byte coalesced loads) and
//      average their rows into qbar (fp32, shared memory);
//   2. score: one thread per key block j computes kQB dot products against
//      kbar_j (fp32 FMA, kbar read through the read-only cache; a head's kbar
//      is shared by all CTAs of that head and stays in L2);
//   3. top-k: one warp per row finds the k-th largest score key bit by bit
//      (a count of keys >= candidate per bit), then emits the selected block
//      indices in ascending order with ballots; among keys equal to the
//      threshold the lowest indices are taken.
#pragma once

#include "common.cuh"

namespace pisa {

constexpr int kSelectQB = 16;        // query blocks per CTA
constexpr int kSelectThreads = 256;

__host__ __device__ constexpr int select_score_ld(int nB) { return ((nB + 31) / 32) * 32 + 4; }

template <int D>
__global__ void __launch_bounds__(kSelectThreads)
select_kernel(const bf16* __restrict__ Q, const float* __restrict__ kbar, int N, int nB,
              int block, int topk, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* sQbar = reinterpret_cast<float*>(smem_raw);  // [kQB][D]
  float* sScore = sQbar + kSelectQB * D;                // [kQB][ld]
  const int ld = select_score_ld(nB);

  const size_t bh = blockIdx.y;
  const int i0 = blockIdx.x * kSelectQB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int CH = D / 8;

  // ---- 1. pooled queries ----
  for (int p = tid; p < kSelectQB * CH; p += kSelectThreads) {
    const int qb = p / CH, ch = p % CH;
    const int i = i0 + qb;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    int n = 0;
    if (i < nB) {
      const int s = i * block;
      n = min(block, N - s);
      const bf16* src = Q + (bh * size_t(N) + s) * D + ch * 8;
#pragma unroll 8
      for (int r = 0; r < n; ++r) {
        const uint4 w = ldg_stream_v4(src + size_t(r) * D);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += bf16_lo(ww[e]);
          acc[2 * e + 1] += bf16_hi(ww[e]);
        }
      }
    }
    const float inv = n > 0 ? 1.f / float(n) : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) sQbar[qb * D + ch * 8 + e] = acc[e] * inv;
  }
  __syncthreads();

  // ---- 2. pooled scores: thread per key block ----
  const float* kb_head = kbar + bh * size_t(nB) * D;
  for (int j = tid; j < nB; j += kSelectThreads) {
    float acc[kSelectQB];
#pragma unroll
    for (int q = 0; q < kSelectQB; ++q) acc[q] = 0.f;
    const float4* krow = reinterpret_cast<const float4*>(kb_head + size_t(j) * D);
#pragma unroll 4
    for (int a4 = 0; a4 < D / 4; ++a4) {
      const float4 k = __ldg(krow + a4);
#pragma unroll
      for (int q = 0; q < kSelectQB; ++q) {
        const float4 x = reinterpret_cast<const float4*>(sQbar + q * D)[a4];
        acc[q] = fmaf(x.x, k.x, acc[q]);
        acc[q] = fmaf(x.y, k.y, acc[q]);
        acc[q] = fmaf(x.z, k.z, acc[q]);
        acc[q] = fmaf(x.w, k.w, acc[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < kSelectQB; ++q) sScore[q * ld + j] = acc[q] + 0.f;  // -0 -> +0
  }
  __syncthreads();

  // ---- 3. top-k per row (one warp per row) ----
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int q = warp; q < kSelectQB; q += kSelectThreads / 32) {
    const int i = i0 + q;
    if (i >= nB) break;
    const float* row = sScore + q * ld;
    uint32_t T = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      unsigned cnt = 0;
      for (int jj = lane; jj < nB; jj += 32) cnt += float_order_key(row[jj]) >= cand;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= unsigned(topk)) T = cand;
    }
    unsigned gt = 0;
    for (int jj = lane; jj < nB; jj += 32) gt += float_order_key(row[jj]) > T;
    gt = __reduce_add_sync(0xffffffffu, gt);
    const int need_eq = topk - int(gt);
    int32_t* out = idx + (bh * size_t(nB) + i) * topk;
    int written = 0, eq_seen = 0;
    for (int base = 0; base < nB; base += 32) {
      const int jj = base + lane;
      const uint32_t key = jj < nB ? float_order_key(row[jj]) : 0u;
      const bool is_gt = jj < nB && key > T;
      const bool is_eq = jj < nB && key == T;
      const unsigned eq_mask = __ballot_sync(0xffffffffu, is_eq);
      const bool sel = is_gt || (is_eq && eq_seen + __popc(eq_mask & lt_mask) < need_eq);
      const unsigned sel_mask = __ballot_sync(0xffffffffu, sel);
      if (sel) out[written + __popc(sel_mask & lt_mask)] = jj;
      written += __popc(sel_mask);
      eq_seen += __popc(eq_mask);
    }
  }
}

inline size_t select_smem_bytes(int D, int nB) {
  return size_t(kSelectQB) * D * sizeof(float) + size_t(kSelectQB) * select_score_ld(nB) * sizeof(float);
}

}  // namespace pisa
