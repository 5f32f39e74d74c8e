// Critical-block selection: pooled-score rows and a per-row warp top-k.
//
// PISA explainer, technical summary section 2, "Covariance-aware routing": the
// blocks most relevant by attention score are routed to the exact path. The
// relevance of key block j to query block i is the pooled score
// qbar_i . kbar_j, with qbar_i the mean of the query block's real rows (fp32
// throughout, so that the ranking matches an exact evaluation except at
// near-ties). With covariance-aware routing (same paragraph) each key block's
// score also carries lambda * M_j, M_j = || S1_j - Hbar ||_F (routing.cuh).
//
// One CTA handles kSelectQB consecutive query blocks of one head:
//   1. pool: stream the query blocks once (16-byte coalesced loads, two row
//      halves per (block, 16-byte column) pair) and average their rows into
//      qbar (fp32, shared memory);
//   2. score: each warp takes 32 consecutive key blocks per pass (lane = key block).
//      Their kbar rows (L2-resident: a head's kbar is shared by all its CTAs)
//      stream through two per-warp shared-memory tiles 16 dimensions at a time, with
//      coalesced 16-byte cp.async copies (eight rows per instruction; the next slab is
//      in flight while the current one is used); each lane then forms
//      kSelectQB fp32 dot products against its own row (conflict-free 16-byte shared
//      reads, query rows broadcast). Scores are stored as order-preserving uint32 keys;
//   3. top-k: one warp per row finds the k-th largest key bit by bit (a count of
//      keys >= candidate per bit, starting below the row's common key prefix),
//      then emits the selected block indices in ascending order with ballots;
//      among keys equal to the threshold the lowest indices are taken.
#pragma once

#include "common.cuh"

namespace pisa {

constexpr int kSelectQB = 8;         // query blocks per CTA
constexpr int kSelectThreads = 256;
constexpr int kSelectSlab = 16;                           // kbar dimensions per tile pass
constexpr int kSelectTileLd = kSelectSlab + 4;            // padded tile row (floats)
constexpr int kSelectTileFloats = 2 * 32 * kSelectTileLd;  // one warp's two tiles

__host__ __device__ constexpr int select_score_ld(int nB) { return ((nB + 31) / 32) * 32 + 4; }

template <int D>
__global__ void __launch_bounds__(kSelectThreads)
select_kernel(const bf16* __restrict__ Q, const float* __restrict__ kbar, const float* __restrict__ route,
              float lambda, int N, int nB, int block, int topk, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* sQbar = reinterpret_cast<float*>(smem_raw);                    // [QB][D]
  float* sHalf = sQbar + kSelectQB * D;                                 // [QB][D] second-half row sums
  uint32_t* sKey = reinterpret_cast<uint32_t*>(sHalf + kSelectQB * D);  // [QB][ld]
  const int ld = select_score_ld(nB);
  float* sTile = reinterpret_cast<float*>(sKey + kSelectQB * ld);        // [8 warps][32][TileLd]

  const size_t bh = blockIdx.y;
  const int i0 = blockIdx.x * kSelectQB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int CH = D / 8;

  // ---- 1. pooled queries: item = (query block, 16-byte column, row half) ----
  for (int p = tid; p < kSelectQB * CH * 2; p += kSelectThreads) {
    const int half = p / (kSelectQB * CH);
    const int qb = (p / CH) % kSelectQB, ch = p % CH;
    const int i = i0 + qb;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (i < nB) {
      const int s = i * block;
      const int n = min(block, N - s);
      const int r0 = half ? (n + 1) / 2 : 0, r1 = half ? n : (n + 1) / 2;
      const bf16* src = Q + (bh * size_t(N) + s) * D + ch * 8;
#pragma unroll 8
      for (int r = r0; r < r1; ++r) {
        const uint4 w = ldg_stream_v4(src + size_t(r) * D);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += bf16_lo(ww[e]);
          acc[2 * e + 1] += bf16_hi(ww[e]);
        }
      }
    }
    float* dst = (half ? sHalf : sQbar) + qb * D + ch * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e] = acc[e];
  }
  __syncthreads();
  for (int p = tid; p < kSelectQB * D; p += kSelectThreads) {
    const int i = i0 + p / D;
    const int n = i < nB ? min(block, N - i * block) : 1;
    sQbar[p] = (sQbar[p] + sHalf[p]) * (1.f / float(n));
  }
  __syncthreads();

  // ---- 2. pooled scores: lane = key block, kbar rows through per-warp tiles ----
  {
    const float* kb_head = kbar + bh * size_t(nB) * D;
    float* tiles = sTile + warp * kSelectTileFloats;
    const uint32_t tiles_u = smem_u32(tiles);
    constexpr int NSLAB = D / kSelectSlab;
    for (int jb = warp * 32; jb < nB; jb += kSelectThreads) {
      // rows (lane >> 2) + 8 i, 16-byte chunk (lane & 3) of the slab; rows past nB are
      // zero-filled
      auto issue = [&](int sl) {
        const uint32_t dst = tiles_u + uint32_t((sl & 1) * 32 * kSelectTileLd) * 4u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = (lane >> 2) + 8 * i;
          const bool in = jb + r < nB;
          const float* src = kb_head + size_t(in ? jb + r : 0) * D + sl * kSelectSlab + (lane & 3) * 4;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst + uint32_t(r * kSelectTileLd + (lane & 3) * 4) * 4u),
                       "l"(src), "r"(in ? 16u : 0u)
                       : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      };
      float acc[kSelectQB];
#pragma unroll
      for (int q = 0; q < kSelectQB; ++q) acc[q] = 0.f;
      issue(0);
#pragma unroll 1
      for (int sl = 0; sl < NSLAB; ++sl) {
        if (sl + 1 < NSLAB) {
          issue(sl + 1);
          asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
          asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncwarp();
        const float4* krow = reinterpret_cast<const float4*>(tiles + (sl & 1) * 32 * kSelectTileLd + lane * kSelectTileLd);
        const int d0 = sl * kSelectSlab;
#pragma unroll
        for (int c = 0; c < kSelectSlab / 4; ++c) {
          const float4 k = krow[c];
#pragma unroll
          for (int q = 0; q < kSelectQB; ++q) {
            const float4 x = reinterpret_cast<const float4*>(sQbar + q * D + d0)[c];
            acc[q] = fmaf(x.x, k.x, acc[q]);
            acc[q] = fmaf(x.y, k.y, acc[q]);
            acc[q] = fmaf(x.z, k.z, acc[q]);
            acc[q] = fmaf(x.w, k.w, acc[q]);
          }
        }
        __syncwarp();  // this tile is refilled two slabs later
      }
      const int j = jb + lane;
      if (j < nB) {
        const float bias = route != nullptr ? lambda * route[bh * size_t(nB) + j] : 0.f;
#pragma unroll
        for (int q = 0; q < kSelectQB; ++q) sKey[q * ld + j] = float_order_key(acc[q] + bias + 0.f);  // -0 -> +0
      }
    }
  }
  __syncthreads();

  // ---- 3. top-k per row (one warp per row) ----
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int q = warp; q < kSelectQB; q += kSelectThreads / 32) {
    const int i = i0 + q;
    if (i >= nB) break;
    const uint32_t* row = sKey + q * ld;
    // the k-th largest key lies between the row's extremes: bits above their
    // first difference are common to every candidate threshold
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int jj = lane; jj < nB; jj += 32) {
      const uint32_t k = row[jj];
      kmin = min(kmin, k);
      kmax = max(kmax, k);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    const uint32_t diff = kmin ^ kmax;
    const int top = diff ? 31 - __clz(diff) : -1;  // highest differing bit
    uint32_t T = top < 0 ? kmax : (top >= 31 ? 0u : (kmax & ~((2u << top) - 1u)));
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      unsigned cnt = 0;
      for (int jj = lane; jj < nB; jj += 32) cnt += row[jj] >= cand;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= unsigned(topk)) T = cand;
    }
    unsigned gt = 0;
    for (int jj = lane; jj < nB; jj += 32) gt += row[jj] > T;
    gt = __reduce_add_sync(0xffffffffu, gt);
    const int need_eq = topk - int(gt);
    int32_t* out = idx + (bh * size_t(nB) + i) * topk;
    int written = 0, eq_seen = 0;
    for (int base = 0; base < nB; base += 32) {
      const int jj = base + lane;
      const uint32_t key = jj < nB ? row[jj] : 0u;
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
  return size_t(2) * kSelectQB * D * sizeof(float) + size_t(kSelectQB) * select_score_ld(nB) * sizeof(uint32_t) +
         size_t(kSelectThreads / 32) * kSelectTileFloats * sizeof(float);
}

}  // namespace pisa
