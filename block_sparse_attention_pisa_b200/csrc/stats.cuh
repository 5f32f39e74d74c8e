// Block statistics: kbar (centroid), S0 (value sum), S1 (first-order matrix).
//
// PISA explainer ("PISA: Piecewise Sparse Attention Is Wiser for Efficient
// Diffusion Transformers"), technical summary section 2, "Hardware
// implementation": the precompute step forms the block centroids and value sums
// before the fused kernel runs. S1_j = sum_n (k_n - kbar_j) v_n^T is the
// first-order Taylor matrix of block j.
//
// Each CTA takes G consecutive blocks of one head and streams them through two
// shared-memory buffers with cp.async: block j + 1 is in flight while block j is
// reduced and contracted, so HBM sees a continuous stream (16-byte coalesced
// copies into padded rows; rows past N are zero-filled). Per block:
//   - kbar_j and S0_j: column sums from shared memory (warp shuffles and a small
//     shared-memory pass);
//   - S1_j = K_j^T V_j - kbar_j S0_j^T: mma.sync bf16 tensor cores (the products
//     are exact, fp32 accumulation), two passes over halves of the value dimension.
//     Order 1 rounds each half once to bf16 and writes it with coalesced 16-byte
//     stores from a staging tile.
//
// The kernel is HBM-bound (K, V in; S1 out). The d x b x d contraction is ~32
// flop/byte, below the tensor ridge, so the warp-level mma.sync path keeps it
// under the memory time.
//
// Hybrid order (section 2, "Core algorithm": one global first-order statistic
// Hbar, the mean of the per-block first-order matrices over all blocks of a head;
// "Hardware implementation": formed in the precompute step). A cluster of
// kHbarCluster CTAs takes one head, CTA r the contiguous blocks
// [r nB / G, (r + 1) nB / G); each keeps the sum of its blocks' S1_j (fp32) in
// registers and stages it in its idle tile buffers. After a cluster barrier, CTA r
// sums its share of the rows over the G partials in rank order (distributed shared
// memory), scales by 1/nB and stores them. The split and every summation order depend
// on nB alone, so Hbar is the same bit for bit for any B, H, stream or device, and it
// needs no zeroing. Per-block S1 is never written.
#pragma once

#include "common.cuh"

namespace pisa {

template <int D, int BLK>
struct StatsCfg {
  static constexpr int kThreads = 256;
  static constexpr int kLd = D + 8;             // padded smem row (elements): conflict-free ldmatrix
  static constexpr int kChunks = D / 8;         // 16-byte chunks per row
  static constexpr int kRowStep = kThreads / kChunks;
  static constexpr int kTileElems = BLK * kLd;  // one of sK / sV
  static constexpr int kStageLd = D / 2 + 8;    // padded row of one value-dimension half of S1
  static constexpr size_t kSmem = size_t(2) * kTileElems * sizeof(bf16)  // sK, sV
                                  + size_t(D) * kStageLd * sizeof(bf16)  // S1 half staging
                                  + size_t(8) * 2 * D * sizeof(float)    // per-warp partial sums
                                  + size_t(2) * D * sizeof(float);       // kbar, S0
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One pass of K_j^T V_j over half of the value dimension on the tensor cores:
// acc (warp tile D/4 x D/4 of the key x value-half plane, 8 warps as 4 x 2) +=
// the block's products. Operands from the padded shared-memory tiles.
template <int D, int BLK>
__device__ __forceinline__ void s1_half_mma(uint32_t sK_u, uint32_t sV_u, int pass,
                                            float (&acc)[D / 64][D / 32][4]) {
  using C = StatsCfg<D, BLK>;
  constexpr int TM = D / 4, TN = D / 4;
  constexpr int MT = TM / 16, NT = TN / 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int a_base = (warp >> 1) * TM;
  const int c_base = pass * (D / 2) + (warp & 1) * TN;
#pragma unroll
  for (int kt = 0; kt < BLK / 16; ++kt) {
    uint32_t af[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      // A[a][n] = K[n][a]: transposed 8x8 loads from rows n, columns a
      const int row = kt * 16 + (lane & 7) + ((lane >> 4) << 3);
      const int col = a_base + mt * 16 + (((lane >> 3) & 1) << 3);
      ldsm_x4_trans(sK_u + (row * C::kLd + col) * 2, af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
    }
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      // B[n][c] = V[n][c]: two n8 tiles per x4 load
      const int row = kt * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
      const int col = c_base + np * 16 + ((lane >> 4) << 3);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(sV_u + (row * C::kLd + col) * 2, b0, b1, b2, b3);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        mma_bf16_16816(acc[mt][2 * np], af[mt], b0, b1);
        mma_bf16_16816(acc[mt][2 * np + 1], af[mt], b2, b3);
      }
    }
  }
}

// statistics modes: column sums only (orders 0, -1), per-block S1 (order 1), Hbar (order 2)
enum StatsMode { kStatsSums = 0, kStatsS1 = 1, kStatsHbar = 2 };

template <int D, int BLK>
struct StatsPipeCfg {
  using S = StatsCfg<D, BLK>;
  static constexpr int kTileBytes = S::kTileElems * 2;                     // one K or V tile
  static constexpr size_t kSmem = size_t(4) * kTileBytes                   // two buffers of (K, V)
                                  + size_t(D) * S::kStageLd * sizeof(bf16)  // S1 half staging
                                  + size_t(8) * 2 * D * sizeof(float)       // per-warp partial sums
                                  + size_t(2) * D * sizeof(float);          // kbar, S0
  static constexpr int blocks_per_cta(int mode) { return mode == kStatsHbar ? 8 : 4; }
};

template <int D, int BLK, int MODE>
__global__ void __launch_bounds__(256, 2)
stats_pipe_kernel(const bf16* __restrict__ K, const bf16* __restrict__ V, int N, int nB,
                  float* __restrict__ kbar, float* __restrict__ S0, bf16* __restrict__ S1,
                  float* __restrict__ Hbar) {
  using C = StatsCfg<D, BLK>;
  using P = StatsPipeCfg<D, BLK>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  bf16* sBuf = reinterpret_cast<bf16*>(smem_raw);                        // [2][K, V] tiles
  bf16* sStage = reinterpret_cast<bf16*>(smem_raw + 4 * P::kTileBytes);  // [D][kStageLd]
  float* sPart = reinterpret_cast<float*>(sStage + D * C::kStageLd);     // [8 warps][2][D]
  float* sKbar = sPart + 8 * 2 * D;
  float* sS0 = sKbar + D;

  constexpr int G = P::blocks_per_cta(MODE);
  constexpr int TM = D / 4, TN = D / 4;
  constexpr int MT = TM / 16, NT = TN / 8;
  const size_t bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ch = tid % C::kChunks;
  const int r0 = tid / C::kChunks;
  const int a_base = (warp >> 1) * TM;
  const int g = lane >> 2, t4 = lane & 3;
  // Hbar mode: the grid's x extent is the cluster, and x is the CTA's rank in it
  const int j0 = MODE == kStatsHbar ? int((int64_t(blockIdx.x) * nB) / kHbarCluster) : int(blockIdx.x) * G;
  const int j1 = MODE == kStatsHbar ? int((int64_t(blockIdx.x + 1) * nB) / kHbarCluster) : min(nB, j0 + G);
  const uint32_t buf_u = smem_u32(sBuf);

  // copies of block j into buffer b: thread (ch, r0) takes 16-byte chunk ch of rows
  // r0, r0 + kRowStep, ...; rows past N read nothing and are zero-filled
  auto issue = [&](int j, int b) {
    const int n = min(BLK, N - j * BLK);
    const bf16* gK = K + (bh * size_t(N) + size_t(j) * BLK) * D;
    const bf16* gV = V + (bh * size_t(N) + size_t(j) * BLK) * D;
    const uint32_t dK = buf_u + uint32_t(2 * b) * P::kTileBytes;
    const uint32_t dV = dK + P::kTileBytes;
#pragma unroll
    for (int r = r0; r < BLK; r += C::kRowStep) {
      const int rs = r < n ? r : 0;
      const uint32_t bytes = r < n ? 16u : 0u;
      const uint32_t off = uint32_t(r * C::kLd + ch * 8) * 2;
      cp_async16(dK + off, gK + size_t(rs) * D + ch * 8, bytes);
      cp_async16(dV + off, gV + size_t(rs) * D + ch * 8, bytes);
    }
    cp_async_commit();
  };

  float acc[2][MT][NT][4];
  if (MODE == kStatsHbar) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[h][mt][nt][e] = 0.f;
  }

  if (j0 < j1) issue(j0, 0);
#pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    const int b = (j - j0) & 1;
    if (j + 1 < j1) {
      issue(j + 1, b ^ 1);  // buffer b ^ 1 was released at the end of the previous block
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const bf16* sK = sBuf + size_t(2 * b) * C::kTileElems;
    const bf16* sV = sK + C::kTileElems;
    const int n = min(BLK, N - j * BLK);

    // ---- kbar_j, S0_j: column sums of the tiles ----
    {
      float ks[8], vs[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ks[e] = vs[e] = 0.f;
#pragma unroll
      for (int r = r0; r < BLK; r += C::kRowStep) {
        const uint4 kv = *reinterpret_cast<const uint4*>(sK + r * C::kLd + ch * 8);
        const uint4 vv = *reinterpret_cast<const uint4*>(sV + r * C::kLd + ch * 8);
        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
        const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          ks[2 * e] += bf16_lo(kw[e]);
          ks[2 * e + 1] += bf16_hi(kw[e]);
          vs[2 * e] += bf16_lo(vw[e]);
          vs[2 * e + 1] += bf16_hi(vw[e]);
        }
      }
      // lanes holding the same chunk index sit kChunks apart inside the warp
#pragma unroll
      for (int off = C::kChunks; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], off);
          vs[e] += __shfl_xor_sync(0xffffffffu, vs[e], off);
        }
      }
      if (lane < C::kChunks) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          sPart[(warp * 2 + 0) * D + ch * 8 + e] = ks[e];
          sPart[(warp * 2 + 1) * D + ch * 8 + e] = vs[e];
        }
      }
      __syncthreads();
      if (tid < 2 * D) {
        const int which = tid / D, col = tid % D;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += sPart[(w * 2 + which) * D + col];
        const size_t o = (bh * size_t(nB) + j) * D + col;
        if (which == 0) {
          const float kb = sum / float(n);
          sKbar[col] = kb;
          kbar[o] = kb;
        } else {
          sS0[col] = sum;
          S0[o] = sum;
        }
      }
      __syncthreads();
    }

    const uint32_t sK_u = smem_u32(sK), sV_u = smem_u32(sV);
    if (MODE == kStatsHbar) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        s1_half_mma<D, BLK>(sK_u, sV_u, h, acc[h]);
        const int c_base = h * (D / 2) + (warp & 1) * TN;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int a = a_base + mt * 16 + g;
          const float k0 = sKbar[a], k1 = sKbar[a + 8];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int c = c_base + nt * 8 + 2 * t4;
            const float s0 = sS0[c], s1 = sS0[c + 1];
            acc[h][mt][nt][0] -= k0 * s0;
            acc[h][mt][nt][1] -= k0 * s1;
            acc[h][mt][nt][2] -= k1 * s0;
            acc[h][mt][nt][3] -= k1 * s1;
          }
        }
      }
    } else if (MODE == kStatsS1) {
      bf16* gS1 = S1 + (bh * size_t(nB) + j) * D * D;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        const int c_base = pass * (D / 2) + (warp & 1) * TN;
        float hacc[MT][NT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) hacc[mt][nt][e] = 0.f;
        s1_half_mma<D, BLK>(sK_u, sV_u, pass, hacc);
        if (pass) __syncthreads();  // the previous half has been copied out of the staging tile
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int a = a_base + mt * 16 + g;
            const int c = c_base + nt * 8 + 2 * t4;  // global value column
            const int cl = c - pass * (D / 2);       // column inside the staged half
            const float k0 = sKbar[a], k1 = sKbar[a + 8];
            const float s0 = sS0[c], s1 = sS0[c + 1];
            *reinterpret_cast<uint32_t*>(sStage + a * C::kStageLd + cl) =
                pack_bf16x2(hacc[mt][nt][0] - k0 * s0, hacc[mt][nt][1] - k0 * s1);
            *reinterpret_cast<uint32_t*>(sStage + (a + 8) * C::kStageLd + cl) =
                pack_bf16x2(hacc[mt][nt][2] - k1 * s0, hacc[mt][nt][3] - k1 * s1);
          }
        }
        __syncthreads();
        // coalesced 16-byte stores of this half: D rows x (D/2) columns
        constexpr int HC = D / 16;  // 16-byte chunks per half row
#pragma unroll 4
        for (int q = tid; q < D * HC; q += C::kThreads) {
          const int a = q / HC, c8 = q % HC;
          *reinterpret_cast<uint4*>(gS1 + size_t(a) * D + pass * (D / 2) + c8 * 8) =
              *reinterpret_cast<const uint4*>(sStage + a * C::kStageLd + c8 * 8);
        }
      }
    }
    __syncthreads();  // this block's buffer, sums and staging tile are free again
  }

  if (MODE == kStatsHbar) {
    // the CTA's partial (zero for an empty slice) -> its idle tile buffers, [D][D + 4] fp32
    constexpr int PD = D + 4;
    static_assert(size_t(D) * PD * 4 <= size_t(4) * P::kTileBytes, "partial staging");
    float* sP = reinterpret_cast<float*>(smem_raw);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int a = a_base + mt * 16 + g;
          const int c = h * (D / 2) + (warp & 1) * TN + nt * 8 + 2 * t4;
          *reinterpret_cast<float2*>(sP + a * PD + c) = make_float2(acc[h][mt][nt][0], acc[h][mt][nt][1]);
          *reinterpret_cast<float2*>(sP + (a + 8) * PD + c) = make_float2(acc[h][mt][nt][2], acc[h][mt][nt][3]);
        }
    cluster_sync_all();  // every partial of the cluster is staged
    constexpr int ROWS = D / kHbarCluster;
    const int rank = int(blockIdx.x);
    const float inv = 1.f / float(nB);
    float* gH = Hbar + bh * size_t(D) * D;
    for (int i = tid; i < ROWS * (D / 4); i += C::kThreads) {
      const int a = rank * ROWS + i / (D / 4), q = i % (D / 4);
      const uint32_t off = smem_u32(sP + a * PD + 4 * q);
      float4 sum = ld_cluster_f4(cluster_map(off, 0));
#pragma unroll
      for (int src = 1; src < kHbarCluster; ++src) {
        const float4 v = ld_cluster_f4(cluster_map(off, uint32_t(src)));
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
      }
      *reinterpret_cast<float4*>(gH + size_t(a) * D + 4 * q) =
          make_float4(sum.x * inv, sum.y * inv, sum.z * inv, sum.w * inv);
    }
    cluster_sync_all();  // no CTA leaves while another still reads its partial
  }
}

}  // namespace pisa
