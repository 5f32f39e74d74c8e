// Block statistics on the 5th-generation tensor cores (d = 128): kbar, S0 and either the
// per-block first-order matrix S1 (stats_tc_kernel) or the head's Hbar (stats_hbar_kernel).
//
// PISA explainer, technical summary section 2, "Hardware implementation": the
// precompute step forms block centroids and value sums; "Core algorithm": the
// first-order Taylor matrix of block j is S1_j = sum_n (k_n - kbar_j) v_n^T, and the
// hybrid order uses their mean over the head's blocks, Hbar.
//
// S1_j = K_j^T V_j - kbar_j S0_j^T. K_j^T V_j is one M128 x N128 x K=b contraction per
// block with both operands straight from the TMA tiles: K_j stored [token][key dim] is
// an MN-major A operand, V_j stored [token][value dim] an MN-major B operand.
//
// stats_tc_kernel: persistent CTAs walk the blocks of all heads. Warp roles:
//   warp 0     TMA producer: K_j and V_j (128-byte swizzled 64-column panels, rows past
//              N zero-filled) into a ring of stages;
//   warp 1     MMA issuer (one thread): K_j^T V_j into one of two TMEM accumulators;
//   warps 8-11 column sums from the stage, one 64-column panel of K or V each: kbar_j
//              (mean of the real rows) and S0_j, to global memory and to shared memory
//              for the epilogue;
//   warps 4-7  epilogue, one TMEM lane (= key dimension a) per thread: subtracts
//              kbar_j[a] S0_j[c], rounds to bf16 into a swizzled staging tile and writes
//              it with TMA stores.
// Every wait is bounded (about a second); on timeout the CTA raises the device error
// word, stops issuing work, drains what it issued and frees TMEM.
#pragma once

#include "tc_ptx.cuh"

namespace pisa {

template <int BLK>
struct StatsTcCfg {
  static constexpr int D = 128;
  static constexpr int kThreads = 384;
  static constexpr int STAGE = 2 * BLK * D * 2;                    // K and V tiles
  static constexpr int STG = D * D * 2;                            // bf16 S1 staging tile
  static constexpr int NSTG = 2;                                   // staging tiles
  static constexpr int STATS = 2 * D * 4;                          // kbar + S0 of one block
  static constexpr int NSTATS = 2;                                 // stats slots
  static constexpr int FIXED = NSTG * STG + NSTATS * STATS + 1024; // + barriers / misc
  static constexpr int NS = (227 * 1024 - 1024 - FIXED) / STAGE;   // ring stages
  static_assert(NS >= 2, "ring");
  // barriers
  static constexpr int B_FULL = 0;              // [NS] stage landed (TMA tx)
  static constexpr int B_EMPTY = B_FULL + NS;   // [NS] stage consumed (MMA commit + 4 sum warps)
  static constexpr int B_AFULL = B_EMPTY + NS;  // [2]  accumulator ready (commit)
  static constexpr int B_AEMPTY = B_AFULL + 2;  // [2]  accumulator and stats slot read (4 warps)
  static constexpr int B_SFULL = B_AEMPTY + 2;  // [2]  kbar / S0 in shared memory (4 warps)
  static constexpr int B_DONE = B_SFULL + 2;    //      every MMA finished (commit)
  static constexpr int NBARS = B_DONE + 1;
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_STG = OFF_RING + NS * STAGE;
  static constexpr int OFF_STATS = OFF_STG + NSTG * STG;
  static constexpr int OFF_BAR = OFF_STATS + NSTATS * STATS;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static constexpr int TMEM_COLS = 256;          // two fp32 accumulators of D columns
};

namespace tc {

// 3-D TMA store of a shared-memory tile (bulk-group completion)
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// named barrier over the four epilogue warps
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

}  // namespace tc

// per-block S1 (order 1), d = 128
template <int BLK>
__global__ void __launch_bounds__(384, 1)
stats_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmS1, int N, int nB, int total_blocks,
                float* __restrict__ kbar, float* __restrict__ S0) {
  using C = StatsTcCfg<BLK>;
  using namespace tc;
  constexpr int D = C::D;
  extern __shared__ __align__(16) uint8_t st_smem_raw[];
  const uint32_t raw_u = smem_u32(st_smem_raw);
  const uint32_t base_u = (raw_u + 1023u) & ~1023u;
  uint8_t* base = st_smem_raw + (base_u - raw_u);
  float* stats = reinterpret_cast<float*>(base + C::OFF_STATS);  // [NSTATS][kbar D, S0 D]
  int* misc = reinterpret_cast<int*>(base + C::OFF_MISC);       // tmem address, abort flag
  volatile int* abort_flag = misc + 1;
  const uint32_t bar0 = base_u + C::OFF_BAR;
#define SBAR(i) (bar0 + 8u * uint32_t(i))
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA-local block sequence t -> global block index blockIdx.x + t * gridDim.x
  const int nblocks = total_blocks > int(blockIdx.x) ? (total_blocks - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  auto block_of = [&](int t, int* bh, int* j) {
    const int u = int(blockIdx.x) + t * int(gridDim.x);
    *bh = u / nB;
    *j = u % nB;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(SBAR(C::B_FULL + s), 1);
      mbar_init(SBAR(C::B_EMPTY + s), 5);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(SBAR(C::B_AFULL + b), 1);
      mbar_init(SBAR(C::B_AEMPTY + b), 4);
      mbar_init(SBAR(C::B_SFULL + b), 4);
    }
    mbar_init(SBAR(C::B_DONE), 1);
    misc[1] = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(base_u + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = uint32_t(misc[0]);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // lanes 0 and 1 issue together (K panels, V panels): one issuing thread delivers
    // about 35-40 B/clk into an SM, two about 60
    if (lane < 2) {
      int t = 0;
      for (; t < nblocks; ++t) {
        const int s = t % C::NS;
        const bool ok = wait_bounded(SBAR(C::B_EMPTY + s), ((t / C::NS) & 1) ^ 1, abort_flag);
        if (!__all_sync(0x3u, ok)) break;
        int bh, j;
        block_of(t, &bh, &j);
        const uint32_t dst = base_u + C::OFF_RING + s * C::STAGE + lane * (BLK * D * 2);
        const uint32_t full = SBAR(C::B_FULL + s);
        if (lane == 0) mbar_arrive_expect_tx(full, C::STAGE);
        __syncwarp(0x3u);
#pragma unroll
        for (int p = 0; p < D / 64; ++p) tma_load_3d(dst + p * BLK * 128, lane ? &tmV : &tmK, full, p * 64, j * BLK, bh);
      }
      // no copy may be in flight when the CTA exits
      if (lane == 0)
        for (int v = t > C::NS ? t - C::NS : 0; v < t; ++v) wait_drain(SBAR(C::B_FULL + v % C::NS), (v / C::NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // S1 partial = K^T V: A = K (MN-major, M = key dims), B = V (MN-major, N = value dims)
      constexpr uint32_t idS = idesc_bf16(128, D, true) | (1u << 15);
      for (int t = 0; t < nblocks; ++t) {
        const int ab = t & 1;  // accumulator of this block
        if (!wait_poll(SBAR(C::B_AEMPTY + ab), ((t >> 1) & 1) ^ 1, abort_flag)) break;
        const int s = t % C::NS;
        if (!wait_poll(SBAR(C::B_FULL + s), (t / C::NS) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t kb = base_u + C::OFF_RING + s * C::STAGE;
        const uint32_t vb = kb + BLK * D * 2;
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk)
          umma_ss(tmem + ab * D, sdesc_sw128(kb + kk * 2048, BLK * 128, 1024),
                  sdesc_sw128(vb + kk * 2048, BLK * 128, 1024), idS, kk ? 1u : 0u);
        umma_commit(SBAR(C::B_EMPTY + s));
        umma_commit(SBAR(C::B_AFULL + ab));
      }
      // nothing of ours may run on after the CTA frees TMEM
      umma_commit(SBAR(C::B_DONE));
      wait_drain(SBAR(C::B_DONE), 0);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ column sums
    // warp 8 + 2 isV + panel: one 64-column panel of K or V; lane = 16-byte chunk lane % 8
    // of the panel and row phase lane / 8 (rows lane / 8, + 4, + 8, ...)
    const bool isV = warp >= 10;
    const int panel = warp & 1;
    const int qc = lane & 7, r0 = lane >> 3;
    for (int t = 0; t < nblocks; ++t) {
      const int s = t % C::NS;
      if (*abort_flag || !__all_sync(0xffffffffu, wait_bounded(SBAR(C::B_FULL + s), (t / C::NS) & 1, abort_flag)))
        break;
      int bh, j;
      block_of(t, &bh, &j);
      const int n = min(BLK, N - j * BLK);
      const uint8_t* tile = base + C::OFF_RING + s * C::STAGE + (isV ? BLK * D * 2 : 0) + panel * BLK * 128;
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int r = r0; r < BLK; r += 4) {  // zero-filled rows past N add nothing (all loads in flight)
        const uint4 w = *reinterpret_cast<const uint4*>(tile + r * 128 + ((qc ^ (r & 7)) << 4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += bf16_lo(ww[e]);
          acc[2 * e + 1] += bf16_hi(ww[e]);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
      }
      warp_arrive(SBAR(C::B_EMPTY + s));  // one arrival per warp (the count is 1 commit + 4 warps)
      const int q16 = panel * 8 + qc;      // 16-byte chunk of the row (8 columns)
      // stats slot t & 1 was read by the epilogue of block t - 2
      if (t >= 2 &&
          !__all_sync(0xffffffffu, wait_bounded(SBAR(C::B_AEMPTY + (t & 1)), ((t >> 1) & 1) ^ 1, abort_flag)))
        break;
      if (lane < 8) {
        float* dst_s = stats + (t & 1) * 2 * D + (isV ? D : 0) + q16 * 8;
        const float f = isV ? 1.f : 1.f / float(n);
        float4 v0 = make_float4(acc[0] * f, acc[1] * f, acc[2] * f, acc[3] * f);
        float4 v1 = make_float4(acc[4] * f, acc[5] * f, acc[6] * f, acc[7] * f);
        reinterpret_cast<float4*>(dst_s)[0] = v0;
        reinterpret_cast<float4*>(dst_s)[1] = v1;
        float* dst_g = (isV ? S0 : kbar) + (size_t(bh) * nB + j) * D + q16 * 8;
        reinterpret_cast<float4*>(dst_g)[0] = v0;
        reinterpret_cast<float4*>(dst_g)[1] = v1;
      }
      warp_arrive(SBAR(C::B_SFULL + (t & 1)));  // one per warp
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (warps 4-7; 2-3 idle)
    const int et = threadIdx.x - 128;  // = TMEM lane = key dimension a
    const int quarter = warp & 3;
    const uint32_t lrow = uint32_t(quarter * 32) << 16;
    const int a = et;
    bool ok = true;
    // the four warps meet at two named barriers per block; a warp whose wait ran out
    // keeps meeting them (skipping the work), so that no warp is left waiting
    for (int t = 0; t < nblocks; ++t) {
      const int ab = t & 1;
      if (ok)
        ok = __all_sync(0xffffffffu, wait_bounded(SBAR(C::B_AFULL + ab), (t >> 1) & 1, abort_flag)) &&
             __all_sync(0xffffffffu, wait_bounded(SBAR(C::B_SFULL + ab), (t >> 1) & 1, abort_flag));
      tc_fence_after();
      int bh, j;
      block_of(t, &bh, &j);
      const float* st = stats + ab * 2 * D;
      const float ka = st[a];
      const uint32_t stg = base_u + C::OFF_STG + ab * C::STG;
      // the TMA store of two blocks ago read this staging tile
      if (et == 0) bulk_wait_read<1>();
      epi_sync();
#pragma unroll
      for (int ch = 0; ch < D / 16 && ok; ++ch) {
        uint32_t r[16];
        tmem_ld16(tmem + lrow + ab * D + ch * 16, r);
        tmem_wait_ld(r);
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = ch * 16 + 2 * e;
          w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) - ka * st[D + c],
                             __uint_as_float(r[2 * e + 1]) - ka * st[D + c + 1]);
        }
        // [panel][row a][16-byte chunk ^ (a & 7)]: the layout a 128-byte swizzled TMA moves
        const int q0 = (ch & 3) * 2, p = ch >> 2;
        uint8_t* rowp = base + (stg - base_u) + p * (D * 128) + a * 128;
        *reinterpret_cast<uint4*>(rowp + (((q0) ^ (a & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(rowp + (((q0 + 1) ^ (a & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
      }
      tc_fence_before();
      if (ok) warp_arrive(SBAR(C::B_AEMPTY + ab));  // accumulator and stats slot are free
      fence_proxy_async_smem();
      epi_sync();
      if (et == 0 && *abort_flag == 0) {
#pragma unroll
        for (int p = 0; p < D / 64; ++p) tma_store_3d(&tmS1, stg + p * (D * 128), p * 64, 0, bh * nB + j);
        bulk_commit();
      }
    }
    if (et == 0) bulk_wait_all();  // the last stores have landed
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
#undef SBAR
}

// ---------------------------------------------------------------------------------------
// Hbar of every head (d = 128), reproducible bit for bit.
//
// Hbar = (1/nB) sum_j S1_j = (1/nB) (sum_j K_j^T V_j - sum_j kbar_j S0_j^T). A cluster of
// kHbarCluster CTAs takes one head; CTA r takes the contiguous blocks
// [r nB / G, (r + 1) nB / G). The split depends on nB alone, and so does every
// summation order below: the result is the same for any B, H, stream or device.
//   warp 0, lanes 0-1  TMA producer: K_j and V_j of the slice into a ring of stages;
//   warp 1             MMA issuer: every K_j^T V_j of the slice into one TMEM accumulator;
//   warps 8-11         column sums: kbar_j, S0_j to global memory and to a ring of slots;
//   warps 4-7          thread a (= key dimension, = TMEM lane) keeps row a of
//                      sum_j kbar_j S0_j^T in registers, taking each block's slot in turn;
//                      at the end it writes row a of (accumulator - that sum) to shared
//                      memory.
// After a cluster barrier, CTA r sums rows [32 r, 32 r + 32) of the G partials in rank
// order through distributed shared memory, scales by 1/nB and stores them: no atomics,
// and Hbar needs no zeroing. Every mbarrier wait is bounded; every thread reaches both
// cluster barriers, whatever happened before.
template <int BLK>
struct StatsHbarCfg {
  static constexpr int D = 128;
  static constexpr int kThreads = 384;
  static constexpr int G = kHbarCluster;
  static constexpr int STAGE = 2 * BLK * D * 2;                  // K and V tiles
  static constexpr int NSL = 8;                                  // kbar / S0 slots
  static constexpr int SLOT = 2 * D * 4;
  static constexpr int PART = D * D * 4;                         // fp32 partial, staged in the ring
  static constexpr int NS = (227 * 1024 - 3 * 1024 - NSL * SLOT) / STAGE;
  static_assert(NS >= 2 && NS * STAGE >= PART, "ring");
  static constexpr int B_FULL = 0;              // [NS]  stage landed (TMA tx)
  static constexpr int B_EMPTY = B_FULL + NS;   // [NS]  stage read (MMA commit + 4 sum warps)
  static constexpr int B_SFULL = B_EMPTY + NS;  // [NSL] slot written (4 sum warps)
  static constexpr int B_SEMPTY = B_SFULL + NSL;  // [NSL] slot read (4 epilogue warps)
  static constexpr int B_DONE = B_SEMPTY + NSL;   //       every MMA finished (commit)
  static constexpr int NBARS = B_DONE + 1;
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_SLOT = OFF_RING + NS * STAGE;
  static constexpr int OFF_BAR = OFF_SLOT + NSL * SLOT;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static constexpr int TMEM_COLS = 128;
  static_assert(D % G == 0, "rows per CTA");
};

template <int BLK>
__global__ void __launch_bounds__(384, 1)
stats_hbar_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, int N, int nB,
                  float* __restrict__ kbar, float* __restrict__ S0, float* __restrict__ Hbar) {
  using C = StatsHbarCfg<BLK>;
  using namespace tc;
  constexpr int D = C::D;
  extern __shared__ __align__(16) uint8_t hb_smem_raw[];
  const uint32_t raw_u = smem_u32(hb_smem_raw);
  const uint32_t base_u = (raw_u + 1023u) & ~1023u;
  uint8_t* base = hb_smem_raw + (base_u - raw_u);
  float* slots = reinterpret_cast<float*>(base + C::OFF_SLOT);  // [NSL][kbar D, S0 D]
  int* misc = reinterpret_cast<int*>(base + C::OFF_MISC);      // tmem address, abort flag
  volatile int* abort_flag = misc + 1;
  const uint32_t bar0 = base_u + C::OFF_BAR;
#define HBAR_BAR(i) (bar0 + 8u * uint32_t(i))
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = int(blockIdx.x);  // the grid's x extent is the cluster
  const int bh = int(blockIdx.y);
  const int j0 = int((int64_t(rank) * nB) / C::G), j1 = int((int64_t(rank + 1) * nB) / C::G);
  const int nb = j1 - j0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(HBAR_BAR(C::B_FULL + s), 1);
      mbar_init(HBAR_BAR(C::B_EMPTY + s), 5);
    }
    for (int k = 0; k < C::NSL; ++k) {
      mbar_init(HBAR_BAR(C::B_SFULL + k), 4);
      mbar_init(HBAR_BAR(C::B_SEMPTY + k), 4);
    }
    mbar_init(HBAR_BAR(C::B_DONE), 1);
    misc[1] = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(base_u + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = uint32_t(misc[0]);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane < 2) {
      int t = 0;
      for (; t < nb; ++t) {
        const int s = t % C::NS;
        const bool ok = wait_bounded(HBAR_BAR(C::B_EMPTY + s), ((t / C::NS) & 1) ^ 1, abort_flag);
        if (!__all_sync(0x3u, ok)) break;
        const uint32_t dst = base_u + C::OFF_RING + s * C::STAGE + lane * (BLK * D * 2);
        const uint32_t full = HBAR_BAR(C::B_FULL + s);
        if (lane == 0) mbar_arrive_expect_tx(full, C::STAGE);
        __syncwarp(0x3u);
#pragma unroll
        for (int p = 0; p < D / 64; ++p)
          tma_load_3d(dst + p * BLK * 128, lane ? &tmV : &tmK, full, p * 64, (j0 + t) * BLK, bh);
      }
      if (lane == 0)
        for (int v = t > C::NS ? t - C::NS : 0; v < t; ++v)
          wait_drain(HBAR_BAR(C::B_FULL + v % C::NS), (v / C::NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // K_j^T V_j: A = K (MN-major, M = key dims), B = V (MN-major, N = value dims)
      constexpr uint32_t idS = idesc_bf16(128, D, true) | (1u << 15);
      for (int t = 0; t < nb; ++t) {
        const int s = t % C::NS;
        if (!wait_poll(HBAR_BAR(C::B_FULL + s), (t / C::NS) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t kb = base_u + C::OFF_RING + s * C::STAGE;
        const uint32_t vb = kb + BLK * D * 2;
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk)
          umma_ss(tmem, sdesc_sw128(kb + kk * 2048, BLK * 128, 1024), sdesc_sw128(vb + kk * 2048, BLK * 128, 1024),
                  idS, (t | kk) ? 1u : 0u);
        umma_commit(HBAR_BAR(C::B_EMPTY + s));
      }
      // the epilogue reads the accumulator after this; nothing of ours runs on after it
      umma_commit(HBAR_BAR(C::B_DONE));
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ column sums
    // warp 8 + 2 isV + panel: one 64-column panel of K or V; lane = 16-byte chunk lane % 8
    // of the panel and row phase lane / 8
    const bool isV = warp >= 10;
    const int panel = warp & 1;
    const int qc = lane & 7, r0 = lane >> 3;
    for (int t = 0; t < nb; ++t) {
      const int s = t % C::NS;
      if (!__all_sync(0xffffffffu, wait_bounded(HBAR_BAR(C::B_FULL + s), (t / C::NS) & 1, abort_flag))) break;
      const int j = j0 + t;
      const int n = min(BLK, N - j * BLK);
      const uint8_t* tile = base + C::OFF_RING + s * C::STAGE + (isV ? BLK * D * 2 : 0) + panel * BLK * 128;
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int r = r0; r < BLK; r += 4) {  // zero-filled rows past N add nothing (all loads in flight)
        const uint4 w = *reinterpret_cast<const uint4*>(tile + r * 128 + ((qc ^ (r & 7)) << 4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += bf16_lo(ww[e]);
          acc[2 * e + 1] += bf16_hi(ww[e]);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
      }
      warp_arrive(HBAR_BAR(C::B_EMPTY + s));
      const int k = t % C::NSL;
      if (t >= C::NSL &&
          !__all_sync(0xffffffffu, wait_bounded(HBAR_BAR(C::B_SEMPTY + k), ((t / C::NSL) & 1) ^ 1, abort_flag)))
        break;
      if (lane < 8) {
        const int q16 = panel * 8 + qc;  // 16-byte chunk of the row (8 columns)
        const float f = isV ? 1.f : 1.f / float(n);
        const float4 v0 = make_float4(acc[0] * f, acc[1] * f, acc[2] * f, acc[3] * f);
        const float4 v1 = make_float4(acc[4] * f, acc[5] * f, acc[6] * f, acc[7] * f);
        float* dst_s = slots + k * 2 * D + (isV ? D : 0) + q16 * 8;
        reinterpret_cast<float4*>(dst_s)[0] = v0;
        reinterpret_cast<float4*>(dst_s)[1] = v1;
        float* dst_g = (isV ? S0 : kbar) + (size_t(bh) * nB + j) * D + q16 * 8;
        reinterpret_cast<float4*>(dst_g)[0] = v0;
        reinterpret_cast<float4*>(dst_g)[1] = v1;
      }
      warp_arrive(HBAR_BAR(C::B_SFULL + k));
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ correction and partial
    const int a = int(threadIdx.x) - 128;  // = TMEM lane = key dimension
    const uint32_t lrow = uint32_t((warp & 3) * 32) << 16;
    float corr[D];  // row a of sum_j kbar_j S0_j^T over the slice
#pragma unroll
    for (int c = 0; c < D; ++c) corr[c] = 0.f;
    bool ok = true;
    for (int t = 0; t < nb; ++t) {
      const int k = t % C::NSL;
      if (!(ok = __all_sync(0xffffffffu, wait_bounded(HBAR_BAR(C::B_SFULL + k), (t / C::NSL) & 1, abort_flag))))
        break;
      const float* sl = slots + k * 2 * D;
      const float ka = sl[a];
#pragma unroll
      for (int c = 0; c < D; c += 4) {
        const float4 s0 = *reinterpret_cast<const float4*>(sl + D + c);
        corr[c] = fmaf(ka, s0.x, corr[c]);
        corr[c + 1] = fmaf(ka, s0.y, corr[c + 1]);
        corr[c + 2] = fmaf(ka, s0.z, corr[c + 2]);
        corr[c + 3] = fmaf(ka, s0.w, corr[c + 3]);
      }
      warp_arrive(HBAR_BAR(C::B_SEMPTY + k));
    }
    // every MMA of the slice has completed once B_DONE has
    if (ok && nb > 0) ok = __all_sync(0xffffffffu, wait_bounded(HBAR_BAR(C::B_DONE), 0, abort_flag));
    tc_fence_after();
    // partial row a -> ring bytes [0, 64 KB): 512-byte rows, 16-byte chunk q at q ^ (a & 7)
    // (the ring is idle: every copy has landed and been read once B_DONE has completed)
    uint8_t* prow = base + C::OFF_RING + a * (D * 4);
#pragma unroll
    for (int ch = 0; ch < D / 16; ++ch) {
      uint32_t r[16];
      if (ok && nb > 0) {
        tmem_ld16(tmem + lrow + ch * 16, r);
        tmem_wait_ld(r);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = 0u;
      }
#pragma unroll
      for (int e4 = 0; e4 < 4; ++e4) {
        const int q = ch * 4 + e4, c = q * 4;
        *reinterpret_cast<float4*>(prow + ((q ^ (a & 7)) << 4)) =
            make_float4(__uint_as_float(r[4 * e4]) - corr[c], __uint_as_float(r[4 * e4 + 1]) - corr[c + 1],
                        __uint_as_float(r[4 * e4 + 2]) - corr[c + 2], __uint_as_float(r[4 * e4 + 3]) - corr[c + 3]);
      }
    }
    tc_fence_before();
  }

  // ---------------------------------------------------------------- cluster reduction
  __syncthreads();
  if (warp == 1 && lane == 0) wait_drain(HBAR_BAR(C::B_DONE), 0);  // no MMA still running
  __syncthreads();
  cluster_sync_all();  // every partial of the cluster is staged
  {
    constexpr int ROWS = D / C::G;
    const float inv = 1.f / float(nB);
    const uint32_t part_u = base_u + C::OFF_RING;
    float* gH = Hbar + size_t(bh) * D * D;
    for (int i = int(threadIdx.x); i < ROWS * (D / 4); i += C::kThreads) {
      const int a = rank * ROWS + i / (D / 4), q = i % (D / 4);
      const uint32_t off = part_u + uint32_t(a * (D * 4)) + uint32_t((q ^ (a & 7)) << 4);
      float4 sum = ld_cluster_f4(cluster_map(off, 0));
#pragma unroll
      for (int src = 1; src < C::G; ++src) {
        const float4 v = ld_cluster_f4(cluster_map(off, uint32_t(src)));
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
      }
      *reinterpret_cast<float4*>(gH + size_t(a) * D + q * 4) =
          make_float4(sum.x * inv, sum.y * inv, sum.z * inv, sum.w * inv);
    }
  }
  cluster_sync_all();  // no CTA leaves while another still reads its partial
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
#undef HBAR_BAR
}

}  // namespace pisa
