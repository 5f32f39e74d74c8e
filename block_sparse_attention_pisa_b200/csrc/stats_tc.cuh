// Block statistics on the 5th-generation tensor cores (d = 128): kbar, S0 and either the
// per-block first-order matrix S1 or the head's Hbar.
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
// Persistent CTAs walk work units (one block for S1; 16 consecutive blocks of one head
// for Hbar, whose K^T V products accumulate in one TMEM accumulator). Warp roles:
//   warp 0     TMA producer: K_j and V_j (128-byte swizzled 64-column panels, rows past
//              N zero-filled) into a ring of stages;
//   warp 1     MMA issuer (one thread): K_j^T V_j into one of two TMEM accumulators;
//   warps 8-11 column sums from the stage, one 64-column panel of K or V each: kbar_j
//              (mean of the real rows) and S0_j, to global memory and to shared memory
//              for the epilogue;
//   warps 4-7  epilogue, one TMEM lane (= key dimension a) per thread: S1 mode
//              subtracts kbar_j[a] S0_j[c], rounds to bf16 into a swizzled staging tile
//              and writes it with TMA stores; Hbar mode subtracts sum_j kbar_j[a] S0_j[c]
//              over the unit and adds 1/nB of the result into Hbar with vector atomics.
// Every wait is bounded (about a second); on timeout the CTA raises the device error
// word, stops issuing work, drains what it issued and frees TMEM.
#pragma once

#include "tc_ptx.cuh"

namespace pisa {

template <int BLK, int MODE>
struct StatsTcCfg {
  static constexpr int D = 128;
  static constexpr int kThreads = 384;
  static constexpr int UNIT = (MODE == 2) ? 16 : 1;               // blocks per work unit
  static constexpr int STAGE = 2 * BLK * D * 2;                    // K and V tiles
  static constexpr int STG = D * D * 2;                            // bf16 S1 staging tile
  static constexpr int NSTG = (MODE == 2) ? 0 : 2;                 // staging tiles
  static constexpr int STATS = 2 * D * 4;                          // kbar + S0 of one block
  static constexpr int NSTATS = (MODE == 2) ? 2 * UNIT : 2;        // stats slots
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

// MODE: kStatsS1 (1) per-block S1, kStatsHbar (2) the head's Hbar. d = 128 only.
template <int BLK, int MODE>
__global__ void __launch_bounds__(384, 1)
stats_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmS1, int N, int nB, int units_per_head, int total_units,
                float* __restrict__ kbar, float* __restrict__ S0, float* __restrict__ Hbar) {
  using C = StatsTcCfg<BLK, MODE>;
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
  const int nunits = total_units > int(blockIdx.x) ? (total_units - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  const int nblocks = nunits * C::UNIT;  // CTA-local block sequence t = unit * UNIT + i

  // block t of this CTA: head and block index (units of a head: UNIT consecutive blocks)
  auto block_of = [&](int t, int* bh, int* j) {
    const int u = int(blockIdx.x) + (t / C::UNIT) * int(gridDim.x);
    *bh = u / units_per_head;
    *j = (u % units_per_head) * C::UNIT + t % C::UNIT;
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
      bool ok = true;
      int t = 0;
      for (int u = 0; u < nunits && ok; ++u) {
        const int ab = u & 1;  // accumulator of this unit
        ok = wait_poll(SBAR(C::B_AEMPTY + ab), ((u >> 1) & 1) ^ 1, abort_flag);
        for (int i = 0; i < C::UNIT && ok; ++i, ++t) {
          const int s = t % C::NS;
          if (!(ok = wait_poll(SBAR(C::B_FULL + s), (t / C::NS) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t kb = base_u + C::OFF_RING + s * C::STAGE;
          const uint32_t vb = kb + BLK * D * 2;
#pragma unroll
          for (int kk = 0; kk < BLK / 16; ++kk)
            umma_ss(tmem + ab * D, sdesc_sw128(kb + kk * 2048, BLK * 128, 1024),
                    sdesc_sw128(vb + kk * 2048, BLK * 128, 1024), idS, (i | kk) ? 1u : 0u);
          umma_commit(SBAR(C::B_EMPTY + s));
        }
        if (ok) umma_commit(SBAR(C::B_AFULL + ab));
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
    int t = 0;
    for (int u = 0; u < nunits; ++u) {
      const int ab = u & 1;
      for (int i = 0; i < C::UNIT; ++i, ++t) {
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
#pragma unroll 4
        for (int r = r0; r < BLK; r += 4) {  // zero-filled rows past N add nothing
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
        const int q16 = panel * 8 + qc;  // 16-byte chunk of the row (8 columns)
        // the stats slot: S1 mode double-buffers per block; Hbar mode keeps the unit's blocks
        const int slot = MODE == 2 ? ab * C::UNIT + i : (t & 1);
        if (MODE != 2 && i == 0 && t >= 2) {
          // slot t & 1 was read by the epilogue of block t - 2
          if (!__all_sync(0xffffffffu, wait_bounded(SBAR(C::B_AEMPTY + (t & 1)), ((t >> 1) & 1) ^ 1, abort_flag))) break;
        }
        if (MODE == 2 && i == 0 && u >= 2) {
          if (!__all_sync(0xffffffffu, wait_bounded(SBAR(C::B_AEMPTY + ab), ((u >> 1) & 1) ^ 1, abort_flag))) break;
        }
        if (lane < 8) {
          // blocks past nB (the zero-filled tail of a head's last Hbar unit) write nothing
          float* dst_s = stats + slot * 2 * D + (isV ? D : 0) + q16 * 8;
          const float f = isV ? 1.f : (n > 0 ? 1.f / float(n) : 0.f);
          float4 v0 = make_float4(acc[0] * f, acc[1] * f, acc[2] * f, acc[3] * f);
          float4 v1 = make_float4(acc[4] * f, acc[5] * f, acc[6] * f, acc[7] * f);
          reinterpret_cast<float4*>(dst_s)[0] = v0;
          reinterpret_cast<float4*>(dst_s)[1] = v1;
          if (j < nB) {
            float* dst_g = (isV ? S0 : kbar) + (size_t(bh) * nB + j) * D + q16 * 8;
            reinterpret_cast<float4*>(dst_g)[0] = v0;
            reinterpret_cast<float4*>(dst_g)[1] = v1;
          }
        }
        const int fb = MODE == 2 ? ab : (t & 1);
        if (MODE != 2 || i == C::UNIT - 1) warp_arrive(SBAR(C::B_SFULL + fb));  // one per warp
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (warps 4-7; 2-3 idle)
    const int et = threadIdx.x - 128;  // = TMEM lane = key dimension a
    const int quarter = warp & 3;
    const uint32_t lrow = uint32_t(quarter * 32) << 16;
    const int a = et;
    bool ok = true;
    // S1 mode: the four warps meet at two named barriers per unit; a warp whose wait ran
    // out keeps meeting them (skipping the work), so that no warp is left waiting
    for (int u = 0; u < nunits && (ok || MODE != 2); ++u) {
      const int ab = u & 1;
      if (ok)
        ok = __all_sync(0xffffffffu, wait_bounded(SBAR(C::B_AFULL + ab), (u >> 1) & 1, abort_flag)) &&
             __all_sync(0xffffffffu, wait_bounded(SBAR(C::B_SFULL + ab), (u >> 1) & 1, abort_flag));
      if (MODE == 2 && !ok) break;
      tc_fence_after();
      int bh, j;
      block_of(u * C::UNIT, &bh, &j);
      if (MODE != 2) {
        const float* st = stats + (u & 1) * 2 * D;
        const float ka = st[a];
        const uint32_t stg = base_u + C::OFF_STG + (u & 1) * C::STG;
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
      } else {
        // Hbar: (sum over the unit of K^T V) - sum_j kbar_j[a] S0_j[c], scaled by 1/nB
        const int nj = min(C::UNIT, nB - j);
        const float* st = stats + ab * C::UNIT * 2 * D;
        const float inv = 1.f / float(nB);
        float* gH = Hbar + (size_t(bh) * D + a) * D;
#pragma unroll 1
        for (int ch = 0; ch < D / 16; ++ch) {
          uint32_t r[16];
          tmem_ld16(tmem + lrow + ab * D + ch * 16, r);
          tmem_wait_ld(r);
          float v[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(r[e]);
          for (int i = 0; i < nj; ++i) {
            const float ka = st[i * 2 * D + a];
            const float* s0 = st + i * 2 * D + D + ch * 16;
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] -= ka * s0[e];
          }
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            atomicAdd(reinterpret_cast<float4*>(gH + ch * 16 + e),
                      make_float4(v[e] * inv, v[e + 1] * inv, v[e + 2] * inv, v[e + 3] * inv));
        }
        tc_fence_before();
        warp_arrive(SBAR(C::B_AEMPTY + ab));
      }
    }
    if (MODE != 2 && et == 0) bulk_wait_all();  // the last stores have landed
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
#undef SBAR
}

}  // namespace pisa
