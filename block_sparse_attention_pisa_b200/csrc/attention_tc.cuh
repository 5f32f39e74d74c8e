// Fused PISA attention on the 5th-generation tensor cores (tcgen05 / TMEM / TMA).
//
// PISA explainer ("PISA: Piecewise Sparse Attention Is Wiser for Efficient
// Diffusion Transformers"), technical summary section 2: "Core algorithm"
// (o_t = N_t / D_t; exact term over the critical blocks S_i; zeroth-order term
// alpha_{t,j} S0_j with alpha = exp(x.kbar_j); a first-order term in the
// numerator) and "Hardware implementation" (a fused FlashAttention-style
// online softmax with an exact stage over the selected blocks and an
// approximate stage over the pooled block statistics). The first-order term is
// the per-block Taylor term alpha_{t,j} S1_j^T x_t with S1_j = sum (k - kbar_j) v^T.
// Two further treatments of the non-critical blocks share the kernel: the hybrid
// order of the same section (zeroth order per block plus one global correction
// (x_t Hbar) sum_{j in U} alpha_{t,j}, Hbar the mean first-order matrix of the
// head), and keep-or-drop (non-critical blocks contribute nothing; the
// block-sparse baseline the explainer contrasts PISA with, section 1).
//
// One CTA computes a tile of 128 query rows of one head (two query blocks at
// b = 64, one at b = 128). Warp roles:
//   warp 0      TMA producer: K_j and V_j of the exact blocks (in one stage when they
//               fit), then S1_j of the approximated blocks, through a ring of
//               shared-memory stages;
//   warp 1      MMA issuer (one thread): every tcgen05.mma of the tile;
//   warps 2-3   build the block lists, then convert fp32 kbar / S0 chunks of 32
//               blocks into bf16 swizzled shared-memory operands (at orders 0 and 2,
//               where the approximate stage is short per chunk, warps 8-9 convert every
//               other chunk as well, into a four-stage conversion ring);
//   warps 4-11  two threads per query row (= TMEM lane): warps w and w + 4 share a
//               lane quarter. Exact stage at b = 64: two independent groups, warps 4-7
//               taking the even exact blocks and warps 8-11 the odd ones, each thread
//               all of its row's scores of its block, with its own accumulator O_g,
//               running maximum and denominator; one group's exponentials overlap the
//               other's hand-offs, and the two accumulators are merged once at the end.
//               Exact stage at b = 128: each thread takes half of the row's score
//               columns and half of O's columns, and a pair agrees on its running
//               maximum through shared memory at one named barrier per block. The
//               approximate stage runs on warps 4-7 alone with full-width operands
//               (its hand-offs are short; fewer warps to wait for pays more there);
//               at orders 0 and 2 the MMA thread issues each chunk's pooled scores
//               before it waits for the previous chunk's alpha.
// Tensor memory (512 columns): O accumulator (D), the tile's queries Q (D/2; the A
// operand of Q K^T and Q Kbar^T), then, in the exact stage, the second group's
// accumulator O_1 (D, b = 64 only) and a ring of exact score buffers S (P overwrites
// its own S), or, in the approximate stage, two pooled-score buffers Sbar (the bf16
// alpha operand overwrites its own Sbar) and four A_j = (alpha_j * scale) (.) q
// operand slots used in pairs.
//
// Exact stage, per block j in the union of the tile's selections:
//   S = Q K_j^T (TS-MMA), P = exp(x.k - m) (zero for rows whose query block
//   did not select j and for keys past N), O += P V_j (TS-MMA, V MN-major).
//   Each half of a row packs P for its own keys into the first half of its own
//   score columns, so the two halves never touch each other's columns.
// Approximate stage, per chunk of 32 key blocks that some row approximates:
//   Sbar = Q Kbar_c^T, alpha = exp(x.kbar - m) (zero for blocks a row's own
//   query block selected), O += alpha S0_c (zeroth order), and, two blocks per
//   hand-off, O += A_j S1_j (TS-MMA, S1 MN-major): the first-order term as one
//   long-K GEMM.
// Hybrid order: the approximate stage runs at order 0 while each row also sums its
//   alpha weights (s_t); the row threads that sit out the approximate stage write
//   Hbar as a bf16 operand into the (then idle) first ring stage, the others write
//   A_H = bf16(s_t x_t) at the end, and one M128 x D x D MMA adds A_H Hbar to O.
// Keep-or-drop: no approximate stage at all.
// Denominator: sum of P plus sum n_j alpha_j, kept in fp32 registers. One running
// row maximum covers both stages; the accumulator is rescaled only when the
// maximum grows by more than 2^8 (exact by construction, rare).
//
// Synchronisation: the MMA thread polls its barriers with the non-suspending
// mbarrier probe and waits as rarely as it can, because every wait it makes costs
// tensor-pipe time: per exact block once for K_j and V_j (one barrier) and once
// for P; per pair of approximated blocks once (the row threads signal a pair only
// after writing both A operands and seeing both S1 tiles land). The exact scores
// run NSB - 1 blocks ahead of the softmax with two groups (two at d = 128, b = 64),
// NSB - 2 otherwise. Hand-off
// barriers count one arrival per warp. Every wait is bounded by clock64; on timeout
// a CTA raises the device error word, drains its copies and MMAs, frees TMEM and
// exits. The two warps of a row pair leave together: their named barriers AND-reduce
// the status.
#pragma once

#include "tc_ptx.cuh"

namespace pisa {

struct TcParams {
  const bf16* Q;
  const float* kbar;
  const float* S0;
  const int32_t* idx;
  const float* hbar;  // hybrid order: fp32 [B*H][D][D]
  bf16* O;
  int N;
  int nB;
  int topk;
  int order;
  float scale;
};

template <int D, int BLK>
struct TcCfg {
  static constexpr int kThreads = 384;
  static constexpr int NS = (D == 128) ? 5 : 10;            // TMA stages
  static constexpr int STAGE = (D == 128) ? 32768 : 16384;  // bytes per stage
  static constexpr int NTF = NS;                            // landed-copy barriers (one per load unit)
  // K_j and V_j of an exact block share one stage when both fit (b = 64 at d = 128 and
  // d = 64): twice the blocks in flight for the same shared memory
  static constexpr bool KV_PACKED = 2 * BLK * D * 2 <= STAGE;
  static constexpr int TPB = KV_PACKED ? 1 : 2;             // ring stages per exact block
  // exact block e's V tile is ring-stage use TPB e + TPB - 1; that stage's release (an MMA
  // commit after the block's P V) is also the signal that P V(e) is done
  __host__ __device__ static constexpr int v_stage(int e) { return (TPB * e + TPB - 1) % NS; }
  __host__ __device__ static constexpr uint32_t v_parity(int e) { return uint32_t((TPB * e + TPB - 1) / NS) & 1u; }
  static constexpr int CHUNK = 32;                          // key blocks per approximate chunk
  static constexpr int CV_HALF = CHUNK * D * 2;             // bf16 kbar (or S0) chunk
  static constexpr int CV_STAGE = 2 * CV_HALF;
  // conversion stages: two of their own; at orders 0 and 2 two more in ring stage 1,
  // which no copy uses once the exact stage is done
  static constexpr int NCV_MAX = 4;
  static_assert(2 * CV_STAGE <= STAGE && NS >= 2, "two conversion stages in ring stage 1");
  __host__ __device__ static constexpr int cv_off(int s) {
    return s < 2 ? OFF_CV + s * CV_STAGE : OFF_RING + STAGE + (s - 2) * CV_STAGE;
  }
  static constexpr int GROUP = 2;                           // approximated blocks per hand-off
  static constexpr int NA = 2 * GROUP;                      // A operand slots (two groups)
  // exact score buffers. At d = 128 as many as the columns after Q hold (the approximate
  // stage's operand slots reuse the same columns later): five at b = 64 measured 1-2%
  // faster than four. At d = 64 a deeper ring measured slower (b = 128: 3.20 vs 3.14 ms).
  // At b = 64 the exact stage runs as two independent groups of row warps (warps 4-7 take
  // the even exact blocks, warps 8-11 the odd ones), each with its own accumulator O_g,
  // running maximum and denominator; the two are merged before the approximate stage.
  static constexpr bool GROUPS = (BLK == 64);
  static constexpr int O1_COL = D + D / 2;              // second exact accumulator (GROUPS)
  static constexpr int SX_COL = GROUPS ? O1_COL + D : D + D / 2;  // exact score buffers
  static constexpr int NSB = GROUPS ? (512 - SX_COL) / BLK : ((D == 128) ? (512 - (D + D / 2)) / BLK : 2);
  // the scores run kLook blocks ahead of the row threads' softmax (two groups: one block
  // further, since the two groups' blocks alternate)
  static constexpr int kLook = GROUPS ? NSB - 1 : (NSB >= 3 ? NSB - 2 : 1);
  static constexpr int MAXB = 2048;
  static constexpr int MAXC = MAXB / CHUNK;
  // tensor-memory columns
  static constexpr int O_COL = 0;
  static constexpr int Q_COL = D;
  static constexpr int R_COL = D + D / 2;
  static constexpr int A_COL0 = R_COL + 2 * CHUNK;
  static constexpr int A_COLS = D / 2;
  static constexpr int TMEM_COLS = 512;
  static_assert(SX_COL + NSB * BLK <= TMEM_COLS, "exact score buffers exceed TMEM");
  static_assert(!GROUPS || NSB >= 3, "two groups need three score buffers");
  static_assert(A_COL0 + NA * A_COLS <= TMEM_COLS, "operand ring exceeds TMEM");
  static_assert(STAGE >= BLK * D * 2 && STAGE >= D * D * 2, "stage too small");
  // barriers
  static constexpr int B_SE = 0;                  // [NS]  stage consumed (MMA commit)
  static constexpr int B_TF = B_SE + NS;          // [NTF] copies of a load unit landed
  static constexpr int B_Q = B_TF + NTF;          //       queries in TMEM (8 row warps)
  static constexpr int B_SF = B_Q + 1;            // [NSB] S ready (commit)
  static constexpr int B_PF = B_SF + NSB;         // [NSB] P written (8 row warps)
  static constexpr int B_CVF = B_PF + NSB;        // [4]   kbar / S0 chunk converted (2 warps)
  static constexpr int B_CVE = B_CVF + NCV_MAX;   // [4]   chunk operands consumed (commit)
  static constexpr int B_SBF = B_CVE + NCV_MAX;   // [2]   Sbar ready (commit)
  static constexpr int B_A0F = B_SBF + 2;         // [2]   alpha operand written (8 warps)
  static constexpr int B_SBE = B_A0F + 2;         // [2]   alpha MMA done (commit)
  static constexpr int B_GA = B_SBE + 2;          // [2]   a pair of A_j written (8 warps)
  static constexpr int B_OSYNC = B_GA + 2;        //       end of the exact stage / of a chunk (commit)
  static constexpr int B_ODONE = B_OSYNC + 1;     //       all MMAs done (commit)
  static constexpr int B_XD = B_ODONE + 1;        //       exact stage done, ring idle (commit; orders 0, 2)
  static constexpr int B_HF = B_XD + 1;           //       Hbar operand converted (4 warps; hybrid)
  static constexpr int B_AH = B_HF + 1;           //       A_H = s x written (4 warps; hybrid)
  static constexpr int B_MG = B_AH + 1;           //       group accumulators merged (8 row warps; GROUPS)
  static constexpr int NBARS = B_MG + 1;
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_CV = OFF_RING + NS * STAGE;
  static constexpr int OFF_EXACT = OFF_CV + 2 * CV_STAGE;   // int16[MAXB]
  static constexpr int OFF_APPROX = OFF_EXACT + 2 * MAXB;   // int16[MAXB]
  static constexpr int OFF_ACTIVE = OFF_APPROX + 2 * MAXB;  // int16[MAXC]
  static constexpr int OFF_CHUNK = OFF_ACTIVE + 2 * MAXC;   // int32[MAXC + 1]
  static constexpr int OFF_MASK = OFF_CHUNK + 4 * (MAXC + 4);
  static constexpr int OFF_XCH = OFF_MASK + 2 * (MAXB / 32) * 4;  // float [2 parity][2 half][128] row maxima
  static constexpr int OFF_XS = OFF_XCH + 2 * 2 * 128 * 4;          // float [2 half][128] alpha sums
  static constexpr int OFF_XL = OFF_XS + 2 * 128 * 4;               // float [2 half][128] denominators
  static constexpr int A0_LD = CHUNK / 2 + 1;                      // padded: conflict-free row access
  static constexpr int OFF_A0 = OFF_XL + 2 * 128 * 4;               // uint32 [128 rows][A0_LD] packed alpha
  static constexpr int OFF_BAR = OFF_A0 + 128 * A0_LD * 4;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM = OFF_MISC + 64 + 1024;  // + alignment slack
  static_assert(OFF_BAR % 8 == 0, "barrier alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

namespace tc {

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// two non-negative finite floats -> packed bf16x2, rounded to nearest (ties up),
// with integer ops instead of the conversion unit (which the exponentials share)
__device__ __forceinline__ uint32_t pack_bf16x2_int(float lo, float hi) {
  return __byte_perm(__float_as_uint(lo) + 0x8000u, __float_as_uint(hi) + 0x8000u, 0x7632);
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
  __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 z = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&z);
}

// named barrier of the two warps of one TMEM lane quarter (64 threads); returns the
// AND of `ok` over them, so that both warps of a pair take the same exits
__device__ __forceinline__ bool pair_sync_and(int id, bool ok) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 64, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(ok ? 1u : 0u), "r"(id)
      : "memory");
  return out != 0;
}

// scale COLS fp32 TMEM columns of one row by f (warp-collective)
template <int COLS>
__device__ __forceinline__ void rescale_row(uint32_t taddr, float f) {
#pragma unroll
  for (int ch = 0; ch < COLS / 16; ++ch) {
    uint32_t o[16];
    tmem_ld16(taddr + ch * 16, o);
    tmem_wait_ld(o);
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
    tmem_st16(taddr + ch * 16, o);
  }
  tmem_wait_st();
}

// One approximate chunk's kbar and S0 (fp32 [rows][D], `rows` real blocks, the rest
// zero) -> bf16 UMMA operands at dk (kbar) and dk + CHUNK*D*2 (S0): [CHUNK blocks][D]
// row-major, 128-byte rows per 64-column panel, 16-byte chunks swizzled by (row % 8).
// The K-major (kbar) and MN-major (S0) operand layouts coincide for this storage.
// Thread ct of NT takes 16-byte output chunks ct, ct + NT, ...; the loads of a batch are
// all issued before the first conversion (one L2 round trip per batch).
template <int D, int CHUNK, int NT, int BATCH>
__device__ __forceinline__ void convert_chunk(uint8_t* dk, const float* gk, const float* gs, int rows, int ct) {
  constexpr int ITEMS = CHUNK * (D / 8) / NT;
  static_assert(ITEMS * NT == CHUNK * (D / 8) && ITEMS % BATCH == 0, "converter items");
  uint8_t* ds = dk + CHUNK * D * 2;
#pragma unroll 1
  for (int b0 = 0; b0 < ITEMS; b0 += BATCH) {
    float4 kf[BATCH][2], sf[BATCH][2];
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      const int q = ct + (b0 + i) * NT;
      const int r = q / (D / 8), c16 = q % (D / 8);
      if (r < rows) {
        kf[i][0] = __ldg(reinterpret_cast<const float4*>(gk + r * D + c16 * 8));
        kf[i][1] = __ldg(reinterpret_cast<const float4*>(gk + r * D + c16 * 8 + 4));
        sf[i][0] = __ldg(reinterpret_cast<const float4*>(gs + r * D + c16 * 8));
        sf[i][1] = __ldg(reinterpret_cast<const float4*>(gs + r * D + c16 * 8 + 4));
      } else {
        kf[i][0] = kf[i][1] = sf[i][0] = sf[i][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      const int q = ct + (b0 + i) * NT;
      const int r = q / (D / 8), c16 = q % (D / 8);
      const uint4 kv = make_uint4(pack_bf16x2(kf[i][0].x, kf[i][0].y), pack_bf16x2(kf[i][0].z, kf[i][0].w),
                                  pack_bf16x2(kf[i][1].x, kf[i][1].y), pack_bf16x2(kf[i][1].z, kf[i][1].w));
      const uint4 sv = make_uint4(pack_bf16x2(sf[i][0].x, sf[i][0].y), pack_bf16x2(sf[i][0].z, sf[i][0].w),
                                  pack_bf16x2(sf[i][1].x, sf[i][1].y), pack_bf16x2(sf[i][1].z, sf[i][1].w));
      const int off = (c16 >> 3) * (CHUNK * 128) + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
      *reinterpret_cast<uint4*>(dk + off) = kv;
      *reinterpret_cast<uint4*>(ds + off) = sv;
    }
  }
}

}  // namespace tc

template <int D, int BLK>
__global__ void __launch_bounds__(384, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmS1, const TcParams p) {
  using C = TcCfg<D, BLK>;
  using namespace tc;
  extern __shared__ __align__(16) uint8_t tc_smem_raw[];
  const uint32_t raw_u = smem_u32(tc_smem_raw);
  const uint32_t base_u = (raw_u + 1023u) & ~1023u;  // 128-byte swizzled tiles need 1024-byte alignment
  uint8_t* base = tc_smem_raw + (base_u - raw_u);
  int16_t* exact_list = reinterpret_cast<int16_t*>(base + C::OFF_EXACT);
  int16_t* approx_list = reinterpret_cast<int16_t*>(base + C::OFF_APPROX);
  int16_t* active = reinterpret_cast<int16_t*>(base + C::OFF_ACTIVE);
  int* chunk_off = reinterpret_cast<int*>(base + C::OFF_CHUNK);
  uint32_t* mask = reinterpret_cast<uint32_t*>(base + C::OFF_MASK);  // [2][MAXB/32]
  int* misc = reinterpret_cast<int*>(base + C::OFF_MISC);  // tmem, abort, n_exact, n_approx, n_active
  volatile int* abort_flag = misc + 1;
  const uint32_t bar0 = base_u + C::OFF_BAR;
#define BAR(i) (bar0 + 8u * uint32_t(i))

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int bh = blockIdx.y;
  const int N = p.N, nB = p.nB;
  const int nW = (nB + 31) >> 5;  // mask words; one chunk per word (CHUNK == 32)
  constexpr bool kTwo = (BLK == 64);
  const int i0 = kTwo ? 2 * tile : tile;
  static_assert(C::CHUNK == 32, "chunk == mask word");

  // ------------------------------------------------------------- prologue
  constexpr uint32_t kRowWarps = 8;  // hand-off barriers count one arrival per row warp
  constexpr uint32_t kApproxWarps = 4;  // the approximate stage runs on one half of the row threads
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) mbar_init(BAR(C::B_SE + s), 1);
    for (int s = 0; s < C::NTF; ++s) mbar_init(BAR(C::B_TF + s), 1);
    for (int s = 0; s < C::NSB; ++s) {
      mbar_init(BAR(C::B_SF + s), 1);
      mbar_init(BAR(C::B_PF + s), C::GROUPS ? kRowWarps / 2 : kRowWarps);  // a group, or both halves
    }
    for (int s = 0; s < C::NCV_MAX; ++s) {
      mbar_init(BAR(C::B_CVF + s), 2);
      mbar_init(BAR(C::B_CVE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(C::B_SBF + s), 1);
      mbar_init(BAR(C::B_A0F + s), kApproxWarps);
      mbar_init(BAR(C::B_SBE + s), 1);
      mbar_init(BAR(C::B_GA + s), kApproxWarps);
    }
    mbar_init(BAR(C::B_Q), kRowWarps);
    mbar_init(BAR(C::B_OSYNC), 1);
    mbar_init(BAR(C::B_ODONE), 1);
    mbar_init(BAR(C::B_XD), 1);
    mbar_init(BAR(C::B_HF), 4);
    mbar_init(BAR(C::B_AH), kApproxWarps);
    mbar_init(BAR(C::B_MG), kRowWarps);
    misc[1] = 0;
    mbar_init_fence();
  }
  if (warp == 2) {
    tmem_alloc(base_u + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 3) {
    // critical-block bitmasks of the tile's query block(s)
    for (int w = lane; w < 2 * (C::MAXB / 32); w += 32) mask[w] = 0u;
    __syncwarp();
    for (int q = 0; q < (kTwo ? 2 : 1); ++q) {
      const int i = i0 + q;
      if (i >= nB) continue;
      const int32_t* row = p.idx + (size_t(bh) * nB + i) * p.topk;
      for (int e = lane; e < p.topk; e += 32) {
        const int j = row[e];
        if (j >= 0 && j < nB) atomicOr(&mask[q * (C::MAXB / 32) + (j >> 5)], 1u << (j & 31));
        else flag_error(kErrBadIndex);
      }
    }
    __syncwarp();
    if (kTwo && i0 + 1 >= nB)  // no second query block: its (padding) rows follow the first
      for (int w = lane; w < nW; w += 32) mask[C::MAXB / 32 + w] = mask[w];
    __syncwarp();
    const uint32_t* m0 = mask;
    const uint32_t* m1 = kTwo ? mask + C::MAXB / 32 : mask;
    // exact list = union of the selections; approximate list = blocks that some row
    // does not take exactly; active chunks = chunks holding approximate blocks;
    // chunk_off[c] = first approximate entry of chunk c. All ascending.
    const unsigned lt = (1u << lane) - 1u;
    int ne = 0, na = 0, nac = 0;
    for (int wb = 0; wb < nW; wb += 32) {
      const int w = wb + lane;
      uint32_t u = 0, a = 0;
      if (w < nW) {
        const uint32_t valid = (w == nW - 1 && (nB & 31)) ? ((1u << (nB & 31)) - 1u) : 0xffffffffu;
        u = (m0[w] | m1[w]) & valid;
        a = ~(m0[w] & m1[w]) & valid;
      }
      const int pu = __popc(u), pa = __popc(a);
      int xu = pu, xa = pa;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int tu = __shfl_up_sync(0xffffffffu, xu, off);
        const int ta = __shfl_up_sync(0xffffffffu, xa, off);
        if (lane >= off) {
          xu += tu;
          xa += ta;
        }
      }
      int eu = ne + xu - pu, ea = na + xa - pa;
      if (w < nW) chunk_off[w] = ea;
      const unsigned act = __ballot_sync(0xffffffffu, a != 0u);
      if (a != 0u) active[nac + __popc(act & lt)] = int16_t(w);
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        exact_list[eu++] = int16_t(w * 32 + bit);
      }
      while (a) {
        const int bit = __ffs(a) - 1;
        a &= a - 1;
        approx_list[ea++] = int16_t(w * 32 + bit);
      }
      ne += __shfl_sync(0xffffffffu, xu, 31);
      na += __shfl_sync(0xffffffffu, xa, 31);
      nac += __popc(act);
    }
    if (lane == 0) {
      chunk_off[nW] = na;
      misc[2] = ne;
      misc[3] = na;
      misc[4] = p.order < 0 ? 0 : nac;  // keep-or-drop: no approximate stage
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = uint32_t(misc[0]);
  const int n_exact = misc[2];
  const int n_active = misc[4];
  const bool hybrid = p.order == 2 && n_active > 0;
  // orders 0 and 2: four conversion stages (two in the idle ring), and each chunk's pooled
  // scores are issued before the previous chunk's alpha is awaited
  const bool deep = (p.order == 0 || p.order == 2) && n_active > 0;
  const int ncv = deep ? C::NCV_MAX : 2;

  if (warp == 0) {
    // ----------------------------------------------------------- TMA producer
    // Lanes 0 and 1 issue the copies together: lane 0 the K panels (or the first panel of
    // each S1 tile), lane 1 the V panels (the second S1 panel). A single issuing thread
    // delivers about 35-40 B/clk into an SM; two reach about 60.
    if (lane < 2) {
      int t = 0, u = 0;  // tiles issued, load units issued
      bool ok = true;
      for (int e = 0; e < n_exact && ok; ++e, ++u) {
        const int j = exact_list[e];
        for (int q = 0; q < C::TPB && ok; ++q)
          ok = wait_bounded(BAR(C::B_SE + (t + q) % C::NS), (((t + q) / C::NS) & 1) ^ 1, abort_flag);
        ok = __all_sync(0x3u, ok);
        if (!ok) break;
        const uint32_t tf = BAR(C::B_TF + u % C::NTF);
        if (lane == 0) mbar_arrive_expect_tx(tf, 2 * BLK * D * 2);
        __syncwarp(0x3u);
        const int kv = lane;
        const uint32_t dst = base_u + C::OFF_RING + ((t + (C::KV_PACKED ? 0 : kv)) % C::NS) * C::STAGE +
                             (C::KV_PACKED ? kv * BLK * D * 2 : 0);
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_3d(dst + pn * BLK * 128, kv ? &tmV : &tmK, tf, pn * 64, j * BLK, bh);
        t += C::TPB;
      }
      if (p.order == 1) {
        for (int ac = 0; ac < n_active && ok; ++ac) {
          const int c = active[ac];
          const int a_end = chunk_off[c + 1];
          for (int a = chunk_off[c]; a < a_end && ok; a += C::GROUP, ++u) {
            const int n = min(C::GROUP, a_end - a);
            for (int q = 0; q < n && ok; ++q)
              ok = wait_bounded(BAR(C::B_SE + (t + q) % C::NS), (((t + q) / C::NS) & 1) ^ 1, abort_flag);
            if (!__all_sync(0x3u, ok)) { ok = false; break; }
            const uint32_t tf = BAR(C::B_TF + u % C::NTF);
            if (lane == 0) mbar_arrive_expect_tx(tf, n * D * D * 2);
            __syncwarp(0x3u);
            for (int q = 0; q < n; ++q, ++t) {
              const uint32_t dst = base_u + C::OFF_RING + (t % C::NS) * C::STAGE;
              const int j = approx_list[a + q];
              for (int pn = lane; pn < D / 64; pn += 2)
                tma_load_3d(dst + pn * D * 128, &tmS1, tf, pn * 64, 0, bh * nB + j);
            }
          }
        }
      }
      // no copy may still be in flight when the CTA exits (each load unit's barrier
      // completes from the copies of both lanes alone)
      if (lane == 0)
        for (int v = u > C::NTF ? u - C::NTF : 0; v < u; ++v) wait_drain(BAR(C::B_TF + v % C::NTF), (v / C::NTF) & 1);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, BLK, false);        // S = Q K^T
      constexpr uint32_t idSB = idesc_bf16(128, C::CHUNK, false);  // Sbar = Q Kbar^T
      constexpr uint32_t idO = idesc_bf16(128, D, true);           // O += {P V, alpha S0, A S1}
      uint32_t o_acc = 0;
      // GROUPS: bit g set once group g's accumulator holds a product (a bit mask, not an
      // array: a runtime index would put the array in local memory)
      uint32_t g_acc = 0u;
      bool ok = wait_poll(BAR(C::B_Q), 0, abort_flag);
      tc_fence_after();
      // P V(e) done: the release of block e's V ring stage (committed right after it)
      auto wait_pv = [&](int e) -> bool {
        return wait_poll(BAR(C::B_SE + C::v_stage(e)), C::v_parity(e), abort_flag);
      };
      auto pv = [&](int e) -> bool {
        const int sb = e % C::NSB;
        if (!wait_poll(BAR(C::B_PF + sb), (e / C::NSB) & 1, abort_flag)) return false;
        tc_fence_after();
        const int sv = (C::TPB * e + C::TPB - 1) % C::NS;
        const uint32_t vb = base_u + C::OFF_RING + sv * C::STAGE + (C::KV_PACKED ? BLK * D * 2 : 0);
        if constexpr (C::GROUPS) {
          // P of keys [16k, 16k + 16) at the start of block e's score columns; O of the
          // block's group
          const uint32_t oc = (e & 1) ? C::O1_COL : C::O_COL;
#pragma unroll
          for (int k = 0; k < BLK / 16; ++k)
            umma_ts(tmem + oc, tmem + C::SX_COL + sb * BLK + k * 8, sdesc_sw128(vb + k * 2048, BLK * 128, 1024), idO,
                    (((g_acc >> (e & 1)) & 1u) | uint32_t(k)) ? 1u : 0u);
          g_acc |= 1u << (e & 1);
        } else {
          // P of keys [16k, 16k + 16): half (k / (BLK/32)) of the row packed it at the
          // start of its own score columns
#pragma unroll
          for (int k = 0; k < BLK / 16; ++k)
            umma_ts(tmem + C::O_COL,
                    tmem + C::SX_COL + sb * BLK + (k / (BLK / 32)) * (BLK / 2) + (k % (BLK / 32)) * 8,
                    sdesc_sw128(vb + k * 2048, BLK * 128, 1024), idO, (o_acc | uint32_t(k)) ? 1u : 0u);
        }
        o_acc = 1;
        umma_commit(BAR(C::B_SE + sv));
        return true;
      };
      // S = Q K_j^T for block e (its buffer was last used by block e - NSB)
      // `waits`: K(e) landed and P V(e - NSB) done are awaited here; after the prologue the
      // row group that signals P(e - kLook) has awaited both before its signal
      auto qk = [&](int e, bool waits) -> bool {
        const int sb = e % C::NSB;
        if (waits) {
          if (e >= C::NSB && !wait_pv(e - C::NSB)) return false;
          if (!wait_poll(BAR(C::B_TF + e % C::NTF), (e / C::NTF) & 1, abort_flag)) return false;
        }
        tc_fence_after();
        const int sk = (C::TPB * e) % C::NS;
        const uint32_t kb = base_u + C::OFF_RING + sk * C::STAGE;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          umma_ts(tmem + C::SX_COL + sb * BLK, tmem + C::Q_COL + k * 8,
                  sdesc_sw128(kb + (k >> 2) * (BLK * 128) + (k & 3) * 32, 16, 1024), idS, k ? 1u : 0u);
        if (!C::KV_PACKED) umma_commit(BAR(C::B_SE + sk));  // a packed stage is released after P V
        umma_commit(BAR(C::B_SF + sb));
        return true;
      };
      for (int e = 0; e < C::kLook && e < n_exact && ok; ++e) ok = qk(e, true);
      for (int e = 0; e < n_exact && ok; ++e) {
        ok = pv(e);
        if (ok && e + C::kLook < n_exact) ok = qk(e + C::kLook, false);
      }
      umma_commit(BAR(C::B_OSYNC));  // completion 0: end of the exact stage
      if (deep) umma_commit(BAR(C::B_XD));

      if (ok && n_active > 0) {
        // the pooled-score and operand columns reuse the exact score buffers (and, with two
        // groups, the second accumulator, which the row threads have merged first)
        if constexpr (C::GROUPS)
          ok = wait_poll(BAR(C::B_MG), 0, abort_flag);
        else
          ok = wait_pv(n_exact - 1);
        auto sbar = [&](int ac) -> bool {
          const int b = ac & 1, cs = ac % ncv;
          if (!wait_poll(BAR(C::B_CVF + cs), (ac / ncv) & 1, abort_flag)) return false;
          if (ac >= 2 && !wait_poll(BAR(C::B_SBE + b), ((ac - 2) >> 1) & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t kb = base_u + C::cv_off(cs);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_ts(tmem + C::R_COL + b * C::CHUNK, tmem + C::Q_COL + k * 8,
                    sdesc_sw128(kb + (k >> 2) * (C::CHUNK * 128) + (k & 3) * 32, 16, 1024), idSB, k ? 1u : 0u);
          umma_commit(BAR(C::B_SBF + b));
          return true;
        };
        if (ok) ok = sbar(0);
        int g = 0;               // pair (hand-off) counter
        int t = C::TPB * n_exact;  // stage-use counter
        int u = n_exact;         // load-unit counter
        for (int ac = 0; ac < n_active && ok; ++ac) {
          const int c = active[ac];
          const int b = ac & 1, cs = ac % ncv;
          // deep: the next chunk's pooled scores first, so that they are ready when the
          // row threads finish this chunk's alpha (their TMEM buffer's last alpha MMA, of
          // chunk ac - 1, was issued in the previous iteration, and sbar waits for it)
          if (deep && ac + 1 < n_active && !(ok = sbar(ac + 1))) break;
          if (!(ok = wait_poll(BAR(C::B_A0F + b), (ac >> 1) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t sb = base_u + C::cv_off(cs) + C::CV_HALF;
          // alpha of blocks [16k, 16k + 16): packed by half k of the row at the start of
          // its own pooled-score columns
#pragma unroll
          for (int k = 0; k < C::CHUNK / 16; ++k)
            umma_ts(tmem + C::O_COL, tmem + C::R_COL + b * C::CHUNK + k * 16,
                    sdesc_sw128(sb + k * 2048, C::CHUNK * 128, 1024), idO, (o_acc | uint32_t(k)) ? 1u : 0u);
          o_acc = 1;
          umma_commit(BAR(C::B_SBE + b));
          umma_commit(BAR(C::B_CVE + cs));
          if (!deep && ac + 1 < n_active && !(ok = sbar(ac + 1))) break;
          if (p.order == 1) {
            const int a_end = chunk_off[c + 1];
            for (int a = chunk_off[c]; a < a_end; a += C::GROUP, ++g, ++u) {
              const int n = min(C::GROUP, a_end - a);
              const int gs = g & 1;
              // the row threads signal a pair only after its S1 copies have landed, so one
              // wait covers both operands
              if (!(ok = wait_poll(BAR(C::B_GA + gs), (g >> 1) & 1, abort_flag))) break;
              tc_fence_after();
              for (int q = 0; q < n; ++q, ++t) {
                const int s = t % C::NS;
                const uint32_t s1 = base_u + C::OFF_RING + s * C::STAGE;
                const uint32_t aa = tmem + C::A_COL0 + (gs * C::GROUP + q) * C::A_COLS;
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                  umma_ts(tmem + C::O_COL, aa + k * 8, sdesc_sw128(s1 + k * 2048, D * 128, 1024), idO, 1u);
                umma_commit(BAR(C::B_SE + s));
              }
            }
          }
          umma_commit(BAR(C::B_OSYNC));  // completion ac + 1: end of active chunk ac
        }
        if (ok && hybrid) {
          // O += A_H Hbar: A_H in the first operand slot, Hbar (MN-major) in ring stage 0
          ok = wait_poll(BAR(C::B_HF), 0, abort_flag) && wait_poll(BAR(C::B_AH), 0, abort_flag);
          if (ok) {
            tc_fence_after();
            const uint32_t hb = base_u + C::OFF_RING;
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
              umma_ts(tmem + C::O_COL, tmem + C::A_COL0 + k * 8, sdesc_sw128(hb + k * 2048, D * 128, 1024), idO,
                      1u);
          }
        }
      }
      umma_commit(BAR(C::B_ODONE));
      wait_drain(BAR(C::B_ODONE), 0);  // nothing of ours may run on after the CTA frees TMEM
    }
  } else if (warp < 4) {
    // ----------------------------------------------------------- kbar / S0 converter
    // Warps 2-3 convert every chunk; in deep mode chunks 0, 1 and the even ones, while
    // warps 8-9 (idle in the approximate stage there) take the odd ones from 3 on.
    const int ct = threadIdx.x - 64;
    bool ring_idle = false;  // deep: the exact stage is done, ring stage 1 holds stages 2, 3
    for (int ac = 0; ac < n_active; ++ac) {
      if (deep && ac >= 3 && (ac & 1)) continue;
      const int c = active[ac];
      const int s = ac % ncv;
      if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_CVE + s), ((ac / ncv) & 1) ^ 1, abort_flag))) break;
      if (s >= 2 && !ring_idle) {
        if (!__all_sync(0xffffffffu, wait_bounded(BAR(C::B_XD), 0, abort_flag))) break;
        ring_idle = true;
      }
      convert_chunk<D, C::CHUNK, 64, 4>(base + C::cv_off(s), p.kbar + (size_t(bh) * nB + size_t(c) * C::CHUNK) * D,
                                        p.S0 + (size_t(bh) * nB + size_t(c) * C::CHUNK) * D,
                                        min(C::CHUNK, nB - c * C::CHUNK), ct);
      fence_proxy_async_smem();
      warp_arrive(BAR(C::B_CVF + s));
    }
  } else {
    // ----------------------------------------------------------- row threads
    // Two threads per query row: half 0 (warps 4-7) and half 1 (warps 8-11) of a lane
    // quarter. Half hf owns score columns [hf * BLK/2, (hf + 1) * BLK/2) of each exact
    // block, blocks [hf * 16, hf * 16 + 16) of each approximate chunk, and O / Q / A
    // columns of dimensions [hf * D/2, (hf + 1) * D/2). Both halves hold the same
    // running maximum m; l and the alpha sum are per-half partial sums.
    const int rt = threadIdx.x - 128;
    const int hf = rt >> 7;                                  // column half
    const int r = rt & 127;                                  // row in tile = TMEM lane
    const int quarter = warp & 3;
    const uint32_t lrow = uint32_t(quarter * 32) << 16;      // this warp's TMEM lane quarter
    const int pair_id = 1 + quarter;                         // named barrier of the pair
    const int grow = tile * 128 + r;
    const bool valid = grow < N;
    const uint32_t* mymask = (kTwo && r >= 64) ? mask + C::MAXB / 32 : mask;
    float* xmax = reinterpret_cast<float*>(base + C::OFF_XCH);
    float* xs = reinterpret_cast<float*>(base + C::OFF_XS);
    float* xl = reinterpret_cast<float*>(base + C::OFF_XL);
    constexpr int HK = BLK / 2;     // exact keys per half
    constexpr int HD = D / 2;       // O / value dimensions per half
    constexpr int HA = D / 4;       // packed bf16 Q / A columns per half
    bool ok = true;

    // queries -> TMEM (the A operand of Q K^T and Q Kbar^T): this half's dimensions
    {
      const uint4* src =
          reinterpret_cast<const uint4*>(p.Q + (size_t(bh) * N + (valid ? grow : 0)) * D + hf * HD);
#pragma unroll
      for (int ch = 0; ch < HA / 16; ++ch) {
        uint32_t t[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = valid ? __ldg(src + ch * 4 + i) : make_uint4(0, 0, 0, 0);
          t[4 * i] = v.x;
          t[4 * i + 1] = v.y;
          t[4 * i + 2] = v.z;
          t[4 * i + 3] = v.w;
        }
        tmem_st16(tmem + lrow + C::Q_COL + hf * HA + ch * 16, t);
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(BAR(C::B_Q));
    }

    const float sl2 = p.scale * 1.4426950408889634f;  // exponents in base 2
    float m = -INFINITY, l = 0.f;
    float s_alpha = 0.f;  // hybrid order: this half's sum of alpha weights (same frame as l)

    // ------------------------------------------------ exact stage
    if constexpr (C::GROUPS) {
      // Group hf takes the exact blocks e = hf, hf + 2, ...: all BLK scores of its row,
      // its own accumulator O_hf, running maximum m and denominator l. No exchange with the
      // other group per block; one merge at the end.
      const uint32_t oc = hf ? C::O1_COL : C::O_COL;
      for (int e = hf; e < n_exact; e += 2) {
        const int j = exact_list[e], sb = e % C::NSB;
        const bool sel = (mymask[j >> 5] >> (j & 31)) & 1u;  // uniform per warp
        const int nreal = min(BLK, N - j * BLK);              // real keys of the block
        ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SF + sb), (e / C::NSB) & 1, abort_flag));
        if (!ok) break;
        const uint32_t sa = tmem + lrow + C::SX_COL + sb * BLK;
        uint32_t pk[BLK / 2];
        float rsp[4] = {0.f, 0.f, 0.f, 0.f};
        if (sel) {
          tc_fence_after();
          uint32_t sc[BLK];
#pragma unroll
          for (int ch = 0; ch < BLK / 16; ++ch)
            tmem_ld16(sa + ch * 16, *reinterpret_cast<uint32_t(*)[16]>(&sc[ch * 16]));
#pragma unroll
          for (int ch = 0; ch < BLK / 16; ++ch) tmem_wait_ld(*reinterpret_cast<uint32_t(*)[16]>(&sc[ch * 16]));
          if (nreal < BLK) {  // ragged last block: keys past N take no weight
#pragma unroll
            for (int k = 0; k < BLK; ++k)
              if (k >= nreal) sc[k] = __float_as_uint(-INFINITY);
          }
          float mxp[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mxp[i] = -INFINITY;
#pragma unroll
          for (int k = 0; k < BLK; ++k) mxp[k & 7] = fmaxf(mxp[k & 7], __uint_as_float(sc[k]));
          const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                                 fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]))) * sl2;
          const bool grow_max = mx > m + 8.f;
          const bool need_o = grow_max && m != -INFINITY;
          if (__any_sync(0xffffffffu, need_o)) {
            // the group's previous product must be in O_hf before it is rescaled
            if (e >= 2)
              ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SE + C::v_stage(e - 2)), C::v_parity(e - 2), abort_flag));
            if (ok) {
              tc_fence_after();
              const float f = need_o ? ex2(m - mx) : 1.f;
              rescale_row<D>(tmem + lrow + oc, f);
              l *= f;
            }
          }
          if (!ok) break;
          if (grow_max) m = mx;
          const float negm = -m;
#pragma unroll
          for (int i = 0; i < BLK / 2; ++i) {
            const float p0 = ex2(fmaf(__uint_as_float(sc[2 * i]), sl2, negm));
            const float p1 = ex2(fmaf(__uint_as_float(sc[2 * i + 1]), sl2, negm));
            rsp[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2_int(p0, p1);
          }
        } else {
          // rows whose query block did not select j take no exact weight
#pragma unroll
          for (int i = 0; i < BLK / 2; ++i) pk[i] = 0u;
        }
#pragma unroll
        for (int ch = 0; ch < BLK / 32; ++ch)
          tmem_st16(sa + ch * 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[ch * 16]));
        l += (rsp[0] + rsp[1]) + (rsp[2] + rsp[3]);
        tmem_wait_st();
        tc_fence_before();
        // what the MMA thread's Q K^T of block e + kLook (issued right after P V(e)) needs:
        // that block's K landed and P V(e + kLook - NSB) done, awaited here so that it
        // issues without a wait (a wait that runs out has raised the abort flag)
        {
          const int en = e + C::kLook;
          if (en < n_exact) {
            bool w = wait_bounded(BAR(C::B_TF + en % C::NTF), (en / C::NTF) & 1, abort_flag);
            if (w && en >= C::NSB)
              w = wait_bounded(BAR(C::B_SE + C::v_stage(en - C::NSB)), C::v_parity(en - C::NSB), abort_flag);
            __syncwarp();
          }
        }
        warp_arrive(BAR(C::B_PF + sb));
      }
      // merge: O_0 <- f_0 O_0 + f_1 O_1 against the common maximum, each group over its own
      // half of the columns, once every product of both groups is in
      xmax[hf * 128 + r] = m;
      xmax[256 + hf * 128 + r] = l;
      ok = pair_sync_and(pair_id, ok);
      const float m_o = xmax[(hf ^ 1) * 128 + r], l_o = xmax[256 + (hf ^ 1) * 128 + r];
      const float mm = fmaxf(m, m_o);
      const float m0 = hf ? m_o : m, m1 = hf ? m : m_o;
      const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - mm);
      const float f1 = m1 == -INFINITY ? 0.f : ex2(m1 - mm);
      if (ok && n_exact >= 2) {  // with a single exact block O_1 holds no product
        ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_OSYNC), 0, abort_flag));
        if (ok) {
          tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < (D / 2) / 16; ++ch) {
            uint32_t a[16], b[16];
            tmem_ld16(tmem + lrow + C::O_COL + hf * (D / 2) + ch * 16, a);
            tmem_ld16(tmem + lrow + C::O1_COL + hf * (D / 2) + ch * 16, b);
            tmem_wait_ld(a);
            tmem_wait_ld(b);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              a[i] = __float_as_uint(fmaf(__uint_as_float(a[i]), f0, __uint_as_float(b[i]) * f1));
            tmem_st16(tmem + lrow + C::O_COL + hf * (D / 2) + ch * 16, a);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      warp_arrive(BAR(C::B_MG));
      // from here on: one accumulator O_0 with maximum mm; the whole denominator with half 0
      l = hf ? 0.f : (hf ? l_o : l) * f0 + (hf ? l : l_o) * f1;
      m = mm;
      ok = pair_sync_and(pair_id, ok);
    } else {
      for (int e = 0; e < n_exact; ++e) {
        const int j = exact_list[e], sb = e % C::NSB;
        const bool sel = (mymask[j >> 5] >> (j & 31)) & 1u;  // uniform per warp
        const int nmine = min(HK, N - j * BLK - hf * HK);     // this half's real keys (may be <= 0)
        if (ok) ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SF + sb), (e / C::NSB) & 1, abort_flag));
        uint32_t s[HK];
        const uint32_t sa = tmem + lrow + C::SX_COL + sb * BLK + hf * HK;
        float pm = -INFINITY;
        if (ok) {
          tc_fence_after();
  #pragma unroll
          for (int ch = 0; ch < HK / 16; ++ch) tmem_ld16(sa + ch * 16, *reinterpret_cast<uint32_t(*)[16]>(&s[ch * 16]));
  #pragma unroll
          for (int ch = 0; ch < HK / 16; ++ch) tmem_wait_ld(*reinterpret_cast<uint32_t(*)[16]>(&s[ch * 16]));
          if (nmine < HK) {  // ragged last block: keys past N take no weight
  #pragma unroll
            for (int k = 0; k < HK; ++k)
              if (k >= nmine) s[k] = __float_as_uint(-INFINITY);
          }
          if (sel) {
            // raw-score maximum (the positive scale commutes with it); independent partial
            // maxima, because one warp per scheduler cannot hide a serial chain
            float mxp[8];
  #pragma unroll
            for (int i = 0; i < 8; ++i) mxp[i] = -INFINITY;
  #pragma unroll
            for (int k = 0; k < HK; ++k) mxp[k & 7] = fmaxf(mxp[k & 7], __uint_as_float(s[k]));
            pm = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                       fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
          }
        }
        xmax[((e & 1) * 2 + hf) * 128 + r] = pm;
        ok = pair_sync_and(pair_id, ok);
        if (!ok) break;
        const float mx = fmaxf(pm, xmax[((e & 1) * 2 + (hf ^ 1)) * 128 + r]) * sl2;
        const bool grow_max = mx > m + 8.f;          // false for rows that did not select j
        const bool need_o = grow_max && m != -INFINITY;
        if (__any_sync(0xffffffffu, need_o)) {
          if (e >= 1)
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SE + C::v_stage(e - 1)), C::v_parity(e - 1), abort_flag));
          if (ok) {
            tc_fence_after();
            const float f = need_o ? ex2(m - mx) : 1.f;
            rescale_row<HD>(tmem + lrow + C::O_COL + hf * HD, f);
            l *= f;
          }
        }
        if (grow_max) m = mx;
        float rsp[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[HK / 2];
        if (sel) {
          const float negm = -m;
  #pragma unroll
          for (int i = 0; i < HK / 2; ++i) {
            const float p0 = ex2(fmaf(__uint_as_float(s[2 * i]), sl2, negm));
            const float p1 = ex2(fmaf(__uint_as_float(s[2 * i + 1]), sl2, negm));
            rsp[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2_int(p0, p1);
          }
        } else {
          // rows whose query block did not select j take no exact weight (m may still be
          // -inf for them, so no exponential is evaluated)
  #pragma unroll
          for (int i = 0; i < HK / 2; ++i) pk[i] = 0u;
        }
  #pragma unroll
        for (int ch = 0; ch < HK / 32; ++ch) tmem_st16(sa + ch * 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[ch * 16]));
        l += (rsp[0] + rsp[1]) + (rsp[2] + rsp[3]);
        tmem_wait_st();
        tc_fence_before();
        // what the MMA thread's Q K^T of block e + kLook (issued right after P V(e)) needs:
        // that block's K landed and P V(e + kLook - NSB) done, awaited here so that it
        // issues without a wait (a wait that runs out has raised the abort flag)
        {
          const int en = e + C::kLook;
          if (en < n_exact) {
            bool w = wait_bounded(BAR(C::B_TF + en % C::NTF), (en / C::NTF) & 1, abort_flag);
            if (w && en >= C::NSB)
              w = wait_bounded(BAR(C::B_SE + C::v_stage(en - C::NSB)), C::v_parity(en - C::NSB), abort_flag);
            __syncwarp();
          }
        }
        warp_arrive(BAR(C::B_PF + sb));
      }
      ok = pair_sync_and(pair_id, ok);
    }

    // ------------------------------------------------ approximate stage
    // Half 0 of each row runs it alone on full-width operands (O, alpha, A_j, A_H): the
    // per-chunk and per-block operand hand-offs then wait on four warps, not eight.
    // Half 1 hands its partial denominator over and goes on to the epilogue.
    if (ok && n_active > 0) {
      xs[hf * 128 + r] = l;
      ok = pair_sync_and(pair_id, ok);
      if (hf == 1) {
        l = 0.f;
        if (ok && hybrid) {
          // Hbar fp32 [D][D] (row a = key dim, column c = value dim) -> bf16 MN-major
          // operand in ring stage 0 (idle once the exact stage is done), laid out as a
          // TMA 128-byte-swizzled load of 64-column panels would place it. Loads are
          // issued in batches of four 16-byte output chunks per thread.
          ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_XD), 0, abort_flag));
          if (ok) {
            const float* gh = p.hbar + size_t(bh) * D * D;
            uint8_t* dh = base + C::OFF_RING;
            constexpr int ITEMS = D * (D / 8) / 128, BATCH = 4;
            static_assert(ITEMS % BATCH == 0, "Hbar conversion batches");
#pragma unroll 1
            for (int b0 = 0; b0 < ITEMS; b0 += BATCH) {
              float4 f[BATCH][2];
#pragma unroll
              for (int i = 0; i < BATCH; ++i) {
                const int q = r + (b0 + i) * 128;
                const int row = q / (D / 8), c16 = q % (D / 8);
                f[i][0] = __ldg(reinterpret_cast<const float4*>(gh + row * D + c16 * 8));
                f[i][1] = __ldg(reinterpret_cast<const float4*>(gh + row * D + c16 * 8 + 4));
              }
#pragma unroll
              for (int i = 0; i < BATCH; ++i) {
                const int q = r + (b0 + i) * 128;
                const int row = q / (D / 8), c16 = q % (D / 8);
                *reinterpret_cast<uint4*>(dh + (c16 >> 3) * (D * 128) + row * 128 + (((c16 & 7) ^ (row & 7)) << 4)) =
                    make_uint4(pack_bf16x2(f[i][0].x, f[i][0].y), pack_bf16x2(f[i][0].z, f[i][0].w),
                               pack_bf16x2(f[i][1].x, f[i][1].y), pack_bf16x2(f[i][1].z, f[i][1].w));
              }
            }
            fence_proxy_async_smem();
            warp_arrive(BAR(C::B_HF));
          }
        }
        if (ok && deep && warp < 10) {
          // the odd chunks from 3 on (ring stage 1 is idle: B_XD)
          ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_XD), 0, abort_flag));
          for (int ac = 3; ac < n_active && ok; ac += 2) {
            const int c = active[ac];
            const int s = ac % ncv;
            if (!(ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_CVE + s), ((ac / ncv) & 1) ^ 1, abort_flag))))
              break;
            convert_chunk<D, C::CHUNK, 64, 4>(base + C::cv_off(s),
                                              p.kbar + (size_t(bh) * nB + size_t(c) * C::CHUNK) * D,
                                              p.S0 + (size_t(bh) * nB + size_t(c) * C::CHUNK) * D,
                                              min(C::CHUNK, nB - c * C::CHUNK), int(threadIdx.x) - 256);
            fence_proxy_async_smem();
            warp_arrive(BAR(C::B_CVF + s));
          }
        }
      } else if (ok) {
        l += xs[128 + r];
        ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_OSYNC), 0, abort_flag));
        uint32_t qf[D / 2];  // all packed query dimensions of the row
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch)
            tmem_ld16(tmem + lrow + C::Q_COL + ch * 16, *reinterpret_cast<uint32_t(*)[16]>(&qf[ch * 16]));
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) tmem_wait_ld(*reinterpret_cast<uint32_t(*)[16]>(&qf[ch * 16]));
        }
        const int nlast = N - (nB - 1) * BLK;
        int g = 0;
        int tl1 = -1, tl2 = -1;  // stage use of the last block of pairs g - 1, g - 2
        for (int ac = 0; ac < n_active && ok; ++ac) {
          const int c = active[ac];
          const int b = ac & 1;
          ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SBF + b), (ac >> 1) & 1, abort_flag));
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = tmem + lrow + C::R_COL + b * C::CHUNK;
          uint32_t sv[C::CHUNK];
          tmem_ld16(sa, *reinterpret_cast<uint32_t(*)[16]>(&sv[0]));
          tmem_ld16(sa + 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[16]));
          tmem_wait_ld(*reinterpret_cast<uint32_t(*)[16]>(&sv[0]));
          tmem_wait_ld(*reinterpret_cast<uint32_t(*)[16]>(&sv[16]));
          const uint32_t myw = mymask[c];
          const int kmax = nB - c * C::CHUNK;
          float mxp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int k = 0; k < C::CHUNK; ++k) {
            const bool mine = k < kmax && !((myw >> k) & 1u);
            const float v = mine ? __uint_as_float(sv[k]) * sl2 : -INFINITY;
            sv[k] = __float_as_uint(v);
            mxp[k & 3] = fmaxf(mxp[k & 3], v);
          }
          const float mx = fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3]));
          const bool need_o = mx > m + 8.f;
          if (__any_sync(0xffffffffu, need_o)) {
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_OSYNC), ac & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const float f = need_o ? ex2(m - mx) : 1.f;
            rescale_row<D>(tmem + lrow + C::O_COL, f);
            l *= f;
            s_alpha *= f;
            if (need_o) m = mx;
          }
          float lsp[4] = {0.f, 0.f, 0.f, 0.f};
          float ssp[2] = {0.f, 0.f};
          uint32_t a0[C::CHUNK / 2];
          // this row's packed alpha of the chunk, also in shared memory for the per-block
          // lookups below (a register array held through the block loop lives in local memory)
          uint32_t* a0s = reinterpret_cast<uint32_t*>(base + C::OFF_A0) + r * C::A0_LD;
#pragma unroll
          for (int k = 0; k < C::CHUNK; k += 2) {
            const float x0 = ex2(__uint_as_float(sv[k]) - m);
            const float x1 = ex2(__uint_as_float(sv[k + 1]) - m);
            const float n0 = (c * C::CHUNK + k == nB - 1) ? float(nlast) : float(BLK);
            const float n1 = (c * C::CHUNK + k + 1 == nB - 1) ? float(nlast) : float(BLK);
            // the denominator (and the hybrid weight sum) take the bf16-rounded alpha that
            // the numerator's MMAs multiply, so both sides weigh each block alike
            const uint32_t w = pack_bf16x2_int(x0, x1);
            const float r0 = bf16_lo(w), r1 = bf16_hi(w);
            lsp[(k >> 1) & 3] = fmaf(n1, r1, fmaf(n0, r0, lsp[(k >> 1) & 3]));
            if (hybrid) ssp[(k >> 1) & 1] += r0 + r1;
            a0[k >> 1] = w;
            a0s[k >> 1] = w;
          }
          l += (lsp[0] + lsp[1]) + (lsp[2] + lsp[3]);
          s_alpha += ssp[0] + ssp[1];
          // alpha of blocks [16k, 16k + 16) at columns [16k, 16k + 8) (the layout the
          // zeroth-order MMA reads)
          {
            uint32_t lo[8], hi[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              lo[i] = a0[i];
              hi[i] = a0[8 + i];
            }
            tmem_st8(sa, lo);
            tmem_st8(sa + 16, hi);
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(BAR(C::B_A0F + b));
          if (p.order != 1) continue;
          // one runtime iteration per pair of approximated blocks (kept rolled: an
          // unrolled copy evicts the MMA warp's instructions)
          const int a_end = chunk_off[c + 1];
#pragma unroll 1
          for (int a = chunk_off[c]; a < a_end; a += C::GROUP, ++g) {
            const int n = min(C::GROUP, a_end - a);
            const int gs = g & 1;
            // operand slots gs were last read by pair g - 2: free once the ring stage of
            // that pair's last block is released (its commit follows every MMA of the pair)
            if (g >= 2) {
              ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SE + tl2 % C::NS), (tl2 / C::NS) & 1, abort_flag));
              if (!ok) break;
            }
            tl2 = tl1;
            tl1 = C::TPB * n_exact + a + n - 1;  // stage use of this pair's last block
            tc_fence_after();
#pragma unroll 1
            for (int qq = 0; qq < n; ++qq) {
              const int k = approx_list[a + qq] - c * C::CHUNK;
              const uint32_t w = a0s[k >> 1];
              const float coef = ((k & 1) ? bf16_hi(w) : bf16_lo(w)) * p.scale;
              const __nv_bfloat162 c2 = __floats2bfloat162_rn(coef, coef);
              const uint32_t cw = *reinterpret_cast<const uint32_t*>(&c2);
              const uint32_t aa = tmem + lrow + C::A_COL0 + (gs * C::GROUP + qq) * C::A_COLS;
#pragma unroll
              for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t t[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) t[i] = hmul2_bf16(qf[ch * 16 + i], cw);
                tmem_st16(aa + ch * 16, t);
              }
            }
            tmem_wait_st();
            tc_fence_before();
            // the pair's S1 tiles (load unit n_exact + g) must have landed as well
            const int u = n_exact + g;
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_TF + u % C::NTF), (u / C::NTF) & 1, abort_flag));
            if (!ok) break;
            warp_arrive(BAR(C::B_GA + gs));
          }
        }
        if (ok && hybrid) {
          // A_H = bf16(s_t * scale * q_t), one rounding from fp32 (operand slot 0)
          const float coef = s_alpha * p.scale;
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t t[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              t[i] = pack_bf16x2(bf16_lo(qf[ch * 16 + i]) * coef, bf16_hi(qf[ch * 16 + i]) * coef);
            tmem_st16(tmem + lrow + C::A_COL0 + ch * 16, t);
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(BAR(C::B_AH));
        }
      }
    }

    // ------------------------------------------------ epilogue
    xl[hf * 128 + r] = l;
    ok = pair_sync_and(pair_id, ok);
    if (ok) {
      ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_ODONE), 0, abort_flag));
      if (ok) {
        tc_fence_after();
        const float inv = 1.f / (l + xl[(hf ^ 1) * 128 + r]);
        bf16* dst = p.O + (size_t(bh) * N + (valid ? grow : 0)) * D + hf * HD;
#pragma unroll
        for (int ch = 0; ch < HD / 16; ++ch) {
          uint32_t o[16];
          tmem_ld16(tmem + lrow + C::O_COL + hf * HD + ch * 16, o);
          tmem_wait_ld(o);
          uint4 w0, w1;
          w0.x = pack_bf16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
          w0.y = pack_bf16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
          w0.z = pack_bf16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
          w0.w = pack_bf16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
          w1.x = pack_bf16x2(__uint_as_float(o[8]) * inv, __uint_as_float(o[9]) * inv);
          w1.y = pack_bf16x2(__uint_as_float(o[10]) * inv, __uint_as_float(o[11]) * inv);
          w1.z = pack_bf16x2(__uint_as_float(o[12]) * inv, __uint_as_float(o[13]) * inv);
          w1.w = pack_bf16x2(__uint_as_float(o[14]) * inv, __uint_as_float(o[15]) * inv);
          if (valid) {
            reinterpret_cast<uint4*>(dst + ch * 16)[0] = w0;
            reinterpret_cast<uint4*>(dst + ch * 16)[1] = w1;
          }
        }
      }
    }
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
#undef BAR
}

}  // namespace pisa
