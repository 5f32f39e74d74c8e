// Plain critical-block selection as one persistent, warp-specialised kernel.
//
// PISA explainer, technical summary section 2, "Covariance-aware routing": the key
// blocks most relevant by attention score go to the exact path; the relevance of key
// block j to query block i is the pooled score qbar_i . kbar_j (qbar_i = mean of the
// query block's real rows), plus lambda * M_j when covariance-aware routing is on. The
// arithmetic is the one of select_kernel (fp32 pooling in packed pairs, fp32 scores as
// even / odd dimension partial sums, top-k with ties to the lower block index); this
// kernel only reorganises the work so that reading Q from HBM, scoring and the top-k
// overlap.
//
// One CTA per SM walks tiles of kSpRows query blocks of one head (tile t, t + grid, ...).
// Warp roles (384 threads: three warps per SM sub-partition, 168 registers each):
//   warp 0      Q producer: each query block of the CTA's tiles (block rows x D bf16,
//               contiguous in HBM) as one bulk copy into a ring of shared-memory stages;
//               it runs ahead of everything else, bounded only by the ring;
//   warp 1      kbar producer: the tile's head's kbar, one 8-dimension plane at a time
//               ([nB rows][32 bytes], 32-byte swizzled, a 3-D TMA box per up to 256
//               rows), through a ring of plane buffers (kbar is L2-resident);
//   warps 2-3   pooling: a landed query block is summed row by row from shared memory
//               and its mean written into the tile's qbar buffer (two buffers: the
//               next tile's pooling overlaps this tile's scoring);
//   warps 4-11  scoring and top-k. Lane (rg, kg) = (lane & 3, lane >> 2) of score warp w
//               accumulates rows rg + 4i (i < 4) against key blocks 64m + 8w + kg
//               (m < KL): the 8 key rows a warp reads per load are consecutive (the
//               32-byte swizzle puts their 16-byte halves in distinct banks) and its 4
//               query rows are consecutive, so every shared-memory read is one
//               wavefront, and the key blocks of a head spread evenly over the warps for
//               any nB. Scores become order-preserving keys in one of two key buffers;
//               after one named barrier each warp takes the top-k of its two rows
//               together (two independent dependency chains) while the next tile is
//               being pooled.
// Ring positions and phases advance incrementally. All waits are bounded; a CTA whose
// wait runs out raises the device error word, its producers drain the copies they
// issued, and the score warps keep meeting their named barrier until the tile loop ends.
#pragma once

#include "tc_ptx.cuh"
#include "select.cuh"

namespace pisa {

constexpr int kSpThreads = 384;
constexpr int kSpRows = 16;        // query blocks per tile
constexpr int kSpPoolWarps = 2;
constexpr int kSpScoreWarps = 8;
constexpr int kSpMaxQS = 8;        // Q ring stages, at most
constexpr int kSpMaxKS = 4;        // kbar plane buffers, at most
constexpr int kSpMaxKL = 10;       // key blocks per lane (nB <= 640)
constexpr int kSpPlane = 8;        // kbar dimensions per plane
constexpr int kSpTkScratchLd = 640;  // top-k scratch words per score warp

struct SpParams {
  const bf16* Q;
  const float* route;  // fp32 [B*H][nB] or nullptr
  float lambda;
  int32_t* idx;
  int N, nB, block, topk;
  int tiles_per_head, tiles;
  int ld;              // key-buffer row stride (uint32), 8 mod 32
  int nqs, nks;        // Q ring stages, kbar plane buffers
  int qstage;          // bytes per Q stage (block * D * 2)
  int prows;           // rows per kbar plane buffer
  int nbox, box_rows;  // TMA boxes per plane and rows per box
  int off_q, off_k, off_qb, off_keys, off_bar;  // shared-memory offsets (1024-aligned base)
  int off_scr;         // top-k scratch of its own, or -1: in the idle key buffer
  int smem;            // dynamic shared memory to request
};

// Shared-memory plan for d = D and nB key blocks with KL key blocks per lane; false when
// it does not fit (the caller then uses select_kernel).
template <int D>
inline bool select_pipe_plan(int nB, int block, int KL, SpParams& p) {
  constexpr int kBudget = 227 * 1024;
  p.nbox = (nB + 255) / 256;
  p.box_rows = ((nB + p.nbox - 1) / p.nbox + 7) / 8 * 8;
  p.prows = 64 * KL > p.nbox * p.box_rows ? 64 * KL : p.nbox * p.box_rows;
  p.ld = (nB + 31) / 32 * 32 + 8;
  p.qstage = block * D * 2;
  const int plane = p.prows * kSpPlane * 4;
  const int keys = 2 * kSpRows * p.ld * 4;
  const int qb = 2 * kSpRows * D * 4;
  const int bars = (2 * kSpMaxQS + 2 * kSpMaxKS + 4) * 8 + 16;
  // top-k scratch: kSpTkScratchLd words per score warp, inside the idle key buffer when it
  // is large enough
  const int scr_need = kSpScoreWarps * kSpTkScratchLd * 4;
  const int scr = kSpRows * p.ld * 4 >= scr_need ? 0 : scr_need;
  for (int nks = kSpMaxKS; nks >= 2; --nks) {
    const int fixed = nks * plane + keys + qb + scr + bars + 1024;  // + base alignment slack
    int nqs = (kBudget - fixed) / p.qstage;
    if (nqs > kSpMaxQS) nqs = kSpMaxQS;
    nqs -= nqs % kSpPoolWarps;  // every stage keeps one consumer warp (see the pooling role)
    if (nqs < kSpPoolWarps) continue;
    p.nks = nks;
    p.nqs = nqs;
    p.off_k = 0;  // plane buffers first: 256-byte alignment for the 32-byte swizzle
    p.off_q = p.off_k + nks * plane;
    p.off_qb = p.off_q + nqs * p.qstage;
    p.off_keys = p.off_qb + qb;
    p.off_scr = scr ? p.off_keys + keys : -1;
    p.off_bar = p.off_keys + keys + scr;
    p.smem = p.off_bar + bars + 1024;
    return true;
  }
  return false;
}

namespace sp {

__device__ __forceinline__ void score_warps_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// position in a ring of n slots and the phase parity of its barrier
struct Ring {
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void step(int by, int n) {
    s += by;
    if (s >= n) {
      s -= n;
      ph ^= 1u;
    }
  }
};

// uint32 order key -> the float it encodes (inverse of float_order_key)
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

constexpr int kTkBins = 256;                      // histogram buckets per row
constexpr int kTkScratch = 2 * kTkBins + 2 * 32 + 2;  // words of scratch per warp (two rows)
static_assert(kTkScratch <= kSpTkScratchLd, "top-k scratch");

// The top k of two rows of L keys (uint32 order keys, larger = better; KPL per lane,
// L <= 32 KPL) in shared memory; row B may be absent (hasB false: it repeats row A and
// nothing is written for it). Result as warp_topk: the k largest keys, among keys equal
// to the k-th largest the lowest positions, written in ascending position order.
//
// Warp collectives have long latency, so the threshold (the k-th largest key T) is found
// with few dependent steps instead of a bit-by-bit search:
//   1. lb, a lower bound of T: with j = ceil(k/32) and L >= 32 j, every lane holds j
//      keys at least as large as its own j-th largest, so at least k keys reach the
//      smallest of those (otherwise lb = the row minimum);
//   2. keys >= lb go to 256 buckets by value, b(x) = floor(256 (x - lb) / (max - lb))
//      clamped to [0, 255]: monotone in x, so a higher bucket holds only larger keys
//      and equal keys share a bucket; counts by shared-memory atomics;
//   3. one suffix scan over the buckets finds b*, the bucket with fewer than k keys
//      above it and at least k from it on; T is the (k - above)-th largest key of b*,
//      found by ranking b*'s keys against each other (a bit search over the whole row
//      when b* holds more than 32 keys, or when the bucket width is not finite);
//   4. emission from ballots: keys > T, then keys == T lowest positions first, up to k.
// Each step is a chain of dependent operations of one warp; two rows run side by side.
// `scr` holds kTkScratch words, this warp's alone for the call.
template <int KPL>
__device__ void topk_two_rows(const uint32_t* rowA, const uint32_t* rowB, bool hasB, int L, int k, int32_t* outA,
                              int32_t* outB, uint32_t* scr) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const uint32_t* rows[2] = {rowA, rowB};
  int32_t* outs[2] = {outA, outB};
  uint32_t* hist = scr;                  // [2][kTkBins]
  uint32_t* list = scr + 2 * kTkBins;    // [2][32]
  uint32_t* cnt = list + 64;             // [2]
  __syncwarp();                          // the previous call's reads of the scratch are done
#pragma unroll
  for (int e = lane; e < 2 * kTkBins; e += 32) hist[e] = 0u;
  if (lane < 2) cnt[lane] = 0u;
  uint32_t key[2][KPL];
  uint32_t m1[2], m2[2], mn[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    m1[r] = 0u;
    m2[r] = 0u;
    mn[r] = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      const int jj = 32 * i + lane;
      key[r][i] = jj < L ? rows[r][jj] : 0u;
      if (jj < L) {
        m2[r] = max(m2[r], min(m1[r], key[r][i]));
        m1[r] = max(m1[r], key[r][i]);
        mn[r] = min(mn[r], key[r][i]);
      }
    }
  }
  const int j = (k + 31) / 32;
  const bool by_lanes = j <= 2 && L >= 32 * j;
  uint32_t mx[2], lb[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    mx[r] = __reduce_max_sync(0xffffffffu, m1[r]);
    lb[r] = __reduce_min_sync(0xffffffffu, by_lanes ? (j == 1 ? m1[r] : m2[r]) : mn[r]);
  }
  float xlb[2], scl[2];
  bool fine[2];  // buckets usable: a finite, nonzero bucket width
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    xlb[r] = key_float(lb[r]);
    scl[r] = float(kTkBins) / (key_float(mx[r]) - xlb[r]);
    fine[r] = lb[r] != mx[r] && isfinite(scl[r]) && scl[r] > 0.f;
  }
  auto bucket = [&](int r, uint32_t kv) -> int {
    const float t = fminf(fmaxf((key_float(kv) - xlb[r]) * scl[r], 0.f), float(kTkBins - 1));
    return int(t);
  };
  __syncwarp();  // cleared histogram visible to every lane
#pragma unroll
  for (int r = 0; r < 2; ++r)
    if (fine[r])
#pragma unroll
      for (int i = 0; i < KPL; ++i)
        if (32 * i + lane < L && key[r][i] >= lb[r]) atomicAdd(&hist[r * kTkBins + bucket(r, key[r][i])], 1u);
  __syncwarp();
  // lane l owns buckets [8 l, 8 l + 8); above = keys in higher buckets
  int bstar[2] = {0, 0}, above[2] = {0, 0};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (!fine[r]) continue;
    uint32_t c[8];
    uint32_t tot = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = hist[r * kTkBins + 8 * lane + e];
      tot += c[e];
    }
    uint32_t suf = tot;  // inclusive suffix over lanes >= l
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += t;
    }
    uint32_t run = suf - tot;  // keys in buckets of higher lanes
    int mine = -1, my_above = 0;
#pragma unroll
    for (int e = 7; e >= 0; --e) {
      if (mine < 0 && run < uint32_t(k) && uint32_t(k) <= run + c[e]) {
        mine = 8 * lane + e;
        my_above = int(run);
      }
      run += c[e];
    }
    const unsigned who = __ballot_sync(0xffffffffu, mine >= 0);
    const int src = __ffs(who) - 1;  // exactly one lane holds b*
    bstar[r] = __shfl_sync(0xffffffffu, mine, src);
    above[r] = __shfl_sync(0xffffffffu, my_above, src);
  }
  // the keys of bucket b* (at most 32 kept)
#pragma unroll
  for (int r = 0; r < 2; ++r)
    if (fine[r])
#pragma unroll
      for (int i = 0; i < KPL; ++i)
        if (32 * i + lane < L && key[r][i] >= lb[r] && bucket(r, key[r][i]) == bstar[r]) {
          const uint32_t slot = atomicAdd(&cnt[r], 1u);
          if (slot < 32u) list[r * 32 + slot] = key[r][i];
        }
  __syncwarp();
  uint32_t T[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int n = int(cnt[r]);
    if (fine[r] && n <= 32) {
      const int need = k - above[r];  // 1 <= need <= n
      const uint32_t v = lane < n ? list[r * 32 + lane] : 0u;
      int gt = 0, ge = 0;
      for (int e = 0; e < n; ++e) {
        const uint32_t w = list[r * 32 + e];
        gt += w > v;
        ge += w >= v;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, lane < n && gt < need && need <= ge);
      T[r] = __shfl_sync(0xffffffffu, v, __ffs(hit) - 1);
    } else if (lb[r] == mx[r]) {
      T[r] = mx[r];  // at least k keys reach lb = max: the k-th largest is the maximum
    } else {
      // bit search over the row: invariant at least k keys >= T; bits above the first
      // difference of lb and max are common to every candidate
      const uint32_t dd = lb[r] ^ mx[r];
      const int top = 31 - __clz(dd);
      uint32_t t = top >= 31 ? 0u : (mx[r] & ~((2u << top) - 1u));
      for (int bit = top; bit >= 0; --bit) {
        const uint32_t cand = t | (1u << bit);
        unsigned c = 0;
#pragma unroll
        for (int i = 0; i < KPL; ++i) c += (32 * i + lane < L) && key[r][i] >= cand;
        if (__reduce_add_sync(0xffffffffu, c) >= unsigned(k)) t = cand;
      }
      T[r] = t;
    }
  }
  // emission: keys > T, then keys == T lowest positions first, up to k
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (r == 1 && !hasB) break;
    unsigned c = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) c += (32 * i + lane < L) && key[r][i] > T[r];
    int eq_left = k - int(__reduce_add_sync(0xffffffffu, c));  // equal keys to take, lowest positions first
    int written = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      const bool in = 32 * i + lane < L;
      unsigned take = __ballot_sync(0xffffffffu, in && key[r][i] > T[r]);
      unsigned e = __ballot_sync(0xffffffffu, in && key[r][i] == T[r]);
      if (eq_left > 0 && e != 0u) {
        if (__popc(e) <= eq_left) {
          take |= e;
          eq_left -= __popc(e);
        } else {
          for (; eq_left > 0; --eq_left) {
            take |= e & (0u - e);  // lowest set bit
            e &= e - 1u;
          }
        }
      }
      if ((take >> lane) & 1u) outs[r][written + __popc(take & lt_mask)] = 32 * i + lane;
      written += __popc(take);
    }
  }
}

}  // namespace sp

template <int D, int KL>
__global__ void __launch_bounds__(kSpThreads, 1)
select_pipe_kernel(const __grid_constant__ CUtensorMap tmKb, const SpParams p) {
  using namespace tc;
  extern __shared__ __align__(16) uint8_t sp_smem_raw[];
  const uint32_t raw_u = smem_u32(sp_smem_raw);
  const uint32_t base_u = (raw_u + 1023u) & ~1023u;
  uint8_t* base = sp_smem_raw + (base_u - raw_u);
  const uint32_t bar0 = base_u + p.off_bar;
  // barriers: QF[kSpMaxQS] QE[kSpMaxQS] KF[kSpMaxKS] KE[kSpMaxKS] QBF[2] QBE[2]
  auto QF = [&](int s) { return bar0 + 8u * uint32_t(s); };
  auto QE = [&](int s) { return bar0 + 8u * uint32_t(kSpMaxQS + s); };
  auto KF = [&](int s) { return bar0 + 8u * uint32_t(2 * kSpMaxQS + s); };
  auto KE = [&](int s) { return bar0 + 8u * uint32_t(2 * kSpMaxQS + kSpMaxKS + s); };
  auto QBF = [&](int b) { return bar0 + 8u * uint32_t(2 * kSpMaxQS + 2 * kSpMaxKS + b); };
  auto QBE = [&](int b) { return bar0 + 8u * uint32_t(2 * kSpMaxQS + 2 * kSpMaxKS + 2 + b); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + p.off_bar + (2 * kSpMaxQS + 2 * kSpMaxKS + 4) * 8);
  constexpr int NPL = D / kSpPlane;  // planes per tile
  constexpr int KPL = (2 * KL + 3) / 4 * 4;  // top-k keys per lane (L <= 64 KL), a multiple of 4
  const int pbytes = p.prows * kSpPlane * 4;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int nt = (p.tiles - int(blockIdx.x) + G - 1) / G;  // tiles of this CTA
  auto tile_of = [&](int lt, int& bh, int& i0, int& nq) {
    const int t = int(blockIdx.x) + lt * G;
    bh = t / p.tiles_per_head;
    i0 = (t % p.tiles_per_head) * kSpRows;
    nq = min(kSpRows, p.nB - i0);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nqs; ++s) {
      mbar_init(QF(s), 1);
      mbar_init(QE(s), 1);  // the pooling warp that summed the stage
    }
    for (int s = 0; s < p.nks; ++s) {
      mbar_init(KF(s), 1);
      mbar_init(KE(s), kSpScoreWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(QBF(b), kSpPoolWarps);
      mbar_init(QBE(b), kSpScoreWarps);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ Q producer
    if (lane == 0) {
      sp::Ring q;
      int issued = 0;
      bool ok = true;
      for (int lt = 0; lt < nt && ok; ++lt) {
        int bh, i0, nq;
        tile_of(lt, bh, i0, nq);
        for (int r = 0; r < nq; ++r) {
          if (!(ok = wait_bounded(QE(q.s), q.ph ^ 1u, abort_flag))) break;
          const int i = i0 + r;
          const int n = min(p.block, p.N - i * p.block);
          const uint32_t bytes = uint32_t(n) * D * 2u;
          mbar_arrive_expect_tx(QF(q.s), bytes);
          bulk_load(base_u + uint32_t(p.off_q + q.s * p.qstage), p.Q + (size_t(bh) * p.N + size_t(i) * p.block) * D,
                    bytes, QF(q.s));
          q.step(1, p.nqs);
          ++issued;
        }
      }
      // no copy may still be in flight when the CTA exits: wait for the last
      // min(issued, nqs) copies, walking the ring backwards from the next position
      for (int c = 0; c < p.nqs && c < issued; ++c) {
        if (q.s == 0) {
          q.s = p.nqs - 1;
          q.ph ^= 1u;
        } else {
          --q.s;
        }
        wait_drain(QF(q.s), q.ph);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ kbar producer
    if (lane == 0) {
      const uint32_t tx = uint32_t(p.nbox * p.box_rows) * kSpPlane * 4u;
      sp::Ring k;
      int issued = 0;
      bool ok = true;
      for (int lt = 0; lt < nt && ok; ++lt) {
        int bh, i0, nq;
        tile_of(lt, bh, i0, nq);
        for (int pl = 0; pl < NPL; ++pl) {
          if (!(ok = wait_bounded(KE(k.s), k.ph ^ 1u, abort_flag))) break;
          mbar_arrive_expect_tx(KF(k.s), tx);
          const uint32_t dst = base_u + uint32_t(p.off_k + k.s * pbytes);
          for (int c = 0; c < p.nbox; ++c)
            tma_load_3d(dst + uint32_t(c * p.box_rows * kSpPlane * 4), &tmKb, KF(k.s), kSpPlane * pl,
                        c * p.box_rows, bh);
          k.step(1, p.nks);
          ++issued;
        }
      }
      for (int c = 0; c < p.nks && c < issued; ++c) {
        if (k.s == 0) {
          k.s = p.nks - 1;
          k.ph ^= 1u;
        } else {
          --k.s;
        }
        wait_drain(KF(k.s), k.ph);
      }
    }
  } else if (warp < 2 + kSpPoolWarps) {
    // ------------------------------------------------------------ pooling
    // Pooling warp pw takes the stage uses u = pw, pw + kSpPoolWarps, ... (query block
    // r of a tile is use ubase + r). The stage count is a multiple of kSpPoolWarps, so
    // each stage has one consumer, which meets every phase of the stage's barrier in
    // order: a consumer that skipped a phase could wait on a parity two phases ahead
    // and pass before its copy has landed.
    // lane: 16-byte chunk c16 of a row (8 dimensions), rows r0, r0 + RSTEP, ...
    constexpr int CH = D / 8, RSTEP = 32 / CH;
    const int pw = warp - 2;
    const int c16 = lane % CH, r0 = lane / CH;
    sp::Ring q;
    q.s = pw;
    int ubase = 0;     // stage uses before this tile
    sp::Ring qbr;      // qbar buffer and the phase of its barriers
    for (int lt = 0; lt < nt; ++lt) {
      int bh, i0, nq;
      tile_of(lt, bh, i0, nq);
      const int b = qbr.s;
      // the buffer was last read by the scoring of tile lt - 2
      if (!__all_sync(0xffffffffu, wait_bounded(QBE(b), qbr.ph ^ 1u, abort_flag))) break;
      float* qb = reinterpret_cast<float*>(base + p.off_qb) + b * (kSpRows * D);  // [D/4 planes][kSpRows][4]
      bool ok = true;
      for (int r = (pw - ubase % kSpPoolWarps + kSpPoolWarps) % kSpPoolWarps; r < kSpRows; r += kSpPoolWarps) {
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        float inv = 0.f;  // rows past the head's last query block pool to zero
        if (r < nq) {
          if (!(ok = __all_sync(0xffffffffu, wait_bounded(QF(q.s), q.ph, abort_flag)))) break;
          const int n = min(p.block, p.N - (i0 + r) * p.block);
          const uint8_t* src = base + p.off_q + q.s * p.qstage + c16 * 16;
#pragma unroll 4
          for (int rr = r0; rr < n; rr += RSTEP) {
            const uint4 w = *reinterpret_cast<const uint4*>(src + rr * (D * 2));
            sel::add2(acc[0], sel::pack2(w.x << 16, w.x & 0xffff0000u));
            sel::add2(acc[1], sel::pack2(w.y << 16, w.y & 0xffff0000u));
            sel::add2(acc[2], sel::pack2(w.z << 16, w.z & 0xffff0000u));
            sel::add2(acc[3], sel::pack2(w.w << 16, w.w & 0xffff0000u));
          }
          warp_arrive(QE(q.s));  // every lane's reads of the stage are done
          q.step(kSpPoolWarps, p.nqs);
          inv = 1.f / float(n);
        }
        // lanes holding the same chunk sit CH apart
#pragma unroll
        for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 v = sel::unpack2(acc[e]);
            const float a = __shfl_xor_sync(0xffffffffu, v.x, off), c = __shfl_xor_sync(0xffffffffu, v.y, off);
            sel::add2(acc[e], sel::pack2(__float_as_uint(a), __float_as_uint(c)));
          }
        }
        if (lane < CH) {
          const float2 v0 = sel::unpack2(acc[0]), v1 = sel::unpack2(acc[1]);
          const float2 v2 = sel::unpack2(acc[2]), v3 = sel::unpack2(acc[3]);
          *reinterpret_cast<float4*>(qb + ((2 * c16) * kSpRows + r) * 4) =
              make_float4(v0.x * inv, v0.y * inv, v1.x * inv, v1.y * inv);
          *reinterpret_cast<float4*>(qb + ((2 * c16 + 1) * kSpRows + r) * 4) =
              make_float4(v2.x * inv, v2.y * inv, v3.x * inv, v3.y * inv);
        }
      }
      if (!ok) break;
      warp_arrive(QBF(b));
      qbr.step(1, 2);
      ubase += nq;
    }
  } else {
    // ------------------------------------------------------------ scoring and top-k
    const int sw = warp - 2 - kSpPoolWarps;
    const int rg = lane & 3, kg = lane >> 2;
    // 16-byte half h of a key row sits at half h ^ ((key >> 2) & 1) (32-byte swizzle);
    // (key >> 2) & 1 = (kg >> 2) & 1 for every key 64m + 8sw + kg of this lane
    const int hx = (kg >> 2) & 1;
    uint32_t* keys0 = reinterpret_cast<uint32_t*>(base + p.off_keys);
    bool ok = true;
    sp::Ring k;
    sp::Ring qbr;
    for (int lt = 0; lt < nt; ++lt) {
      int bh, i0, nq;
      tile_of(lt, bh, i0, nq);
      const int b = qbr.s;
      const float* qb = reinterpret_cast<const float*>(base + p.off_qb) + b * (kSpRows * D);
      uint32_t* keys = keys0 + b * (kSpRows * p.ld);
      uint64_t acc[4][KL];  // (even-dimension, odd-dimension) partial sums
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < KL; ++m) acc[i][m] = 0ull;
      if (ok) ok = __all_sync(0xffffffffu, wait_bounded(QBF(b), qbr.ph, abort_flag));
      if (ok) {
#pragma unroll 1
        for (int pl = 0; pl < NPL; ++pl) {
          if (!(ok = __all_sync(0xffffffffu, wait_bounded(KF(k.s), k.ph, abort_flag)))) break;
          const uint8_t* kp = base + p.off_k + k.s * pbytes + (8 * sw + kg) * (kSpPlane * 4);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint64_t xa[4], xb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 x = *reinterpret_cast<const uint4*>(qb + ((2 * pl + h) * kSpRows + rg + 4 * i) * 4);
              xa[i] = sel::pack2(x.x, x.y);
              xb[i] = sel::pack2(x.z, x.w);
            }
#pragma unroll
            for (int m = 0; m < KL; ++m) {
              const uint4 kv = *reinterpret_cast<const uint4*>(kp + m * (64 * kSpPlane * 4) + ((h ^ hx) << 4));
              const uint64_t ka = sel::pack2(kv.x, kv.y), kb = sel::pack2(kv.z, kv.w);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                sel::fma2(acc[i][m], xa[i], ka);
                sel::fma2(acc[i][m], xb[i], kb);
              }
            }
          }
          warp_arrive(KE(k.s));
          k.step(1, p.nks);
        }
        if (ok) warp_arrive(QBE(b));
      }
      // every score warp has finished the previous tile's top-k, whose scratch may lie in
      // the key buffer written next
      sp::score_warps_sync();
      if (ok) {
        const float* route_head = p.route ? p.route + size_t(bh) * p.nB : nullptr;
#pragma unroll
        for (int m = 0; m < KL; ++m) {
          const int j = 64 * m + 8 * sw + kg;
          if (j < p.nB) {
            const float bias = route_head != nullptr ? p.lambda * route_head[j] : 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 sc = sel::unpack2(acc[i][m]);
              keys[(rg + 4 * i) * p.ld + j] = float_order_key((sc.x + sc.y) + bias + 0.f);  // -0 -> +0
            }
          }
        }
      }
      qbr.step(1, 2);
      sp::score_warps_sync();  // met by every score warp on every tile, also after a failed wait
      if (ok && sw < nq) {
        const int rb = sw + kSpScoreWarps;
        const bool hasB = rb < nq;
        int32_t* out = p.idx + (size_t(bh) * p.nB + i0) * p.topk;
        // scratch: this warp's slice of the other key buffer (no score warp writes it before
        // the barrier that follows the next tile's plane loop), or a region of its own
        uint32_t* scr = (p.off_scr < 0 ? keys0 + (b ^ 1) * (kSpRows * p.ld)
                                       : reinterpret_cast<uint32_t*>(base + p.off_scr)) +
                        sw * kSpTkScratchLd;
        sp::topk_two_rows<KPL>(keys + sw * p.ld, keys + (hasB ? rb : sw) * p.ld, hasB, p.nB, p.topk,
                               out + size_t(sw) * p.topk, out + size_t(hasB ? rb : sw) * p.topk, scr);
      }
    }
  }
}

}  // namespace pisa
