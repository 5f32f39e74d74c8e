// Critical-block selection: pooled queries, fp32 pooled scores and a per-row warp top-k,
// with optional grouped proxy queries.
//
// PISA explainer, technical summary section 2, "Covariance-aware routing": the blocks
// most relevant by attention score are routed to the exact path. The relevance of key
// block j to query block i is the pooled score qbar_i . kbar_j, with qbar_i the mean of
// the query block's real rows (fp32 throughout, so that the ranking matches an exact
// evaluation except at near-ties); with covariance-aware routing each key block's score
// also carries lambda * M_j, M_j = || S1_j - Hbar ||_F (routing.cuh).
//
// Grouped proxies (PIVOT page, "Two observations behind PIVOT"): g consecutive query
// blocks share one proxy query, the mean of all their real rows; the proxy is scored
// against every key block and keeps its `cand` best as a candidate list; each member
// query block then keeps the topk best of those candidates by its own pooled score
// (cand = topk hands the proxy's list to every member unchanged: the reuse mode).
//
// Kernel layout: persistent CTAs (one per SM), each walking its tiles of QB query blocks
// (QB = 8 for plain selection; a whole number of groups otherwise). Per tile:
//   1. pool: the tile's query rows stream through a shared-memory ring of 64-row stages
//      filled by bulk copies (cp.async.bulk, completion on an mbarrier per stage). Warp
//      r sums query block r alone (16-byte shared reads, packed f32x2 adds, one shuffle
//      reduction), then refills the ring slot it just read with the stage `ring` stages
//      ahead -- the next tile's rows land while this tile is scored;
//   2. score: rows (pooled queries, or proxies) against key blocks. Each lane owns two
//      key blocks of 32-block groups spread over the warps and every row of the tile;
//      kbar streams through per-warp padded slabs (8 dimensions, cp.async, double
//      buffered, conflict-free 16-byte reads) and the products accumulate as packed
//      f32x2 FMAs in even / odd dimension pairs. Scores become order-preserving uint32
//      keys in shared memory;
//   3. top-k: one warp per row finds the k-th largest key bit by bit (starting below
//      the row's common prefix) and emits the winners in ascending block order with
//      ballots; among keys equal to the threshold the lowest indices are taken;
//   4. grouped selection only: proxies first keep `cand` candidates (steps 2-3 over all
//      key blocks), then the members are scored against their group's candidates
//      (kbar rows gathered by index) and keep topk of them.
// Every mbarrier wait is bounded (about a second); a wait that runs out raises the
// device error word and the CTA stops issuing work.
#pragma once

#include "common.cuh"

namespace pisa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelQB = 8;                   // query blocks per tile (plain selection)
constexpr int kSelMaxGroup = 8;             // query blocks per proxy, at most
constexpr int kSelStageRows = 64;           // query rows per ring stage
constexpr int kSelSlab = 8;                 // kbar dimensions per slab
constexpr int kSelSlabLd = 12;              // padded slab row (floats): conflict-free 16-byte reads
constexpr int kSelSlabBuf = 2 * 32 * kSelSlabLd;  // one slab buffer: two 32-row groups (floats)
constexpr long long kSelWaitCycles = 2000000000LL;

struct SelParams {
  const bf16* Q;
  const float* kbar;
  const float* route;  // fp32 [B*H][nB] or nullptr
  float lambda;
  int32_t* idx;
  int N, nB, block, topk;
  int group;           // query blocks per proxy (1: each query block is its own)
  int cand;            // candidate list length (nB with group 1: plain selection)
  int QB;              // query blocks per tile (a multiple of group)
  int tiles_per_head, total_tiles;
  int ring;            // ring stages
  int ld;              // key row stride (uint32)
};

__host__ __device__ constexpr int select_key_ld(int nB) { return ((nB + 31) / 32) * 32 + 4; }

// shared-memory carve-up (byte offsets; the ring comes first, 128-byte aligned)
struct SelSmem {
  int ring_off, bar_off, qsum_off, qmean_off, proxy_off, key_off, cand_off, slab_off, misc_off, bytes;
};

__host__ __device__ inline SelSmem select_smem(int D, int nB, int ring) {
  SelSmem s{};
  int off = 0;
  auto take = [&](int bytes, int align) {
    off = (off + align - 1) / align * align;
    const int at = off;
    off += bytes;
    return at;
  };
  s.ring_off = take(ring * kSelStageRows * D * 2, 128);
  s.bar_off = take(ring * 8, 8);
  s.qsum_off = take(kSelQB * D * 4, 16);
  s.qmean_off = take(kSelQB * D * 4, 16);
  s.proxy_off = take(kSelQB * D * 4, 16);
  s.key_off = take(kSelQB * select_key_ld(nB) * 4, 16);
  s.cand_off = take(kSelQB * ((nB + 7) / 8 * 8) * 2, 16);
  s.slab_off = take(kSelWarps * 2 * kSelSlabBuf * 4, 16);
  s.misc_off = take(16, 16);
  s.bytes = off;
  return s;
}

namespace sel {

__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}
// acc += x, two fp32 lanes, round to nearest
__device__ __forceinline__ void add2(uint64_t& acc, uint64_t x) { asm("add.rn.f32x2 %0, %0, %1;" : "+l"(acc) : "l"(x)); }
// acc += a * b, two fp32 lanes, one rounding each
__device__ __forceinline__ void fma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait: false (and the device error word raised) when it runs out
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (clock64() - t0 > kSelWaitCycles) {
      flag_error(kErrTimeout);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Top `k` of row[0, L) (uint32 keys, larger = better) by one warp; writes the winning
// positions, mapped through `map` when given, to out[0, k) in ascending position order.
// Keys equal to the k-th largest are taken lowest position first.
template <typename OutT>
__device__ void warp_topk(const uint32_t* row, int L, int k, OutT* out, const int16_t* map) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  // the k-th largest key lies between the row's extremes: bits above their first
  // difference are common to every candidate threshold
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int jj = lane; jj < L; jj += 32) {
    const uint32_t v = row[jj];
    kmin = min(kmin, v);
    kmax = max(kmax, v);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const uint32_t diff = kmin ^ kmax;
  const int top = diff ? 31 - __clz(diff) : -1;  // highest differing bit
  uint32_t T = top < 0 ? kmax : (top >= 31 ? 0u : (kmax & ~((2u << top) - 1u)));
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    unsigned cnt = 0;
    for (int jj = lane; jj < L; jj += 32) cnt += row[jj] >= cand;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= unsigned(k)) T = cand;
  }
  unsigned gt = 0;
  for (int jj = lane; jj < L; jj += 32) gt += row[jj] > T;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need_eq = k - int(gt);
  int written = 0, eq_seen = 0;
  for (int base = 0; base < L; base += 32) {
    const int jj = base + lane;
    const uint32_t key = jj < L ? row[jj] : 0u;
    const bool is_gt = jj < L && key > T;
    const bool is_eq = jj < L && key == T;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const bool take = is_gt || (is_eq && eq_seen + __popc(eq_mask & lt_mask) < need_eq);
    const unsigned take_mask = __ballot_sync(0xffffffffu, take);
    if (take) out[written + __popc(take_mask & lt_mask)] = OutT(map ? int(map[jj]) : jj);
    written += __popc(take_mask);
    eq_seen += __popc(eq_mask);
  }
}

// Scores of R rows (fp32 [R][D] in shared memory) against the key blocks list[0, L)
// (list == nullptr: blocks 0..L-1), as keys[r * ld + position]. Work units are 32-block
// groups, two per pass per warp, spread over the CTA's warps. The caller synchronises
// the CTA before and after.
template <int D, int R>
__device__ void score_rows(int nrows, const float* rows, const float* kb_head, const float* route_head, float lambda,
                           const int16_t* list, int L, uint32_t* keys, int ld, float* slab) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ngroups = (L + 31) / 32;
  const uint32_t slab_u = smem_u32(slab);
  constexpr int NSL = D / kSelSlab;
  for (int g0 = warp; g0 < ngroups; g0 += 2 * kSelWarps) {
    const int g1 = g0 + kSelWarps;  // second group of the pass (may not exist)
    // the 4 copies of this lane per slab: (group, row, 16-byte chunk)
    const float* src[4];
    uint32_t dst[4], nbytes[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = lane + 32 * i;
      const int gg = q >> 6, rr = (q >> 1) & 31, cc = q & 1;
      const int pos = (gg ? g1 : g0) * 32 + rr;
      const bool in = pos < L;
      const int j = in ? (list ? int(list[pos]) : pos) : 0;
      src[i] = kb_head + size_t(j) * D + cc * 4;
      dst[i] = uint32_t((gg * 32 + rr) * kSelSlabLd + cc * 4) * 4u;
      nbytes[i] = in ? 16u : 0u;
    }
    auto issue = [&](int sl) {
      const uint32_t b = slab_u + uint32_t((sl & 1) * kSelSlabBuf) * 4u;
#pragma unroll
      for (int i = 0; i < 4; ++i) cp16(b + dst[i], src[i] + sl * kSelSlab, nbytes[i]);
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    uint64_t acc[R][2];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = 0ull;
    issue(0);
#pragma unroll 1
    for (int sl = 0; sl < NSL; ++sl) {
      if (sl + 1 < NSL) {
        issue(sl + 1);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncwarp();
      const float* buf = slab + (sl & 1) * kSelSlabBuf;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint4 k0 = *reinterpret_cast<const uint4*>(buf + lane * kSelSlabLd + 4 * c);
        const uint4 k1 = *reinterpret_cast<const uint4*>(buf + (32 + lane) * kSelSlabLd + 4 * c);
        const uint64_t k0a = pack2(k0.x, k0.y), k0b = pack2(k0.z, k0.w);
        const uint64_t k1a = pack2(k1.x, k1.y), k1b = pack2(k1.z, k1.w);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint4 x = *reinterpret_cast<const uint4*>(rows + r * D + sl * kSelSlab + 4 * c);
          const uint64_t xa = pack2(x.x, x.y), xb = pack2(x.z, x.w);
          fma2(acc[r][0], xa, k0a);
          fma2(acc[r][0], xb, k0b);
          fma2(acc[r][1], xa, k1a);
          fma2(acc[r][1], xb, k1b);
        }
      }
      __syncwarp();  // this buffer is refilled two slabs later
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int pos = (t ? g1 : g0) * 32 + lane;
      if (pos < L) {
        const int j = list ? int(list[pos]) : pos;
        const float bias = route_head != nullptr ? lambda * route_head[j] : 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float2 s = unpack2(acc[r][t]);
          if (r < nrows) keys[r * ld + pos] = float_order_key((s.x + s.y) + bias + 0.f);  // -0 -> +0
        }
      }
    }
  }
}

template <int D>
__device__ void score_dispatch(int R, const float* rows, const float* kb_head, const float* route_head, float lambda,
                               const int16_t* list, int L, uint32_t* keys, int ld, float* slab) {
  // rows past R read whatever the row buffer holds; their keys are not stored
  if (R <= 1) score_rows<D, 1>(R, rows, kb_head, route_head, lambda, list, L, keys, ld, slab);
  else if (R <= 2) score_rows<D, 2>(R, rows, kb_head, route_head, lambda, list, L, keys, ld, slab);
  else if (R <= 4) score_rows<D, 4>(R, rows, kb_head, route_head, lambda, list, L, keys, ld, slab);
  else score_rows<D, 8>(R, rows, kb_head, route_head, lambda, list, L, keys, ld, slab);
}

}  // namespace sel

template <int D>
__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(const SelParams p) {
  extern __shared__ __align__(16) uint8_t sel_smem_raw[];
  uint8_t* sel_smem = sel_smem_raw + ((128u - (smem_u32(sel_smem_raw) & 127u)) & 127u);
  const SelSmem L = select_smem(D, p.nB, p.ring);
  uint8_t* ring = sel_smem + L.ring_off;
  const uint32_t ring_u = smem_u32(ring);
  const uint32_t bar_u = smem_u32(sel_smem + L.bar_off);
  float* qsum = reinterpret_cast<float*>(sel_smem + L.qsum_off);    // [QB][D] row sums
  float* qmean = reinterpret_cast<float*>(sel_smem + L.qmean_off);  // [QB][D] pooled queries
  float* proxy = reinterpret_cast<float*>(sel_smem + L.proxy_off);  // [groups][D] proxy queries
  uint32_t* keys = reinterpret_cast<uint32_t*>(sel_smem + L.key_off);
  int16_t* cand = reinterpret_cast<int16_t*>(sel_smem + L.cand_off);
  const int cand_ld = (p.nB + 7) / 8 * 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* slab = reinterpret_cast<float*>(sel_smem + L.slab_off) + warp * 2 * kSelSlabBuf;
  volatile int* abort_flag = reinterpret_cast<int*>(sel_smem + L.misc_off);

  constexpr int SB = kSelStageRows * D * 2;  // bytes per ring stage
  const int spb = p.block / kSelStageRows;   // stages per query block
  const int spt = p.QB * spb;                // stages per tile
  const int ntiles = p.total_tiles > int(blockIdx.x) ? (p.total_tiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  const bool grouped = p.group > 1 || p.cand < p.nB;
  const int G = p.QB / p.group;              // proxies per tile

  // stage u of this CTA: tile u / spt, query block (u % spt) / spb, part (u % spt) % spb
  auto issue = [&](int u) {
    const int it = u / spt;
    if (it >= ntiles) return;
    const int T = int(blockIdx.x) + it * int(gridDim.x);
    const int k = u % spt, r = k / spb, s = k % spb;
    const int bh = T / p.tiles_per_head;
    const int i = (T % p.tiles_per_head) * p.QB + r;
    int rows = 0;
    if (i < p.nB) rows = max(0, min(kSelStageRows, min(p.block, p.N - i * p.block) - s * kSelStageRows));
    const uint32_t bar = bar_u + 8u * uint32_t(u % p.ring);
    sel::mbar_expect_tx(bar, uint32_t(rows) * D * 2);
    if (rows > 0)
      sel::bulk_load(ring_u + uint32_t(u % p.ring) * SB,
                     p.Q + (size_t(bh) * p.N + size_t(i) * p.block + s * kSelStageRows) * D, uint32_t(rows) * D * 2,
                     bar);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ring; ++s) sel::mbar_init(bar_u + 8u * s, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int u = 0; u < p.ring; ++u) issue(u);

  for (int it = 0; it < ntiles; ++it) {
    const int T = int(blockIdx.x) + it * int(gridDim.x);
    const int bh = T / p.tiles_per_head;
    const int i0 = (T % p.tiles_per_head) * p.QB;
    const int nq = min(p.QB, p.nB - i0);

    // ---- 1. pool: warp r sums query block i0 + r, stage by stage ----
    if (warp < p.QB) {
      constexpr int CH = D / 8;         // 16-byte chunks per row
      constexpr int RSTEP = 32 / CH;    // rows between a lane's rows
      const int c16 = lane % CH, r0 = lane / CH;
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      const int i = i0 + warp;
      const int n = i < p.nB ? min(p.block, p.N - i * p.block) : 0;
      for (int s = 0; s < spb; ++s) {
        const int u = it * spt + warp * spb + s;
        const bool ok = *abort_flag == 0 && sel::mbar_wait(bar_u + 8u * uint32_t(u % p.ring), (u / p.ring) & 1);
        if (!ok) *abort_flag = 1;
        const int rows = max(0, min(kSelStageRows, n - s * kSelStageRows));
        const uint8_t* st = ring + size_t(u % p.ring) * SB;
        if (ok) {
#pragma unroll 4
          for (int r = r0; r < rows; r += RSTEP) {
            const uint4 w = *reinterpret_cast<const uint4*>(st + r * (D * 2) + c16 * 16);
            sel::add2(acc[0], sel::pack2(w.x << 16, w.x & 0xffff0000u));
            sel::add2(acc[1], sel::pack2(w.y << 16, w.y & 0xffff0000u));
            sel::add2(acc[2], sel::pack2(w.z << 16, w.z & 0xffff0000u));
            sel::add2(acc[3], sel::pack2(w.w << 16, w.w & 0xffff0000u));
          }
        }
        __syncwarp();
        // every read of this slot is done: refill it with the stage `ring` ahead
        if (lane == 0 && *abort_flag == 0) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue(u + p.ring);
        }
      }
      // lanes holding the same chunk sit CH apart
#pragma unroll
      for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 v = sel::unpack2(acc[e]);
          const float a = __shfl_xor_sync(0xffffffffu, v.x, off), b = __shfl_xor_sync(0xffffffffu, v.y, off);
          sel::add2(acc[e], sel::pack2(__float_as_uint(a), __float_as_uint(b)));
        }
      }
      if (lane < CH) {
        float* dst = qsum + warp * D + c16 * 8;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 v = sel::unpack2(acc[e]);
          dst[2 * e] = v.x;
          dst[2 * e + 1] = v.y;
        }
      }
    }
    __syncthreads();
    if (*abort_flag) break;
    // pooled queries (means of the real rows) and the groups' proxies
    for (int e = threadIdx.x; e < p.QB * D; e += kSelThreads) {
      const int r = e / D, i = i0 + r;
      const int n = i < p.nB ? min(p.block, p.N - i * p.block) : 1;
      qmean[e] = qsum[e] * (1.f / float(n));
    }
    if (grouped) {
      for (int e = threadIdx.x; e < G * D; e += kSelThreads) {
        const int m = e / D, c = e % D;
        float s = 0.f;
        int n = 0;
        for (int r = m * p.group; r < (m + 1) * p.group; ++r) {
          const int i = i0 + r;
          if (i < p.nB) {
            s += qsum[r * D + c];
            n += min(p.block, p.N - i * p.block);
          }
        }
        proxy[e] = n > 0 ? s * (1.f / float(n)) : 0.f;
      }
    }
    __syncthreads();

    const float* kb_head = p.kbar + size_t(bh) * p.nB * D;
    const float* route_head = p.route ? p.route + size_t(bh) * p.nB : nullptr;
    int32_t* idx_tile = p.idx + (size_t(bh) * p.nB + i0) * p.topk;
    if (!grouped) {
      // ---- 2-3. plain selection ----
      sel::score_dispatch<D>(nq, qmean, kb_head, route_head, p.lambda, nullptr, p.nB, keys, p.ld, slab);
      __syncthreads();
      if (warp < nq) sel::warp_topk(keys + warp * p.ld, p.nB, p.topk, idx_tile + size_t(warp) * p.topk, nullptr);
      __syncthreads();
      continue;
    }
    // ---- 4. grouped: proxies keep `cand` candidates, members keep topk of those ----
    const int ng = (nq + p.group - 1) / p.group;  // groups present in this tile
    sel::score_dispatch<D>(ng, proxy, kb_head, route_head, p.lambda, nullptr, p.nB, keys, p.ld, slab);
    __syncthreads();
    if (warp < ng) sel::warp_topk(keys + warp * p.ld, p.nB, p.cand, cand + warp * cand_ld, nullptr);
    __syncthreads();
    if (p.cand == p.topk) {  // reuse: every member takes its group's list
      for (int e = threadIdx.x; e < nq * p.topk; e += kSelThreads)
        idx_tile[e] = cand[(e / p.topk / p.group) * cand_ld + e % p.topk];
      __syncthreads();
      continue;
    }
    for (int m = 0; m < ng; ++m) {
      const int rows = min(p.group, nq - m * p.group);
      sel::score_dispatch<D>(rows, qmean + m * p.group * D, kb_head, route_head, p.lambda, cand + m * cand_ld, p.cand,
                             keys + m * p.group * p.ld, p.ld, slab);
    }
    __syncthreads();
    if (warp < nq)
      sel::warp_topk(keys + warp * p.ld, p.cand, p.topk, idx_tile + size_t(warp) * p.topk,
                     cand + (warp / p.group) * cand_ld);
    __syncthreads();
  }
}

}  // namespace pisa
