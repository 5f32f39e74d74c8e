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
// Kernel layout: one CTA (256 threads, two per SM) per tile of QB query blocks of one
// head (QB = 8 for plain selection; a whole number of groups otherwise):
//   1. pool: warp r sums query block r alone: batches of 16 independent 16-byte loads
//      per lane (every load of a batch in flight before the first add), packed f32x2
//      adds, one shuffle reduction, no CTA barrier;
//   2. score: rows (pooled queries, or proxies) against key blocks. Each lane owns two
//      key blocks of 32-block groups spread over the warps and every row of the tile;
//      kbar streams through per-warp padded slabs (8 dimensions, cp.async, three
//      buffers: two slabs in flight while one is used; conflict-free 16-byte reads) and
//      the products accumulate as packed f32x2 FMAs in even / odd dimension pairs.
//      Scores become order-preserving uint32 keys in shared memory;
//   3. top-k: one warp per row, the row's keys in registers (up to 1024 of them), finds
//      the k-th largest key bit by bit (starting below the row's common prefix) and
//      emits the winners in ascending block order with ballots; among keys equal to
//      the threshold the lowest indices are taken;
//   4. grouped selection only: proxies first keep `cand` candidates (steps 2-3 over all
//      key blocks), then the members are scored against their group's candidates
//      (kbar rows gathered by index) and keep topk of them.
// Two CTAs share an SM, so one CTA's pooling (HBM) overlaps the other's scoring (FMA).
#pragma once

#include "common.cuh"

namespace pisa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelQB = 8;                   // query blocks per tile (plain selection)
constexpr int kSelMaxGroup = 8;             // query blocks per proxy, at most
constexpr int kSelSlab = 8;                 // kbar dimensions per slab
constexpr int kSelSlabLd = 12;              // padded slab row (floats): conflict-free 16-byte reads
constexpr int kSelSlabBuf = 2 * 32 * kSelSlabLd;  // one slab buffer: two 32-row groups (floats)
constexpr int kSelSlabBufs = 3;             // slab buffers per warp (two in flight)
constexpr int kSelPoolBatch = 16;           // 16-byte query loads in flight per lane

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
  int tiles_per_head;
  int ld;              // key row stride (uint32)
};

__host__ __device__ constexpr int select_key_ld(int nB) { return ((nB + 31) / 32) * 32 + 4; }

// shared-memory carve-up (byte offsets)
struct SelSmem {
  int qsum_off, qmean_off, proxy_off, key_off, cand_off, slab_off, bytes;
};

// (the proxy rows and candidate lists exist only for grouped selection)
__host__ __device__ inline SelSmem select_smem(int D, int nB, bool grouped) {
  SelSmem s{};
  int off = 0;
  auto take = [&](int bytes) {
    const int at = off;
    off += (bytes + 15) / 16 * 16;
    return at;
  };
  s.qsum_off = take(kSelQB * D * 4);
  s.qmean_off = take(kSelQB * D * 4);
  s.proxy_off = take(grouped ? kSelQB * D * 4 : 0);
  s.key_off = take(kSelQB * select_key_ld(nB) * 4);
  s.cand_off = take(grouped ? kSelQB * ((nB + 7) / 8 * 8) * 2 : 0);
  s.slab_off = take(kSelWarps * kSelSlabBufs * kSelSlabBuf * 4);
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

// warp_topk with the row's keys held in registers (KPL per lane, L <= 32 KPL): the bit
// search then reads no shared memory. Positions past L hold key 0, which no threshold
// of real (finite) scores reaches.
template <int KPL, typename OutT>
__device__ void warp_topk_reg(const uint32_t* row, int L, int k, OutT* out, const int16_t* map) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  uint32_t key[KPL];
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int jj = 32 * i + lane;
    key[i] = jj < L ? row[jj] : 0u;
    if (jj < L) {
      kmin = min(kmin, key[i]);
      kmax = max(kmax, key[i]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const uint32_t diff = kmin ^ kmax;
  const int top = diff ? 31 - __clz(diff) : -1;  // highest differing bit
  uint32_t T = top < 0 ? kmax : (top >= 31 ? 0u : (kmax & ~((2u << top) - 1u)));
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    unsigned cnt = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) cnt += key[i] >= cand;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= unsigned(k)) T = cand;
  }
  unsigned gt = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) gt += key[i] > T;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need_eq = k - int(gt);
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int jj = 32 * i + lane;
    const bool in = jj < L;
    const bool is_gt = in && key[i] > T;
    const bool is_eq = in && key[i] == T;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const bool take = is_gt || (is_eq && eq_seen + __popc(eq_mask & lt_mask) < need_eq);
    const unsigned take_mask = __ballot_sync(0xffffffffu, take);
    if (take) out[written + __popc(take_mask & lt_mask)] = OutT(map ? int(map[jj]) : jj);
    written += __popc(take_mask);
    eq_seen += __popc(eq_mask);
  }
}

template <typename OutT>
__device__ void topk_dispatch(const uint32_t* row, int L, int k, OutT* out, const int16_t* map) {
  if (L <= 32 * 16) warp_topk_reg<16>(row, L, k, out, map);
  else if (L <= 32 * 32) warp_topk_reg<32>(row, L, k, out, map);
  else warp_topk(row, L, k, out, map);
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
    // slab sl lives in buffer sl % 3; two slabs are in flight while one is used (an
    // empty commit group keeps the group count uniform at the tail)
    auto issue = [&](int sl) {
      if (sl < NSL) {
        const uint32_t b = slab_u + uint32_t((sl % kSelSlabBufs) * kSelSlabBuf) * 4u;
#pragma unroll
        for (int i = 0; i < 4; ++i) cp16(b + dst[i], src[i] + sl * kSelSlab, nbytes[i]);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    uint64_t acc[R][2];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = 0ull;
    issue(0);
    issue(1);
#pragma unroll 1
    for (int sl = 0; sl < NSL; ++sl) {
      issue(sl + 2);
      asm volatile("cp.async.wait_group 2;" ::: "memory");
      __syncwarp();
      const float* buf = slab + (sl % kSelSlabBufs) * kSelSlabBuf;
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
      __syncwarp();  // this buffer is refilled by the issue of the next iteration
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
__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(const SelParams p) {
  extern __shared__ __align__(16) uint8_t sel_smem[];
  const bool grouped = p.group > 1 || p.cand < p.nB;
  const SelSmem L = select_smem(D, p.nB, grouped);
  float* qsum = reinterpret_cast<float*>(sel_smem + L.qsum_off);    // [QB][D] row sums
  float* qmean = reinterpret_cast<float*>(sel_smem + L.qmean_off);  // [QB][D] pooled queries
  float* proxy = reinterpret_cast<float*>(sel_smem + L.proxy_off);  // [groups][D] proxy queries
  uint32_t* keys = reinterpret_cast<uint32_t*>(sel_smem + L.key_off);
  int16_t* cand = reinterpret_cast<int16_t*>(sel_smem + L.cand_off);
  const int cand_ld = (p.nB + 7) / 8 * 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* slab = reinterpret_cast<float*>(sel_smem + L.slab_off) + warp * kSelSlabBufs * kSelSlabBuf;
  const int G = p.QB / p.group;  // proxies per tile
  {
    const int T = blockIdx.x;
    const int bh = T / p.tiles_per_head;
    const int i0 = (T % p.tiles_per_head) * p.QB;
    const int nq = min(p.QB, p.nB - i0);

    // ---- 1. pool: warp r sums query block i0 + r ----
    if (warp < nq) {
      constexpr int CH = D / 8;         // 16-byte chunks per row
      constexpr int RSTEP = 32 / CH;    // rows between a lane's rows
      const int c16 = lane % CH, r0 = lane / CH;
      const int i = i0 + warp;
      const int n = min(p.block, p.N - i * p.block);
      const bf16* src = p.Q + (size_t(bh) * p.N + size_t(i) * p.block) * D + c16 * 8;
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      for (int rb = r0; rb < n; rb += kSelPoolBatch * RSTEP) {
        uint4 w[kSelPoolBatch];
#pragma unroll
        for (int b = 0; b < kSelPoolBatch; ++b) {
          const int r = rb + b * RSTEP;
          w[b] = r < n ? ldg_stream_v4(src + size_t(r) * D) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int b = 0; b < kSelPoolBatch; ++b) {
          sel::add2(acc[0], sel::pack2(w[b].x << 16, w[b].x & 0xffff0000u));
          sel::add2(acc[1], sel::pack2(w[b].y << 16, w[b].y & 0xffff0000u));
          sel::add2(acc[2], sel::pack2(w[b].z << 16, w[b].z & 0xffff0000u));
          sel::add2(acc[3], sel::pack2(w[b].w << 16, w[b].w & 0xffff0000u));
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
    } else if (warp < p.QB) {
      for (int c = lane; c < D; c += 32) qsum[warp * D + c] = 0.f;  // a tile tail without rows
    }
    __syncthreads();
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
      if (warp < nq) sel::topk_dispatch(keys + warp * p.ld, p.nB, p.topk, idx_tile + size_t(warp) * p.topk, nullptr);
      return;
    }
    // ---- 4. grouped: proxies keep `cand` candidates, members keep topk of those ----
    const int ng = (nq + p.group - 1) / p.group;  // groups present in this tile
    sel::score_dispatch<D>(ng, proxy, kb_head, route_head, p.lambda, nullptr, p.nB, keys, p.ld, slab);
    __syncthreads();
    if (warp < ng) sel::topk_dispatch(keys + warp * p.ld, p.nB, p.cand, cand + warp * cand_ld, nullptr);
    __syncthreads();
    if (p.cand == p.topk) {  // reuse: every member takes its group's list
      for (int e = threadIdx.x; e < nq * p.topk; e += kSelThreads)
        idx_tile[e] = cand[(e / p.topk / p.group) * cand_ld + e % p.topk];
      return;
    }
    for (int m = 0; m < ng; ++m) {
      const int rows = min(p.group, nq - m * p.group);
      sel::score_dispatch<D>(rows, qmean + m * p.group * D, kb_head, route_head, p.lambda, cand + m * cand_ld, p.cand,
                             keys + m * p.group * p.ld, p.ld, slab);
    }
    __syncthreads();
    if (warp < nq)
      sel::topk_dispatch(keys + warp * p.ld, p.cand, p.topk, idx_tile + size_t(warp) * p.topk,
                         cand + (warp / p.group) * cand_ld);
  }
}

}  // namespace pisa
