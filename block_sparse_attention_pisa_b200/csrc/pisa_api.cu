// C ABI of the PISA kernels: argument validation, device checks and launches.
// The entry points and their contracts are declared in include/pisa.h.
#include <cstdarg>
#include <cstdio>
#include <cmath>
#include <mutex>
#include <string>

#include <cudaTypedefs.h>

#include "../../include/pisa.h"
#include "common.cuh"
#include "stats.cuh"
#include "select.cuh"
#include "select_pipe.cuh"
#include "routing.cuh"
#include "attention_simt.cuh"
#include "attention_tc.cuh"
#include "stats_tc.cuh"
#include "host_pipeline.cuh"

using pisa::bf16;

namespace {

thread_local std::string g_last_error;

pisa_status_t fail(pisa_status_t s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

pisa_status_t ok() { return PISA_OK; }

#define PISA_TRY(expr)                        \
  do {                                        \
    pisa_status_t _s = (expr);                \
    if (_s != PISA_OK) return _s;             \
  } while (0)

inline int64_t num_blocks(const pisa_shape_t& s) { return (int64_t(s.N) + s.block - 1) / s.block; }

// Shape sanity. Sets *empty for B*H*N == 0 (nothing to do, nothing touched).
pisa_status_t check_shape(const pisa_shape_t& s, bool* empty) {
  *empty = false;
  if (s.B < 0 || s.H < 0 || s.N < 0)
    return fail(PISA_ERR_INVALID_ARG, "negative shape (B=%d H=%d N=%d)", s.B, s.H, s.N);
  if (s.d <= 0 || s.block <= 0)
    return fail(PISA_ERR_INVALID_ARG, "d and block must be positive (d=%d block=%d)", s.d, s.block);
  if (int64_t(s.B) * s.H * s.N == 0) {
    *empty = true;
    return ok();
  }
  return ok();
}

pisa_status_t check_support(const pisa_shape_t& s) {
  if (s.d != 64 && s.d != 128) return fail(PISA_ERR_UNSUPPORTED, "head dimension d=%d (supported: 64, 128)", s.d);
  if (s.block != 64 && s.block != 128)
    return fail(PISA_ERR_UNSUPPORTED, "block=%d (supported: 64, 128)", s.block);
  if (num_blocks(s) > PISA_MAX_BLOCKS)
    return fail(PISA_ERR_UNSUPPORTED, "nB=%lld exceeds PISA_MAX_BLOCKS=%d", (long long)num_blocks(s),
                PISA_MAX_BLOCKS);
  if (int64_t(s.B) * s.H > 65535)
    return fail(PISA_ERR_UNSUPPORTED, "B*H=%lld exceeds 65535", (long long)(int64_t(s.B) * s.H));
  return ok();
}

pisa_status_t check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(PISA_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) & 15u) return fail(PISA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return ok();
}

pisa_status_t check_order(int32_t order) {
  if (order < PISA_ORDER_DROP || order > PISA_ORDER_HYBRID)
    return fail(PISA_ERR_INVALID_ARG, "order=%d (must be -1, 0, 1 or 2)", order);
  return ok();
}

pisa_status_t check_topk(const pisa_shape_t& s, int32_t topk) {
  if (topk < 1 || topk > num_blocks(s))
    return fail(PISA_ERR_INVALID_ARG, "topk=%d outside [1, nB=%lld]", topk, (long long)num_blocks(s));
  return ok();
}

// Compute capability 10.0 (B200 / GB200) on the current device; cached per device.
pisa_status_t check_device(int* sm_count) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PISA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  static std::mutex mu;
  static int cached_ok[64] = {0};
  static int cached_sms[64] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && cached_ok[dev]) {
    *sm_count = cached_sms[dev];
    return ok();
  }
  int major = 0, minor = 0, sms = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return fail(PISA_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
  if (major != 10 || minor != 0)
    return fail(PISA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                minor);
  if (dev >= 0 && dev < 64) {
    cached_ok[dev] = 1;
    cached_sms[dev] = sms;
  }
  *sm_count = sms;
  return ok();
}

pisa_status_t check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PISA_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
  return ok();
}

template <typename Kernel>
pisa_status_t set_smem(Kernel k, size_t bytes) {
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  if (e != cudaSuccess) return fail(PISA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  return ok();
}

template <int D, int BLK, int MODE>
pisa_status_t launch_stats_mode(const pisa_shape_t& s, const bf16* K, const bf16* V, float* kbar, float* S0,
                                bf16* S1, float* Hbar, cudaStream_t st) {
  using P = pisa::StatsPipeCfg<D, BLK>;
  auto k = pisa::stats_pipe_kernel<D, BLK, MODE>;
  PISA_TRY(set_smem(k, P::kSmem));
  const int nB = int(num_blocks(s));
  const int G = P::blocks_per_cta(MODE);
  dim3 grid((nB + G - 1) / G, s.B * s.H);
  k<<<grid, pisa::StatsCfg<D, BLK>::kThreads, P::kSmem, st>>>(K, V, s.N, nB, kbar, S0, S1, Hbar);
  return check_launch("stats_pipe_kernel");
}

pisa_status_t make_map(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1);
pisa_status_t make_plane_map(CUtensorMap* m, const float* kbar, uint64_t D, uint64_t nB, uint64_t BH, uint32_t rows);

// d = 128, order 1: the tensor-core statistics kernel (persistent, one CTA per SM)
template <int BLK>
pisa_status_t launch_stats_tc(const pisa_shape_t& s, const bf16* K, const bf16* V, float* kbar, float* S0, bf16* S1,
                              int sms, cudaStream_t st) {
  using C = pisa::StatsTcCfg<BLK>;
  const int nB = int(num_blocks(s));
  const uint64_t BH = uint64_t(s.B) * s.H;
  CUtensorMap mK, mV, mS;
  PISA_TRY(make_map(&mK, K, 128, uint64_t(s.N), BH, BLK));
  PISA_TRY(make_map(&mV, V, 128, uint64_t(s.N), BH, BLK));
  PISA_TRY(make_map(&mS, S1, 128, 128, BH * nB, 128));
  auto k = pisa::stats_tc_kernel<BLK>;
  PISA_TRY(set_smem(k, C::SMEM));
  const int64_t total = int64_t(BH) * nB;
  if (total > (int64_t(1) << 30)) return fail(PISA_ERR_UNSUPPORTED, "too many statistics blocks");
  const int grid = int(total < sms ? total : sms);
  k<<<grid, C::kThreads, C::SMEM, st>>>(mK, mV, mS, s.N, nB, int(total), kbar, S0);
  return check_launch("stats_tc_kernel");
}

// Hbar: one cluster of kHbarCluster CTAs per head, grid (kHbarCluster, B*H)
template <typename Kernel, typename... Args>
pisa_status_t launch_hbar_clusters(Kernel k, const pisa_shape_t& s, int threads, size_t smem, cudaStream_t st,
                                   const char* what, Args... args) {
  PISA_TRY(set_smem(k, smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pisa::kHbarCluster, unsigned(s.B) * unsigned(s.H), 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pisa::kHbarCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k, args...);
  if (e != cudaSuccess) return fail(PISA_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
  return check_launch(what);
}

template <int D, int BLK>
pisa_status_t launch_stats(const pisa_shape_t& s, const bf16* K, const bf16* V, int order, float* kbar,
                           float* S0, void* S1, int sms, cudaStream_t st) {
  if (order == PISA_ORDER_HYBRID) {
    // every element of Hbar is stored once (no zeroing, no atomics)
    float* Hbar = static_cast<float*>(S1);
    const int nB = int(num_blocks(s));
    if constexpr (D == 128) {
      using C = pisa::StatsHbarCfg<BLK>;
      const uint64_t BH = uint64_t(s.B) * s.H;
      CUtensorMap mK, mV;
      PISA_TRY(make_map(&mK, K, 128, uint64_t(s.N), BH, BLK));
      PISA_TRY(make_map(&mV, V, 128, uint64_t(s.N), BH, BLK));
      return launch_hbar_clusters(pisa::stats_hbar_kernel<BLK>, s, C::kThreads, size_t(C::SMEM), st,
                                  "stats_hbar_kernel", mK, mV, s.N, nB, kbar, S0, Hbar);
    } else {
      using P = pisa::StatsPipeCfg<D, BLK>;
      return launch_hbar_clusters(pisa::stats_pipe_kernel<D, BLK, pisa::kStatsHbar>, s,
                                  pisa::StatsCfg<D, BLK>::kThreads, P::kSmem, st, "stats_pipe_kernel", K, V, s.N,
                                  nB, kbar, S0, static_cast<bf16*>(nullptr), Hbar);
    }
  }
  if (order == PISA_ORDER_FIRST) {
    if (D == 128) return launch_stats_tc<BLK>(s, K, V, kbar, S0, static_cast<bf16*>(S1), sms, st);
    return launch_stats_mode<D, BLK, pisa::kStatsS1>(s, K, V, kbar, S0, static_cast<bf16*>(S1), nullptr, st);
  }
  return launch_stats_mode<D, BLK, pisa::kStatsSums>(s, K, V, kbar, S0, nullptr, nullptr, st);
}

// plain selection, nB <= 640: the persistent pipelined kernel (KL key blocks per lane)
template <int D, int KL>
pisa_status_t launch_select_pipe(const pisa_shape_t& s, const float* kbar, pisa::SpParams& p, int sms,
                                 cudaStream_t st) {
  const uint64_t BH = uint64_t(s.B) * s.H;
  CUtensorMap m;
  PISA_TRY(make_plane_map(&m, kbar, D, uint64_t(p.nB), BH, uint32_t(p.box_rows)));
  auto k = pisa::select_pipe_kernel<D, KL>;
  PISA_TRY(set_smem(k, size_t(p.smem)));
  const int grid = p.tiles < sms ? p.tiles : sms;
  k<<<grid, pisa::kSpThreads, p.smem, st>>>(m, p);
  return check_launch("select_pipe_kernel");
}

template <int D>
pisa_status_t try_select_pipe(const pisa_shape_t& s, const bf16* Q, const float* kbar, const float* route,
                              float lambda, int topk, int32_t* idx, int sms, cudaStream_t st, bool& done) {
  done = false;
  const int nB = int(num_blocks(s));
  const int need = (nB + 63) / 64;
  const int KL = need <= 2 ? need : (need <= 4 ? 4 : (need <= 6 ? 6 : (need <= 8 ? 8 : 10)));
  if (need > pisa::kSpMaxKL) return ok();
  pisa::SpParams p{};
  if (!pisa::select_pipe_plan<D>(nB, s.block, KL, p)) return ok();
  const int64_t tiles = int64_t(s.B) * s.H * ((nB + pisa::kSpRows - 1) / pisa::kSpRows);
  if (tiles > (int64_t(1) << 31) - 1) return ok();
  p.Q = Q;
  p.route = route;
  p.lambda = lambda;
  p.idx = idx;
  p.N = s.N;
  p.nB = nB;
  p.block = s.block;
  p.topk = topk;
  p.tiles_per_head = (nB + pisa::kSpRows - 1) / pisa::kSpRows;
  p.tiles = int(tiles);
  done = true;
  switch (KL) {
    case 1: return launch_select_pipe<D, 1>(s, kbar, p, sms, st);
    case 2: return launch_select_pipe<D, 2>(s, kbar, p, sms, st);
    case 4: return launch_select_pipe<D, 4>(s, kbar, p, sms, st);
    case 6: return launch_select_pipe<D, 6>(s, kbar, p, sms, st);
    case 8: return launch_select_pipe<D, 8>(s, kbar, p, sms, st);
    default: return launch_select_pipe<D, 10>(s, kbar, p, sms, st);
  }
}

template <int D>
pisa_status_t launch_select(const pisa_shape_t& s, const bf16* Q, const float* kbar, const float* route,
                            float lambda, int topk, int group, int cand, int32_t* idx, int sms, cudaStream_t st) {
  auto k = pisa::select_kernel<D>;
  const int nB = int(num_blocks(s));
  if (group == 1 && cand == nB) {
    bool done = false;
    const pisa_status_t r = try_select_pipe<D>(s, Q, kbar, route, lambda, topk, idx, sms, st, done);
    if (done || r != PISA_OK) return r;
  }
  pisa::SelParams p{};
  p.Q = Q;
  p.kbar = kbar;
  p.route = route;
  p.lambda = lambda;
  p.idx = idx;
  p.N = s.N;
  p.nB = nB;
  p.block = s.block;
  p.topk = topk;
  p.group = group;
  p.cand = cand;
  p.QB = group * (pisa::kSelQB / group > 1 ? pisa::kSelQB / group : 1);
  p.tiles_per_head = (nB + p.QB - 1) / p.QB;
  const int64_t tiles = int64_t(s.B) * s.H * p.tiles_per_head;
  if (tiles > (int64_t(1) << 31) - 1)
    return fail(PISA_ERR_UNSUPPORTED, "too many select tiles (%lld)", (long long)tiles);
  p.ld = pisa::select_key_ld(nB);
  const size_t smem = size_t(pisa::select_smem(D, nB, group > 1 || cand < nB).bytes);
  if (smem > size_t(227 * 1024)) return fail(PISA_ERR_UNSUPPORTED, "select shared memory for nB=%d exceeds the limit", nB);
  PISA_TRY(set_smem(k, smem));
  (void)sms;
  k<<<unsigned(tiles), pisa::kSelThreads, smem, st>>>(p);
  return check_launch("select_kernel");
}

pisa_status_t launch_routing(const pisa_shape_t& s, const bf16* S1, float* Hbar, float* M, cudaStream_t st) {
  const int nB = int(num_blocks(s));
  const int dd = s.d * s.d;
  const unsigned BH = unsigned(s.B) * unsigned(s.H);
  // every element of Hbar and M is stored once (no zeroing, no atomics)
  pisa::routing_hbar_kernel<<<dim3(dd / pisa::kHbarSlice, BH), pisa::kHbarThreads, 0, st>>>(S1, nB, dd, Hbar);
  PISA_TRY(check_launch("routing_hbar_kernel"));
  const dim3 grid((nB + pisa::kRouteChunk - 1) / pisa::kRouteChunk, BH);
  if (s.d == 128) pisa::routing_norm_kernel<128><<<grid, pisa::kRouteThreads, 0, st>>>(S1, Hbar, nB, M);
  else pisa::routing_norm_kernel<64><<<grid, pisa::kRouteThreads, 0, st>>>(S1, Hbar, nB, M);
  return check_launch("routing_norm_kernel");
}

template <int D>
pisa_status_t launch_attention_simt(const pisa_shape_t& s, const bf16* Q, const bf16* K, const bf16* V,
                                    const float* kbar, const float* S0, const void* S1, const int32_t* idx,
                                    int topk, int order, float scale, bf16* O, cudaStream_t st) {
  auto k = pisa::attention_simt_kernel<D>;
  const size_t smem = pisa::SimtCfg<D>::smem_bytes();
  PISA_TRY(set_smem(k, smem));
  const int nB = int(num_blocks(s));
  dim3 grid(nB, s.B * s.H);
  const bf16* s1 = order == PISA_ORDER_FIRST ? static_cast<const bf16*>(S1) : nullptr;
  const float* hbar = order == PISA_ORDER_HYBRID ? static_cast<const float*>(S1) : nullptr;
  k<<<grid, s.block, smem, st>>>(Q, K, V, kbar, S0, s1, hbar, idx, s.N, nB, s.block, topk, order, scale, O);
  return check_launch("attention_simt_kernel");
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3-D bf16 tensor [d2][d1][d0] (d0 innermost), box {64, box1, 1}, 128-byte swizzle,
// out-of-range rows read as zero
pisa_status_t make_map(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1) {
  auto fn = encode_fn();
  if (!fn) return fail(PISA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PISA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return ok();
}

// kbar fp32 [BH][nB][D] as planes of kSpPlane = 8 dimensions: box = 8 dimensions x `rows`
// key blocks (32-byte rows, 32-byte swizzle); rows past nB read as zero
pisa_status_t make_plane_map(CUtensorMap* m, const float* kbar, uint64_t D, uint64_t nB, uint64_t BH, uint32_t rows) {
  auto fn = encode_fn();
  if (!fn) return fail(PISA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {D, nB, BH};
  cuuint64_t strides[2] = {D * 4, D * nB * 4};
  cuuint32_t box[3] = {uint32_t(pisa::kSpPlane), rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(kbar), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PISA_ERR_CUDA, "cuTensorMapEncodeTiled (kbar planes) failed (%d)", int(r));
  return ok();
}

template <int D, int BLK>
pisa_status_t launch_attention_tc(const pisa_shape_t& s, const bf16* Q, const bf16* K, const bf16* V,
                                  const float* kbar, const float* S0, const void* S1, const int32_t* idx, int topk,
                                  int order, float scale, bf16* O, cudaStream_t st) {
  using C = pisa::TcCfg<D, BLK>;
  const int nB = int(num_blocks(s));
  const uint64_t BH = uint64_t(s.B) * s.H;
  CUtensorMap mK, mV, mS1;
  PISA_TRY(make_map(&mK, K, D, uint64_t(s.N), BH, BLK));
  PISA_TRY(make_map(&mV, V, D, uint64_t(s.N), BH, BLK));
  if (order == PISA_ORDER_FIRST) PISA_TRY(make_map(&mS1, S1, D, D, BH * nB, D));
  else mS1 = mK;  // never read at the other orders
  auto k = pisa::attention_tc_kernel<D, BLK>;
  PISA_TRY(set_smem(k, C::SMEM));
  const float* hbar = order == PISA_ORDER_HYBRID ? static_cast<const float*>(S1) : nullptr;
  pisa::TcParams p{Q, kbar, S0, idx, hbar, O, s.N, nB, topk, order, scale};
  dim3 grid((s.N + 127) / 128, unsigned(BH));
  k<<<grid, C::kThreads, C::SMEM, st>>>(mK, mV, mS1, p);
  return check_launch("attention_tc_kernel");
}

struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  const float* kbar;
  const float* S0;
  const void* S1;
  const int32_t* idx;
  int32_t topk;
  int32_t order;
  float scale;
  void* O;
};

pisa_status_t validate_attention(const pisa_shape_t& shape, const AttnArgs& a, bool* empty) {
  PISA_TRY(check_shape(shape, empty));
  if (*empty) return ok();
  PISA_TRY(check_ptr(a.Q, "Q"));
  PISA_TRY(check_ptr(a.K, "K"));
  PISA_TRY(check_ptr(a.V, "V"));
  PISA_TRY(check_ptr(a.idx, "idx"));
  PISA_TRY(check_ptr(a.O, "O"));
  PISA_TRY(check_order(a.order));
  if (a.order != PISA_ORDER_DROP) {
    PISA_TRY(check_ptr(a.kbar, "kbar"));
    PISA_TRY(check_ptr(a.S0, "S0"));
  }
  if (a.order == PISA_ORDER_FIRST) PISA_TRY(check_ptr(a.S1, "S1"));
  if (a.order == PISA_ORDER_HYBRID) PISA_TRY(check_ptr(a.S1, "Hbar (S1)"));
  PISA_TRY(check_topk(shape, a.topk));
  if (!std::isfinite(a.scale) || !(a.scale > 0.f))
    return fail(PISA_ERR_INVALID_ARG, "scale=%g (must be finite and > 0)", double(a.scale));
  return check_support(shape);
}

}  // namespace

extern "C" {

pisa_status_t pisa_block_stats(const void* K, const void* V, pisa_shape_t shape, int32_t order, float* kbar,
                               float* S0, void* S1, void* stream) {
  bool empty = false;
  PISA_TRY(check_shape(shape, &empty));
  if (empty) return ok();
  PISA_TRY(check_ptr(K, "K"));
  PISA_TRY(check_ptr(V, "V"));
  PISA_TRY(check_ptr(kbar, "kbar"));
  PISA_TRY(check_ptr(S0, "S0"));
  PISA_TRY(check_order(order));
  if (order == PISA_ORDER_FIRST) PISA_TRY(check_ptr(S1, "S1"));
  if (order == PISA_ORDER_HYBRID) PISA_TRY(check_ptr(S1, "Hbar (S1)"));
  PISA_TRY(check_support(shape));
  int sms = 0;
  PISA_TRY(check_device(&sms));
  auto st = static_cast<cudaStream_t>(stream);
  auto k = static_cast<const bf16*>(K);
  auto v = static_cast<const bf16*>(V);
  if (shape.d == 128 && shape.block == 64) return launch_stats<128, 64>(shape, k, v, order, kbar, S0, S1, sms, st);
  if (shape.d == 128 && shape.block == 128) return launch_stats<128, 128>(shape, k, v, order, kbar, S0, S1, sms, st);
  if (shape.d == 64 && shape.block == 64) return launch_stats<64, 64>(shape, k, v, order, kbar, S0, S1, sms, st);
  return launch_stats<64, 128>(shape, k, v, order, kbar, S0, S1, sms, st);
}

pisa_status_t pisa_select_grouped(const void* Q, const float* kbar, const float* route, float lambda,
                                  pisa_shape_t shape, int32_t topk, int32_t group, int32_t candidates, int32_t* idx,
                                  void* stream) {
  bool empty = false;
  PISA_TRY(check_shape(shape, &empty));
  if (empty) return ok();
  PISA_TRY(check_ptr(Q, "Q"));
  PISA_TRY(check_ptr(kbar, "kbar"));
  PISA_TRY(check_ptr(idx, "idx"));
  if (route != nullptr) {
    PISA_TRY(check_ptr(route, "route"));
    if (!std::isfinite(lambda) || lambda < 0.f)
      return fail(PISA_ERR_INVALID_ARG, "lambda=%g (must be finite and >= 0)", double(lambda));
  }
  PISA_TRY(check_topk(shape, topk));
  if (group < 1 || group > pisa::kSelMaxGroup)
    return fail(PISA_ERR_INVALID_ARG, "group=%d outside [1, %d]", group, pisa::kSelMaxGroup);
  if (candidates < topk || candidates > num_blocks(shape))
    return fail(PISA_ERR_INVALID_ARG, "candidates=%d outside [topk=%d, nB=%lld]", candidates, topk,
                (long long)num_blocks(shape));
  PISA_TRY(check_support(shape));
  int sms = 0;
  PISA_TRY(check_device(&sms));
  auto st = static_cast<cudaStream_t>(stream);
  auto q = static_cast<const bf16*>(Q);
  if (shape.d == 128) return launch_select<128>(shape, q, kbar, route, lambda, topk, group, candidates, idx, sms, st);
  return launch_select<64>(shape, q, kbar, route, lambda, topk, group, candidates, idx, sms, st);
}

pisa_status_t pisa_select(const void* Q, const float* kbar, const float* route, float lambda, pisa_shape_t shape,
                          int32_t topk, int32_t* idx, void* stream) {
  bool empty = false;
  PISA_TRY(check_shape(shape, &empty));
  if (empty) return ok();
  // plain selection: every query block is its own proxy and every key block a candidate
  return pisa_select_grouped(Q, kbar, route, lambda, shape, topk, 1, int32_t(num_blocks(shape)), idx, stream);
}

pisa_status_t pisa_routing_norms(const void* S1, pisa_shape_t shape, float* Hbar, float* M, void* stream) {
  bool empty = false;
  PISA_TRY(check_shape(shape, &empty));
  if (empty) return ok();
  PISA_TRY(check_ptr(S1, "S1"));
  PISA_TRY(check_ptr(Hbar, "Hbar"));
  PISA_TRY(check_ptr(M, "M"));
  PISA_TRY(check_support(shape));
  int sms = 0;
  PISA_TRY(check_device(&sms));
  return launch_routing(shape, static_cast<const bf16*>(S1), Hbar, M, static_cast<cudaStream_t>(stream));
}

pisa_status_t pisa_attention(const void* Q, const void* K, const void* V, const float* kbar, const float* S0,
                             const void* S1, const int32_t* idx, pisa_shape_t shape, int32_t topk, int32_t order,
                             float scale, void* O, void* stream) {
  AttnArgs a{Q, K, V, kbar, S0, S1, idx, topk, order, scale, O};
  bool empty = false;
  PISA_TRY(validate_attention(shape, a, &empty));
  if (empty) return ok();
  int sms = 0;
  PISA_TRY(check_device(&sms));
  auto st = static_cast<cudaStream_t>(stream);
  auto q = static_cast<const bf16*>(Q);
  auto k = static_cast<const bf16*>(K);
  auto v = static_cast<const bf16*>(V);
  const void* s1 = S1;
  auto o = static_cast<bf16*>(O);
  if (shape.d == 128 && shape.block == 64)
    return launch_attention_tc<128, 64>(shape, q, k, v, kbar, S0, s1, idx, topk, order, scale, o, st);
  if (shape.d == 128 && shape.block == 128)
    return launch_attention_tc<128, 128>(shape, q, k, v, kbar, S0, s1, idx, topk, order, scale, o, st);
  if (shape.d == 64 && shape.block == 64)
    return launch_attention_tc<64, 64>(shape, q, k, v, kbar, S0, s1, idx, topk, order, scale, o, st);
  return launch_attention_tc<64, 128>(shape, q, k, v, kbar, S0, s1, idx, topk, order, scale, o, st);
}

pisa_status_t pisa_attention_simt(const void* Q, const void* K, const void* V, const float* kbar,
                                  const float* S0, const void* S1, const int32_t* idx, pisa_shape_t shape,
                                  int32_t topk, int32_t order, float scale, void* O, void* stream) {
  AttnArgs a{Q, K, V, kbar, S0, S1, idx, topk, order, scale, O};
  bool empty = false;
  PISA_TRY(validate_attention(shape, a, &empty));
  if (empty) return ok();
  int sms = 0;
  PISA_TRY(check_device(&sms));
  auto st = static_cast<cudaStream_t>(stream);
  auto q = static_cast<const bf16*>(Q);
  auto k = static_cast<const bf16*>(K);
  auto v = static_cast<const bf16*>(V);
  const void* s1 = S1;
  auto o = static_cast<bf16*>(O);
  if (shape.d == 128) return launch_attention_simt<128>(shape, q, k, v, kbar, S0, s1, idx, topk, order, scale, o, st);
  return launch_attention_simt<64>(shape, q, k, v, kbar, S0, s1, idx, topk, order, scale, o, st);
}

}  // extern "C"

namespace {

// options with their defaults filled in, checked against the problem
pisa_status_t host_options(const pisa_shape_t& s, int32_t topk, const pisa_host_options_t* in,
                           pisa_host_options_t* out) {
  pisa_host_options_t o{0.f, 1, 0, 8};
  if (in != nullptr) o = *in;
  if (o.group == 0) o.group = 1;
  if (o.chunks == 0) o.chunks = 32;  // at most B*H ranges are used
  const int32_t nB = int32_t(num_blocks(s));
  if (o.candidates == 0) o.candidates = nB;
  if (!std::isfinite(o.route_lambda) || o.route_lambda < 0.f)
    return fail(PISA_ERR_INVALID_ARG, "route_lambda=%g (must be finite and >= 0)", double(o.route_lambda));
  if (o.chunks < 1) return fail(PISA_ERR_INVALID_ARG, "chunks=%d (must be >= 1)", o.chunks);
  if (o.group < 1 || o.group > pisa::kSelMaxGroup)
    return fail(PISA_ERR_INVALID_ARG, "group=%d outside [1, %d]", o.group, pisa::kSelMaxGroup);
  if (o.candidates < topk || o.candidates > nB)
    return fail(PISA_ERR_INVALID_ARG, "candidates=%d outside [topk=%d, nB=%d]", o.candidates, topk, nB);
  *out = o;
  return ok();
}

}  // namespace

// The device workspace of pisa_run_host_static: one region per device, part of the
// library's module (no allocation at call time); its address is looked up once per device.
static __device__ __align__(256) unsigned char g_static_workspace[PISA_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};

pisa_status_t static_workspace(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PISA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(PISA_ERR_UNSUPPORTED, "device %d (at most %d)", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);  // the current device's copy
    if (e != cudaSuccess)
      return fail(PISA_ERR_CUDA, "cudaGetSymbolAddress(static workspace): %s", cudaGetErrorString(e));
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return ok();
}

}  // namespace

extern "C" {

pisa_status_t pisa_run_host_workspace(pisa_shape_t shape, int32_t topk, int32_t order,
                                      const pisa_host_options_t* options, size_t* bytes) {
  if (bytes == nullptr) return fail(PISA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = 0;
  bool empty = false;
  PISA_TRY(check_shape(shape, &empty));
  if (empty) return ok();
  PISA_TRY(check_order(order));
  PISA_TRY(check_topk(shape, topk));
  pisa_host_options_t o;
  PISA_TRY(host_options(shape, topk, options, &o));
  PISA_TRY(check_support(shape));
  *bytes = pisa_host::workspace_bytes(shape, topk, order, o.route_lambda > 0.f, o.chunks);
  return ok();
}

pisa_status_t pisa_run_host(const void* Q, const void* K, const void* V, pisa_shape_t shape, int32_t topk,
                            int32_t order, float scale, const pisa_host_options_t* options, void* workspace,
                            size_t workspace_bytes, void* O, void* stream) {
  size_t need = 0;
  PISA_TRY(pisa_run_host_workspace(shape, topk, order, options, &need));
  if (need == 0) return ok();  // empty problem: nothing touched
  pisa_host_options_t opt;
  PISA_TRY(host_options(shape, topk, options, &opt));
  const float route_lambda = opt.route_lambda;
  const int32_t chunks = opt.chunks;
  const void* host[4] = {Q, K, V, O};
  const char* names[4] = {"Q", "K", "V", "O"};
  for (int i = 0; i < 4; ++i)
    if (host[i] == nullptr) return fail(PISA_ERR_INVALID_ARG, "%s is NULL", names[i]);
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(PISA_ERR_INVALID_ARG, "scale=%g (must be finite and > 0)", double(scale));
  if (workspace == nullptr) return fail(PISA_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(workspace) % pisa_host::kAlign)
    return fail(PISA_ERR_INVALID_ARG, "workspace is not %zu-byte aligned", pisa_host::kAlign);
  if (workspace_bytes < need)
    return fail(PISA_ERR_INVALID_ARG, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
  int sms = 0;
  PISA_TRY(check_device(&sms));
  for (int i = 0; i < 4; ++i) {
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, host[i]) == cudaSuccess && at.type == cudaMemoryTypeDevice)
      return fail(PISA_ERR_INVALID_ARG, "%s is device memory; pisa_run_host takes host buffers", names[i]);
    cudaGetLastError();  // an unregistered host pointer may leave an error behind
  }

  const int64_t BH = int64_t(shape.B) * shape.H;
  const int nc = int(chunks < BH ? chunks : BH);
  const int slots = nc < pisa_host::kSlots ? nc : pisa_host::kSlots;
  const int64_t nB = num_blocks(shape);
  const bool routed = route_lambda > 0.f;
  const pisa_host::SlotLayout L =
      pisa_host::slot_layout(pisa_host::range_size(BH, nc), shape.N, shape.d, nB, topk, order, routed);
  const size_t row_bytes = size_t(shape.N) * shape.d * 2;  // one (batch, head) slice of Q, K, V or O
  auto cs = static_cast<cudaStream_t>(stream);
  // the ranges' kernels alternate between the caller's stream and one more, so that a
  // range's first CTAs fill the SMs the previous range's last wave leaves idle
  cudaStream_t in_s = nullptr, out_s = nullptr, cs2 = nullptr;
  std::vector<cudaEvent_t> ev;  // entry, then landed / computed / drained per range
  pisa_status_t st = PISA_OK;
  cudaError_t e = cudaSuccess;
  auto cuda_fail = [&](const char* what) { return fail(PISA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e)); };
  auto event = [&](cudaEvent_t* out) {
    e = cudaEventCreateWithFlags(out, cudaEventDisableTiming);
    if (e == cudaSuccess) ev.push_back(*out);
    return e == cudaSuccess;
  };
  cudaEvent_t entry = nullptr;
  std::vector<cudaEvent_t> landed(nc), computed(nc), drained(nc);
  do {
    if ((e = cudaStreamCreateWithFlags(&in_s, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&out_s, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&cs2, cudaStreamNonBlocking)) != cudaSuccess) {
      st = cuda_fail("cudaStreamCreateWithFlags");
      break;
    }
    // the copy streams start after whatever the caller's stream already holds (earlier
    // users of the workspace)
    if (!event(&entry) || (e = cudaEventRecord(entry, cs)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(in_s, entry, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(out_s, entry, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(cs2, entry, 0)) != cudaSuccess) {
      st = cuda_fail("entry event");
      break;
    }
    for (int c = 0; c < nc && st == PISA_OK; ++c) {
      const int64_t a = BH * c / nc, b = BH * (c + 1) / nc, n = b - a;
      cudaStream_t ks = (c & 1) ? cs2 : cs;  // this range's kernels
      uint8_t* base = static_cast<uint8_t*>(workspace) + size_t(c % slots) * L.bytes;
      if (!event(&landed[c]) || !event(&computed[c]) || !event(&drained[c])) {
        st = cuda_fail("cudaEventCreate");
        break;
      }
      // copy in, once the slot's previous range has been copied out
      if (c >= slots && (e = cudaStreamWaitEvent(in_s, drained[c - slots], 0)) != cudaSuccess) {
        st = cuda_fail("cudaStreamWaitEvent");
        break;
      }
      const size_t off = size_t(a) * row_bytes, len = size_t(n) * row_bytes;
      const size_t dst[3] = {L.q, L.k, L.v};
      for (int t = 0; t < 3 && e == cudaSuccess; ++t)
        e = cudaMemcpyAsync(base + dst[t], static_cast<const uint8_t*>(host[t]) + off, len, cudaMemcpyHostToDevice,
                            in_s);
      if (e != cudaSuccess || (e = cudaEventRecord(landed[c], in_s)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(ks, landed[c], 0)) != cudaSuccess) {
        st = cuda_fail("copy-in");
        break;
      }
      // the path on this range's kernel stream, as a [1, n, N, d] problem
      pisa_shape_t rs{1, int32_t(n), shape.N, shape.d, shape.block};
      float* kbar = reinterpret_cast<float*>(base + L.kbar);
      float* S0 = reinterpret_cast<float*>(base + L.s0);
      void* S1 = base + L.s1;
      int32_t* idx = reinterpret_cast<int32_t*>(base + L.idx);
      const int stats_order = routed ? PISA_ORDER_FIRST : order;
      const void* first = order == PISA_ORDER_FIRST || order == PISA_ORDER_HYBRID ? S1 : nullptr;
      const float* route = nullptr;
      if ((st = pisa_block_stats(base + L.k, base + L.v, rs, stats_order, kbar, S0,
                                 stats_order >= PISA_ORDER_FIRST ? S1 : nullptr, ks)) != PISA_OK)
        break;
      if (routed) {
        float* hbar = reinterpret_cast<float*>(base + L.hbar);
        float* M = reinterpret_cast<float*>(base + L.m);
        if ((st = pisa_routing_norms(S1, rs, hbar, M, ks)) != PISA_OK) break;
        route = M;
        if (order == PISA_ORDER_HYBRID) first = hbar;
      }
      if ((st = pisa_select_grouped(base + L.q, kbar, route, route_lambda, rs, topk, opt.group, opt.candidates, idx,
                                    ks)) != PISA_OK)
        break;
      if ((st = pisa_attention(base + L.q, base + L.k, base + L.v, kbar, S0, first, idx, rs, topk, order, scale,
                               base + L.o, ks)) != PISA_OK)
        break;
      // copy out, once the range's kernels are done
      if ((e = cudaEventRecord(computed[c], ks)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(out_s, computed[c], 0)) != cudaSuccess ||
          (e = cudaMemcpyAsync(static_cast<uint8_t*>(O) + off, base + L.o, len, cudaMemcpyDeviceToHost, out_s)) !=
              cudaSuccess ||
          (e = cudaEventRecord(drained[c], out_s)) != cudaSuccess) {
        st = cuda_fail("copy-out");
        break;
      }
    }
  } while (false);
  // whatever happened, nothing may still run on the workspace or the host buffers when
  // the call returns
  for (int i = 0; i < 4; ++i) {
    cudaStream_t s = i == 0 ? in_s : (i == 1 ? out_s : (i == 2 ? cs2 : cs));
    if (i < 3 && s == nullptr) continue;  // an internal stream that was never created
    cudaError_t se = cudaStreamSynchronize(s);
    if (se != cudaSuccess && st == PISA_OK) {
      e = se;
      st = cuda_fail("cudaStreamSynchronize");
    }
  }
  for (cudaEvent_t x : ev) cudaEventDestroy(x);
  if (in_s) cudaStreamDestroy(in_s);
  if (out_s) cudaStreamDestroy(out_s);
  if (cs2) cudaStreamDestroy(cs2);
  return st;
}

pisa_status_t pisa_run_host_static(const void* Q, const void* K, const void* V, pisa_shape_t shape, int32_t topk,
                                   int32_t order, float scale, const pisa_host_options_t* options, void* O,
                                   void* stream) {
  size_t need = 0;
  PISA_TRY(pisa_run_host_workspace(shape, topk, order, options, &need));
  if (need == 0) return ok();  // empty problem: nothing touched
  if (need > size_t(PISA_STATIC_WORKSPACE_BYTES))
    return fail(PISA_ERR_UNSUPPORTED,
                "the problem needs %zu bytes of workspace, the static region holds %zu (more chunks make the ranges "
                "smaller)",
                need, size_t(PISA_STATIC_WORKSPACE_BYTES));
  // argument errors before the first device call
  const void* host[4] = {Q, K, V, O};
  const char* names[4] = {"Q", "K", "V", "O"};
  for (int i = 0; i < 4; ++i)
    if (host[i] == nullptr) return fail(PISA_ERR_INVALID_ARG, "%s is NULL", names[i]);
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(PISA_ERR_INVALID_ARG, "scale=%g (must be finite and > 0)", double(scale));
  void* ws = nullptr;
  PISA_TRY(static_workspace(&ws));
  return pisa_run_host(Q, K, V, shape, topk, order, scale, options, ws, size_t(PISA_STATIC_WORKSPACE_BYTES), O,
                       stream);
}

pisa_status_t pisa_device_error(void* stream) {
  auto st = static_cast<cudaStream_t>(stream);
  // one caller at a time: the exchanged word passes through one device variable
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  pisa::take_error_kernel<<<1, 1, 0, st>>>();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PISA_ERR_CUDA, "take_error_kernel launch: %s", cudaGetErrorString(e));
  unsigned word = 0;
  if ((e = cudaMemcpyFromSymbolAsync(&word, pisa::g_pisa_error_taken, sizeof(word), 0, cudaMemcpyDeviceToHost, st)) !=
          cudaSuccess ||
      (e = cudaStreamSynchronize(st)) != cudaSuccess)
    return fail(PISA_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
  if (word & pisa::kErrTimeout) return fail(PISA_ERR_TIMEOUT, "a bounded device wait ran out (word=0x%x)", word);
  if (word & pisa::kErrBadIndex) return fail(PISA_ERR_INVALID_ARG, "idx held an out-of-range block (word=0x%x)", word);
  return ok();
}

const char* pisa_status_string(pisa_status_t status) {
  switch (status) {
    case PISA_OK: return "PISA_OK";
    case PISA_ERR_INVALID_ARG: return "PISA_ERR_INVALID_ARG: invalid argument";
    case PISA_ERR_UNSUPPORTED: return "PISA_ERR_UNSUPPORTED: shape or device not supported";
    case PISA_ERR_CUDA: return "PISA_ERR_CUDA: CUDA call failed";
    case PISA_ERR_TIMEOUT: return "PISA_ERR_TIMEOUT: bounded device wait ran out";
  }
  return "unknown pisa_status_t";
}

const char* pisa_last_error(void) { return g_last_error.c_str(); }

int32_t pisa_version(void) { return 200; }  // 0.2.0: orders -1 and 2, covariance-aware routing

}  // extern "C"
