/*
 * pisa.h -- C ABI of the PISA piecewise-sparse-attention kernels (NVIDIA B200, sm_100a).
 *
 * Method: "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
 * Transformers" (Li, Shao, Zhong, Zhou, Bai, Xiong, Xie, 2026; explainer of arXiv
 * 2602.01077 on gist.science), technical summary section 2 (Methodology). Each query
 * block attends exactly to its top-k critical key blocks; every other key block is
 * replaced by a block-level Taylor expansion of exp(x.k) around the block's mean key,
 * and both parts share one softmax numerator and denominator.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Q, K, V, O are bf16 (__nv_bfloat16), layout [B, H, N, d] row-major (d innermost,
 *    each head's N x d slice contiguous).
 *  - block = b, the key-block and query-block size. nB = ceil(N / b). Block j holds
 *    tokens [j*b, min((j+1)*b, N)); its real count n_j may be smaller for the last one.
 *    The caller never pads: N is the true sequence length.
 *  - x_t = scale * q_t is the scaled query (the softmax scale is applied to every
 *    exponent, including the Taylor term).
 *  - All pointers are DEVICE pointers owned by the caller, 16-byte aligned, on the
 *    current CUDA device. The library allocates no device memory and never frees or
 *    retains caller memory after the call returns (TMA descriptors are encoded on the
 *    host for each call and passed by value to the kernel).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call only
 *    enqueues work on it and returns; results are ready when the stream has reached them.
 *  - Supported: d in {64, 128}; block in {64, 128}; nB <= PISA_MAX_BLOCKS; compute
 *    capability 10.0 (B200/GB200) only. Anything else returns PISA_ERR_UNSUPPORTED.
 *  - Empty problems (B*H*N == 0) return PISA_OK without touching any pointer.
 *  - Argument errors are detected on the host before any launch and return
 *    PISA_ERR_INVALID_ARG with a message readable through pisa_last_error().
 *  - Launch failures return PISA_ERR_CUDA. Every wait inside the kernels is bounded;
 *    a wait that runs out (or an out-of-range entry in `idx`) sets a device error word
 *    that pisa_device_error() reports as PISA_ERR_TIMEOUT / PISA_ERR_INVALID_ARG.
 *  - The calls are thread-safe with respect to one another; pisa_last_error() is per
 *    host thread. The device error word is shared per device (see pisa_device_error).
 *
 * Orders (how the non-critical blocks U_i of a query block enter the softmax)
 * -------------------------------------------------------------------------
 *  PISA_ORDER_DROP   (-1) keep-or-drop: they are left out (block-sparse attention,
 *                         the baseline class of the explainer's section 1).
 *  PISA_ORDER_ZERO    (0) zeroth-order Taylor term alpha_{t,j} S0_j.
 *  PISA_ORDER_FIRST   (1) zeroth order plus the per-block first-order term
 *                         alpha_{t,j} S1_j^T x_t.
 *  PISA_ORDER_HYBRID  (2) section 2, "Core algorithm": zeroth order per block plus ONE
 *                         global first-order correction (x_t Hbar) sum_{j in U_i}
 *                         alpha_{t,j}, Hbar the mean over all blocks of the head of
 *                         the per-block first-order matrices.
 */
#ifndef PISA_H_
#define PISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PISA_MAX_BLOCKS 2048

#define PISA_ORDER_DROP (-1)
#define PISA_ORDER_ZERO 0
#define PISA_ORDER_FIRST 1
#define PISA_ORDER_HYBRID 2

typedef enum {
  PISA_OK = 0,
  PISA_ERR_INVALID_ARG = 1,  /* bad pointer, alignment, shape, topk, order or scale  */
  PISA_ERR_UNSUPPORTED = 2,  /* valid, but outside the compiled d / block / device set */
  PISA_ERR_CUDA = 3,         /* a CUDA runtime or driver call failed                  */
  PISA_ERR_TIMEOUT = 4       /* a bounded device-side wait ran out                    */
} pisa_status_t;

typedef struct {
  int32_t B;      /* batch                          */
  int32_t H;      /* heads                          */
  int32_t N;      /* tokens (true length, not padded) */
  int32_t d;      /* head dimension (64 or 128)     */
  int32_t block;  /* block size b (64 or 128)       */
} pisa_shape_t;

/*
 * pisa_block_stats -- per-block statistics of the keys and values.
 *
 * Follows section 2, "Hardware implementation", precompute step (block centroids
 * and value sums), and the first-order Taylor term of exp(x.k) around the centroid:
 *   kbar_j = (1/n_j) sum_{n in j} k_n                 fp32  [B, H, nB, d]
 *   S0_j   = sum_{n in j} v_n                         fp32  [B, H, nB, d]
 *   S1_j   = sum_{n in j} (k_n - kbar_j) v_n^T        bf16  [B, H, nB, d, d]
 *            (row a = key dimension, column c = value dimension; fp32 accumulation,
 *             rounded once to bf16)
 *   Hbar   = (1/nB) sum_j S1_j                        fp32  [B, H, d, d]
 * K, V: bf16 [B, H, N, d]. order (-1, 0, 1 or 2) selects what the S1 argument receives:
 *   order 1: S1 = the per-block matrices, bf16 [B, H, nB, d, d];
 *   order 2: S1 = Hbar, fp32 [B, H, d, d], every element stored once (it need not be
 *            zeroed); per-block S1 is not written. A cluster of 4 CTAs per head takes
 *            the head's blocks in 4 contiguous slices and adds the 4 partial sums in
 *            a fixed order, without atomics, so the result depends only on K, V, N,
 *            d and b: the same bits for any B, H, stream or device;
 *   order 0, -1: S1 is not touched and may be NULL.
 */
pisa_status_t pisa_block_stats(const void* K, const void* V, pisa_shape_t shape, int32_t order,
                               float* kbar, float* S0, void* S1, void* stream);

/*
 * pisa_select -- top-k critical key blocks of every query block.
 *
 * Section 2, "Covariance-aware routing": the relevance of key block j to query block
 * i is the pooled score qbar_i . kbar_j, with qbar_i the mean of query block i's real
 * rows, plus, when `route` is given, the covariance term lambda * M_j (M from
 * pisa_routing_norms); computed in fp32. idx[b,h,i,:] receives the topk blocks with
 * the largest scores, equal scores resolved toward the lower block index, written in
 * ascending block order.
 * Q: bf16 [B, H, N, d]; kbar: fp32 [B, H, nB, d] (from pisa_block_stats);
 * route: fp32 [B, H, nB] or NULL (plain relevance); lambda: finite, >= 0 (ignored
 * when route is NULL); idx: int32 [B, H, nB, topk]; 1 <= topk <= nB.
 */
pisa_status_t pisa_select(const void* Q, const float* kbar, const float* route, float lambda,
                          pisa_shape_t shape, int32_t topk, int32_t* idx, void* stream);

/*
 * pisa_select_grouped -- pisa_select with one proxy query per group of query blocks.
 *
 * PIVOT page ("PIVOT slashes sparse-attention indexer cost 4x and cuts latency 1.6x"),
 * "Two observations behind PIVOT": neighbouring queries pick nearly the same blocks, so
 * `group` consecutive query blocks [m*group, (m+1)*group) share a proxy query, the mean
 * of all their real rows. The proxy is scored against every key block (qbar . kbar_j,
 * plus lambda * M_j with `route`) and keeps its `candidates` best as a candidate list;
 * each member query block then keeps the topk candidates with its own best pooled
 * scores. candidates == topk is the reuse mode (every member takes the proxy's list);
 * group == 1 with candidates == nB is pisa_select. Ties go to the lower block index,
 * rows are written ascending. 1 <= group <= 8; topk <= candidates <= nB; other
 * arguments as pisa_select.
 */
pisa_status_t pisa_select_grouped(const void* Q, const float* kbar, const float* route, float lambda,
                                  pisa_shape_t shape, int32_t topk, int32_t group, int32_t candidates, int32_t* idx,
                                  void* stream);

/*
 * pisa_routing_norms -- the covariance-aware routing statistic.
 *
 * Section 2, "Covariance-aware routing": the selection score of a block carries the
 * norm of its first-order matrix's deviation from the global statistic,
 *   Hbar = (1/nB) sum_j S1_j                          fp32  [B, H, d, d]
 *   M_j  = || S1_j - Hbar ||_F                         fp32  [B, H, nB]
 * (the pages write a 2-norm without naming it; this is the Frobenius norm). S1 is the
 * per-block bf16 output of pisa_block_stats at order 1, read as stored, so this Hbar
 * is the mean of the stored bf16 matrices; it serves as the Hbar argument of
 * pisa_attention at order 2 as well. Hbar and M are overwritten, each element stored
 * once after sums taken in a fixed order (no atomics): the same bits on every call.
 */
pisa_status_t pisa_routing_norms(const void* S1, pisa_shape_t shape, float* Hbar, float* M,
                                 void* stream);

/*
 * pisa_attention -- fused exact + Taylor attention.
 *
 * Section 2, "Core algorithm" (o_t = N_t / D_t; the exact sparse term over the
 * critical blocks; the zeroth-order term alpha_{t,j} S0_j with alpha_{t,j} =
 * exp(x_t . kbar_j); a first-order term in the numerator) and "Hardware
 * implementation" (one FlashAttention-style online softmax over an exact stage and an
 * approximate stage). For query row t of block i with critical set S_i = idx[b,h,i,:]:
 *   N_t = sum_{j in S_i} sum_n e^{x_t.k_n} v_n
 *       + sum_{j not in S_i} e^{x_t.kbar_j} (S0_j + [order == 1] S1_j^T x_t)
 *       + [order == 2] (x_t Hbar) sum_{j not in S_i} e^{x_t.kbar_j}
 *   D_t = sum_{j in S_i} sum_n e^{x_t.k_n} + sum_{j not in S_i} n_j e^{x_t.kbar_j}
 *   O_t = N_t / D_t                                  bf16 [B, H, N, d]
 * (at order -1 both sums over j not in S_i are absent).
 * All exponents are taken relative to one running row maximum (a single online-softmax
 * accumulator). idx rows must hold topk distinct blocks in [0, nB) (the order inside a
 * row does not matter); out-of-range entries are ignored and flagged in the device
 * error word. S1 is the per-block bf16 S1 at order 1 and the fp32 Hbar at order 2 (from
 * pisa_block_stats at the same order, or the Hbar of pisa_routing_norms); it may be NULL
 * at orders 0 and -1, and kbar and S0 may be NULL at order -1. scale must be finite and
 * > 0.
 */
pisa_status_t pisa_attention(const void* Q, const void* K, const void* V, const float* kbar,
                             const float* S0, const void* S1, const int32_t* idx,
                             pisa_shape_t shape, int32_t topk, int32_t order, float scale,
                             void* O, void* stream);

/*
 * pisa_attention_simt -- the same operation as pisa_attention, computed by a plain
 * CUDA-core kernel (one thread per query row, blocks visited in ascending order, the
 * accumulator rescaled whenever the running maximum grows). Same arguments, layouts
 * and errors as pisa_attention. It exists to cross-check the fused tensor-core kernel
 * on sizes where a CPU reference is slow; it is not tuned for speed.
 */
pisa_status_t pisa_attention_simt(const void* Q, const void* K, const void* V, const float* kbar,
                                  const float* S0, const void* S1, const int32_t* idx,
                                  pisa_shape_t shape, int32_t topk, int32_t order, float scale,
                                  void* O, void* stream);

/* Options of the host-buffer entry point (NULL: all defaults). */
typedef struct {
  float route_lambda;  /* 0 (default): plain relevance; > 0: covariance-aware routing weight */
  int32_t group;       /* query blocks per proxy query for the selection (default / 0: 1)     */
  int32_t candidates;  /* proxy candidate-list length (default / 0: every key block)           */
  int32_t chunks;      /* (batch, head) ranges pipelined through the workspace (default / 0: 32) */
} pisa_host_options_t;

/*
 * pisa_run_host_workspace -- bytes of device workspace that pisa_run_host needs for
 * this problem: *bytes = 0 for an empty problem. Same argument checks as pisa_run_host
 * (no device is touched). The figure is about min(3, chunks) ranges of
 * ceil(B*H / chunks) (batch, head) pairs, each holding its Q, K, V, O and statistics.
 */
pisa_status_t pisa_run_host_workspace(pisa_shape_t shape, int32_t topk, int32_t order,
                                      const pisa_host_options_t* options, size_t* bytes);

/*
 * pisa_run_host -- the whole path on HOST buffers: pisa_block_stats, (with
 * route_lambda > 0) pisa_routing_norms, pisa_select (pisa_select_grouped with a group
 * or a candidate count) and pisa_attention, as one call.
 *
 * Section 2 of the explainer, "Hardware implementation": a precompute step, routing,
 * then the fused kernel. Every step is independent across (batch, head) pairs, so the
 * call splits the B*H pairs into `chunks` contiguous ranges and pipelines them through
 * the workspace: the host-to-device copy of a range, the kernels of the ranges before it
 * and the device-to-host copy of earlier ones overlap. The ranges' kernels alternate
 * between `stream` and one internal stream, so one range's first CTAs fill the SMs the
 * previous range's last wave leaves idle; the copies run on two more internal streams.
 * The result is bit for bit that of the device calls on the whole batch.
 * Q, K, V: HOST bf16 [B, H, N, d] (page-locked memory lets the copies overlap the
 * kernels; pageable memory works, with less overlap); O: HOST bf16 [B, H, N, d],
 * written; topk, order, scale as in pisa_attention. With route_lambda > 0, order 1
 * attends with the per-block S1 and order 2 with the routing call's Hbar.
 * workspace: DEVICE memory owned by the caller, 256-byte aligned, of at least the
 * size pisa_run_host_workspace reports for the same arguments; its contents are
 * scratch. The call BLOCKS until O holds the whole result and nothing runs on the
 * workspace or the host buffers any more. Device pointers passed as Q, K, V or O are
 * rejected with PISA_ERR_INVALID_ARG.
 */
pisa_status_t pisa_run_host(const void* Q, const void* K, const void* V, pisa_shape_t shape, int32_t topk,
                            int32_t order, float scale, const pisa_host_options_t* options, void* workspace,
                            size_t workspace_bytes, void* O, void* stream);

/* Size of the library's own device workspace region used by pisa_run_host_static. */
#define PISA_STATIC_WORKSPACE_BYTES (32u << 20)

/*
 * pisa_run_host_static -- pisa_run_host with no workspace from the caller: for callers
 * that cannot allocate device memory. The explainer has no counterpart; this is an
 * entry point of this library only.
 * Arguments, result and errors are those of pisa_run_host without `workspace` and
 * `workspace_bytes`: the device workspace is a fixed region of PISA_STATIC_WORKSPACE_BYTES
 * (32 MiB, 256-byte aligned) that the library holds on every device as part of its
 * loaded code, and the call allocates no memory (it creates and destroys its two copy
 * streams and events as pisa_run_host does). A problem whose pisa_run_host_workspace
 * figure exceeds the region is rejected with PISA_ERR_UNSUPPORTED before anything runs
 * (more `chunks` make each range, and the figure, smaller).
 * Nothing in the region has to start at zero: every byte the path reads there was
 * written earlier in the same call.
 * The region is ONE PER DEVICE, shared by every call on that device: calls that overlap
 * in time (from other host threads, or on other streams) race on it, and the caller
 * must serialise them. Each call blocks until it is done, so consecutive calls from one
 * thread are safe.
 * The first call on a device looks the region's address up (cudaGetSymbolAddress, with
 * that device current): make that first call outside any stream capture.
 */
pisa_status_t pisa_run_host_static(const void* Q, const void* K, const void* V, pisa_shape_t shape, int32_t topk,
                                   int32_t order, float scale, const pisa_host_options_t* options, void* O,
                                   void* stream);

/*
 * pisa_device_error -- takes the device error word that the kernels set, after all
 * work already enqueued on `stream`, and synchronises `stream`. Returns PISA_OK,
 * PISA_ERR_TIMEOUT (a bounded wait ran out), PISA_ERR_INVALID_ARG (an idx entry was out
 * of range) or PISA_ERR_CUDA.
 * The word is ONE PER DEVICE, shared by every stream and host thread that uses the
 * library on the current device: a bit raised by a kernel on any stream is reported by
 * the first pisa_device_error() that takes the word after the bit was raised, whatever
 * stream that call names, and is cleared by it. The take is one atomic exchange on the
 * device (read and clear cannot interleave with a kernel's raise), so no bit is lost; a
 * caller that needs per-launch attribution serialises its launches with this call.
 */
pisa_status_t pisa_device_error(void* stream);

/* Static description of a status code. Never NULL. */
const char* pisa_status_string(pisa_status_t status);

/* Detail of the last non-OK status returned on this host thread ("" if none). */
const char* pisa_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t pisa_version(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* PISA_H_ */
