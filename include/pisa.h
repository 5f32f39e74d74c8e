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
 *    retains caller memory after the call returns (it does cache TMA descriptors that
 *    hold the pointer values, keyed by pointer and shape).
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
 *    host thread.
 */
#ifndef PISA_H_
#define PISA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PISA_MAX_BLOCKS 2048

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
 * K, V: bf16 [B, H, N, d]. order: 0 or 1; S1 is written only when order == 1 and may
 * be NULL when order == 0.
 */
pisa_status_t pisa_block_stats(const void* K, const void* V, pisa_shape_t shape, int32_t order,
                               float* kbar, float* S0, void* S1, void* stream);

/*
 * pisa_select -- top-k critical key blocks of every query block.
 *
 * Section 2, "Covariance-aware routing" (selection by attention relevance; the
 * covariance term is not part of this call): the relevance of key block j to query
 * block i is the pooled score qbar_i . kbar_j, with qbar_i the mean of query block
 * i's real rows, computed in fp32. idx[b,h,i,:] receives the topk blocks with the
 * largest scores, equal scores resolved toward the lower block index, written in
 * ascending block order.
 * Q: bf16 [B, H, N, d]; kbar: fp32 [B, H, nB, d] (from pisa_block_stats);
 * idx: int32 [B, H, nB, topk]; 1 <= topk <= nB.
 */
pisa_status_t pisa_select(const void* Q, const float* kbar, pisa_shape_t shape, int32_t topk,
                          int32_t* idx, void* stream);

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
 *   D_t = sum_{j in S_i} sum_n e^{x_t.k_n} + sum_{j not in S_i} n_j e^{x_t.kbar_j}
 *   O_t = N_t / D_t                                  bf16 [B, H, N, d]
 * All exponents are taken relative to one running row maximum (a single online-softmax
 * accumulator). idx rows must hold topk distinct blocks in [0, nB) (the order inside a
 * row does not matter); out-of-range entries are ignored and flagged in the device
 * error word. S1 may be NULL when order == 0. scale must be finite and > 0.
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

/*
 * pisa_device_error -- synchronises `stream`, then reads and clears the device error
 * word that the kernels set. Returns PISA_OK, PISA_ERR_TIMEOUT (a bounded wait ran
 * out), PISA_ERR_INVALID_ARG (an idx entry was out of range) or PISA_ERR_CUDA.
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
