/*
 * bt_ops.h -- single-kernel entry points of the Block Transformer library.
 *
 * These expose individual kernels of the bt.h path so that each can be
 * checked and timed on its own. Same conventions as bt.h: *_dev pointers
 * are device pointers; `stream` is a cudaStream_t as void* (NULL = legacy
 * default stream); work is enqueued and the call returns; negative
 * bt_status codes on error; no device memory is allocated (scratch is
 * passed in). dtype is a bt_dtype: BT_BF16 tensors hold bf16, BT_FP32
 * tensors fp32; accumulation is fp32 in both.
 */
#ifndef BT_OPS_H_
#define BT_OPS_H_

#include <stddef.h>
#include <stdint.h>

#include "bt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Block-decoder decode attention, split-K flash decoding ("Block
 * Transformer: Global-to-Local Language Modeling for Fast Inference", §3.4
 * "The Block Decoder": one new block per sequence attends over its block KV
 * cache).
 *   q_dev       [B, ldq] dtype; head h of sequence b at q[b*ldq + h*d ...]
 *   k_dev,v_dev [B, H, cap, d] dtype; entries 0..n-1 are read
 *   out_dev     [B, ld_out] dtype; out[b*ld_out + h*d + e]
 *   softmax(q k^T / sqrt(d)) v over the n entries, per (b, h).
 *   scratch_dev >= bt_op_decode_attention_scratch_bytes(...) bytes, 256-byte
 *   aligned, zero-filled before its first use; the call leaves it ready for
 *   further calls with the same B and H (re-zero it when B or H changes).
 * Requires d in {32, 64, 128}, 1 <= n <= cap, 16-byte aligned rows.
 * Calls that share a scratch buffer must not overlap on the GPU. */
BT_API size_t bt_op_decode_attention_scratch_bytes(int dtype, int B, int H, int d, int cap);
BT_API int bt_op_decode_attention(int dtype, const void *q_dev, int ldq, const void *k_dev,
                           const void *v_dev, int B, int H, int d, int cap, int n, void *out_dev,
                           int ld_out, void *scratch_dev, size_t scratch_bytes, void *stream);

/* bt_op_decode_attention without a scratch argument, for callers that cannot
 * allocate device memory at the time they run it (for example while recording
 * a CUDA graph, where cudaMalloc is not a capturable operation, or inside a
 * runtime whose device memory is a fixed pool carved at start-up). The paper
 * has no counterpart: this is an integration convenience of this library.
 *   Arguments and result as bt_op_decode_attention (q, k, v, out are still the
 *   caller's). The split-K merge state lives in one fixed array compiled into
 *   the library (about 4.3 MB, held on every GPU that loads the library until
 *   the process exits), so it allocates nothing: it calls no cudaMalloc,
 *   cudaFree or allocating library routine.
 *   Limits: B*H <= 8192 and d <= 128; larger problems return BT_ECAPACITY.
 *   The first call on each device looks up the array's device address (with
 *   that device current) and caches it; make that first call before any
 *   stream capture. Every call zeroes the merge counters it uses on `stream`.
 *   All calls share the one array: calls that may overlap on the GPU (other
 *   streams, other threads) race and must be serialised by the caller. */
BT_API int bt_op_decode_attention_noalloc(int dtype, const void *q_dev, int ldq,
                                          const void *k_dev, const void *v_dev, int B, int H,
                                          int d, int cap, int n, void *out_dev, int ld_out,
                                          void *stream);

/* Causal attention of the block decoder at prefill: queries are the n rows
 * b*n + i of q_dev [B*n, ldq]; query i attends to cache entries 0..i of
 * k_dev/v_dev [B, H, cap, d]; out rows likewise. */
BT_API int bt_op_prefill_attention(int dtype, const void *q_dev, int ldq, const void *k_dev,
                            const void *v_dev, int B, int H, int d, int cap, int n,
                            void *out_dev, int ld_out, void *stream);

/* Tensor-core form of bt_op_prefill_attention (bf16, d in {64, 128}): the same
 * causal attention, with V read through its transpose vt_dev [B*H][d][vt_ld]
 * (vt[(b*H + h)*d + e][i] = V[b][h][i][e]); vt_ld a multiple of 8. Returns
 * BT_ENOTSUP for other types or head sizes. */
BT_API int bt_op_prefill_attention_tc(const void *q_dev, int ldq, const void *k_dev,
                                      const void *vt_dev, int vt_ld, int B, int H, int d, int cap,
                                      int n, void *out_dev, int ld_out, void *stream);

/* Dense projection out = X W^T (+ bias): X [M, ldx] dtype, W [N, K] dtype
 * row-major, bias fp32 [N] or NULL, out fp32 [M, ld_out]. path: 0 automatic
 * (tensor cores when the shape allows), 1 SIMT FFMA, 2 tensor cores only
 * (BT_ENOTSUP if the shape is not supported). scratch as bt.h's GEMMs:
 * >= bt_op_linear_scratch_bytes(M, N) bytes, zero-filled before first use. */
BT_API size_t bt_op_linear_scratch_bytes(int M, int N);
BT_API int bt_op_linear(int dtype, const void *x_dev, int ldx, const void *w_dev, const float *bias_dev,
                 float *out_dev, int ld_out, int M, int N, int K, int path, void *scratch_dev,
                 size_t scratch_bytes, void *stream);

/* out[m] = LayerNorm(h[m]) * g + b over D features (biased variance):
 * h fp32 [M, D], g/b fp32 [D], out dtype [M, D]. */
BT_API int bt_op_layernorm(int dtype, const float *h_dev, int M, int D, const float *g_dev,
                    const float *b_dev, float eps, void *out_dev, void *stream);

/* Embedder (§3.4 "The Embedder"): h[b*n + i, j*D/L + e] =
 * table[tokens[b, i*L + j], e], n = T / L. tokens int32 [B, T]; table dtype
 * [V, D/L]; h fp32 [B*n, D]. Ids outside [0, V) read row 0 and set bit 1 of
 * *status_dev (int32, may be NULL). */
BT_API int bt_op_embed_prompt(int dtype, const int32_t *tokens_dev, int B, int T, int L,
                       const void *table_dev, int V, int D, float *h_dev, int32_t *status_dev,
                       void *stream);

/* Self-test of the bounded grid-wide barrier that the persistent decode kernel
 * uses between its phases (failure detection without a GPU fault; the pages
 * have no counterpart). Launches one CTA per SM, cooperatively, each passing
 * `rounds` barriers.
 *   words_dev   3 uint32, zero before the call: arrival counter, exit counter,
 *               abort word. The kernel leaves the counters zero; a timeout
 *               leaves the abort word set (clear it before reusing the words).
 *   withhold_cta -1, or a CTA index (< number of SMs) that does not arrive at
 *               the first barrier: every CTA's wait then runs out after
 *               wait_cycles SM clock cycles, ST_WAIT_TIMEOUT (2) is or-ed into
 *               *status_dev, the abort word is set, and every CTA returns.
 *   passed_dev  int, zero before the call; receives the sum over CTAs of the
 *               barriers passed (rounds * number of SMs when nothing ran out).
 * Returns BT_ENOTSUP if the device cannot launch cooperatively. */
BT_API int bt_op_grid_barrier_selftest(int rounds, int withhold_cta, long long wait_cycles,
                                       unsigned *words_dev, int *status_dev, int *passed_dev,
                                       void *stream);

#ifdef __cplusplus
}
#endif
#endif /* BT_OPS_H_ */
