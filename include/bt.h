/*
 * bt.h -- Block Transformer global-to-local inference on B200 (sm_100a).
 *
 * The model is the Block Transformer of "Block Transformer: Global-to-Local
 * Language Modeling for Fast Inference" (arXiv 2406.02657; explainer page of
 * that title, cited here by section):
 *   embedder       token ids -> block embeddings, L_B lookups of width D/L_B
 *                  concatenated (§3.4 "The Embedder" [orig. §2.2]);
 *   block decoder  causal transformer over blocks, KV cache L_B times
 *                  shorter than the token sequence (§3.4 "The Block Decoder"
 *                  [orig. §2.3]);
 *   prefix         context embedding c_i -> P prefix rows by a linear map
 *                  (§3.4 "The Token Decoder", prefix mechanism [orig. §2.4]);
 *   token decoder  causal transformer over [prefix; current block's tokens]
 *                  only (§3.2 item 3, §3.4 "The Token Decoder");
 *   LM head        next-token logits, greedy argmax.
 * The inference stages are those of §3.4 "Prefill vs. decode": one prefill
 * call per prompt, then one decode call per generated token.
 *
 * Conventions for every entry point below
 *   - Pointers named *_dev are device pointers on the current CUDA device;
 *     host pointers are named without the suffix.
 *   - All device work is enqueued on the stream given to bt_create (a
 *     cudaStream_t passed as void*, NULL = the legacy default stream) and the
 *     call returns after enqueueing. Outputs are valid once that stream has
 *     reached them (bt_sync, or any later stream-ordered consumer).
 *   - The library never allocates device memory: all device state lives in
 *     the caller's workspace. It creates one private CUDA stream (graph
 *     capture) per model.
 *   - Errors are returned as negative bt_status codes; the library never
 *     aborts the process and never traps the device. Device-side failures
 *     (a token id outside [0, vocab), a bounded wait that ran out) set a
 *     status word in the workspace, reported by the next bt_sync.
 *   - A bt_model is not thread-safe; calls on one model are serialised by
 *     the caller.
 */
#ifndef BT_H_
#define BT_H_

#include <stddef.h>
#include <stdint.h>

/* Symbols of the shared library are exported; everything else is hidden. */
#if defined(__GNUC__)
#define BT_API __attribute__((visibility("default")))
#else
#define BT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bt_status {
  BT_OK = 0,
  BT_EINVAL = -1,      /* bad argument or configuration                      */
  BT_EWORKSPACE = -2,  /* workspace NULL, misaligned (256 B) or too small    */
  BT_ECAPACITY = -3,   /* batch > max_batch or tokens would exceed max_seq   */
  BT_ESTATE = -4,      /* decode before prefill                              */
  BT_ECUDA = -5,       /* a CUDA runtime call failed (see bt_last_cuda_error) */
  BT_EDEVICE = -6,     /* a kernel reported a failure through the status word */
  BT_ENOTSUP = -7      /* valid but unsupported shape (see message)          */
} bt_status;

typedef enum bt_dtype { BT_FP32 = 0, BT_BF16 = 1 } bt_dtype;

/* Model hyper-parameters. Pythia-style layers: LayerNorm (biased variance,
 * eps ln_eps), parallel attention + MLP residual, rotary embedding on the
 * first rotary_dims dims of each head (rotate-half pairing, base rope_base),
 * exact-erf GELU, MLP width 4*d_model, untied LM head without bias. */
typedef struct bt_config {
  int32_t vocab;             /* V                                             */
  int32_t d_model;           /* D; multiple of n_heads, of block_len and of 8  */
  int32_t n_heads;           /* H; d_head = D / H in {32, 64, 128}             */
  int32_t block_len;         /* L_B >= 1                                      */
  int32_t n_block_layers;    /* N_b >= 0                                      */
  int32_t n_token_layers;    /* N_t >= 0 (ignored when use_token_decoder = 0) */
  int32_t prefix_len;        /* P >= 1 (ignored when use_token_decoder = 0)   */
  int32_t rotary_dims;       /* even, <= d_head                               */
  int32_t use_token_decoder; /* 0: vanilla model, requires block_len = 1; the
                                LM head reads LN_b of the block decoder      */
  int32_t max_batch;         /* B_max. Every device buffer must hold fewer
                                than 2^31 elements (kernels index within one
                                buffer in 32 bits): B_max * ceil(max_seq/L_B)
                                * 5 d_model, B_max * vocab and B_max * d_model
                                * ceil(max_seq/L_B) (rounded up to 64) must
                                stay below 2^31, else BT_ENOTSUP            */
  int32_t max_seq;           /* prompt + generated tokens, per sequence       */
  int32_t dtype;             /* bt_dtype: storage and GEMM-input type; fp32
                                accumulation and fp32 residual stream always  */
  float ln_eps;              /* 1e-5 for Pythia                               */
  float rope_base;           /* 10000 for Pythia                              */
  /* How the context embedding c reaches the token decoder (explainer page
   * §3.4 "The Token Decoder" and its alternatives to prefix tokens; App. B.3
   * for the window). 0 = prefix: the last context_window context embeddings
   * are each projected to P rows (W_p [P*D, D], shared), oldest first, zero
   * vectors before the first block; 1 = summation: c is projected to L_B
   * vectors s_0..s_{L_B-1} (W_p [L_B*D, D]), s_0 is the token decoder's
   * first row and s_{j+1} is added to the input row of token j of the block
   * (requires prefix_len = 1 and context_window = 1). Both default to the
   * base model when zero-initialised. Variants other than the base model
   * run the token decoder as a chain of kernels; context_window > 1 does not
   * support ragged batches (bt_prefill_ragged returns BT_ENOTSUP). */
  int32_t context_injection;
  int32_t context_window;    /* w >= 1 (0 is read as 1)                       */
  /* Key/value heads of the block decoder's attention (grouped-query
   * attention, explainer page §3.4 "The Block Decoder": standard attention,
   * so MQA/GQA apply); query head h reads key/value head h / (H / H_kv);
   * 0 = n_heads; must divide n_heads. The token decoder keeps H heads. */
  int32_t n_kv_heads;
} bt_config;

/* One Pythia layer. Matrices are row-major [out, in] (torch Linear layout) in
 * the config dtype; vectors are in the config dtype too.
 *   w_qkv [3D, D] rows ordered q | k | v, each head-major [H, d_head]; b_qkv [3D]
 *     (block-decoder layers with n_kv_heads = H_kv: [D + 2 H_kv d_head, D],
 *     k and v with H_kv heads each)
 *   w_o [D, D], b_o [D]; w_1 [4D, D], b_1 [4D]; w_2 [D, 4D], b_2 [D]
 *   ln1_* feeds attention, ln2_* feeds the MLP (parallel residual). */
typedef struct bt_layer_weights {
  const void *ln1_g_dev, *ln1_b_dev, *ln2_g_dev, *ln2_b_dev;
  const void *w_qkv_dev, *b_qkv_dev, *w_o_dev, *b_o_dev;
  const void *w_1_dev, *b_1_dev, *w_2_dev, *b_2_dev;
} bt_layer_weights;

/* Whole-model parameters (config dtype):
 *   blk_emb  [V, D/L_B] embedder table        lnf_b_* [D] final LN of the block decoder
 *   w_prefix [P*D, D], b_prefix [P*D]  Proj   tok_emb [V, D] token-decoder table
 *   lnf_t_*  [D] final LN of the token decoder  w_lm [V, D] LM head
 * w_prefix, b_prefix, tok_emb and lnf_t_* may be NULL when
 * use_token_decoder = 0. block_layers / token_layers are HOST arrays of
 * n_block_layers / n_token_layers entries. */
typedef struct bt_weights {
  const void *blk_emb_dev, *lnf_b_g_dev, *lnf_b_b_dev;
  const void *w_prefix_dev, *b_prefix_dev, *tok_emb_dev;
  const void *lnf_t_g_dev, *lnf_t_b_dev, *w_lm_dev;
  const bt_layer_weights *block_layers;
  const bt_layer_weights *token_layers;
} bt_weights;

typedef struct bt_model bt_model;

/* Bytes of device workspace bt_create needs for cfg (weights repacked into
 * fused layouts, block and local KV caches, activations, scratch). Returns 0
 * if cfg is invalid. */
BT_API size_t bt_workspace_bytes(const bt_config *cfg);

/* Validate cfg, carve the workspace, and enqueue on `stream` the copy of all
 * weights into the workspace (q|k|v|fc1 rows concatenated into one [7D, D]
 * matrix; [W_o | W_2] into one [D, 5D] matrix; vectors converted to fp32).
 * The caller's weight buffers must stay valid until that copy has run (e.g.
 * until bt_sync returns); afterwards they are not read again. The workspace
 * (256-byte aligned, >= bt_workspace_bytes(cfg)) is owned by the caller and
 * must outlive the model. On success *out receives the handle. */
BT_API int bt_create(const bt_config *cfg, const bt_weights *w, void *workspace_dev,
              size_t workspace_bytes, void *stream, bt_model **out);

/* Prefill: process prompts tokens_dev [batch, prompt_len] (int32,
 * row-major, ids in [0, V)) for all `batch` sequences, resetting any earlier
 * state. Runs the embedder and the block decoder over the n =
 * floor(prompt_len / L_B) complete blocks (filling the block KV cache), then
 * the prefix projection of the last complete block's context and the token
 * decoder over the P prefix rows followed by the r = prompt_len mod L_B
 * trailing tokens, which are the first tokens of the current block (earlier
 * blocks never enter the token decoder, §3.4 token-decoder cost analysis;
 * prompts that end inside a block, §3.4 "The Embedder"). Writes the logits
 * predicting token prompt_len to logits_dev [batch, V] fp32 (if non-NULL)
 * and their greedy argmax (lowest id among ties) to next_tokens_dev [batch]
 * int32 (if non-NULL).
 * Requires 1 <= batch <= max_batch, prompt_len >= L_B, prompt_len < max_seq. */
BT_API int bt_prefill(bt_model *m, const int32_t *tokens_dev, int32_t batch,
               int32_t prompt_len, float *logits_dev, int32_t *next_tokens_dev);

/* Prefill of a ragged batch: sequence b's prompt is the first lengths[b]
 * tokens of row b of tokens_dev [batch, row_stride] (int32, device);
 * `lengths` is a HOST array of `batch` entries, 1 <= lengths[b] <= row_stride.
 *   pad_id >= 0: inference left padding (§3.4 "The Embedder", prompts whose
 *     length is not a multiple of L_B): each prompt is preceded by
 *     (-lengths[b]) mod L_B pad tokens of id pad_id, so that every sequence
 *     ends on a block boundary.
 *   pad_id < 0: no padding; every lengths[b] must leave the same remainder
 *     mod L_B (the remainder's trailing tokens enter the token decoder as in
 *     bt_prefill).
 * Each sequence keeps its own number of blocks: the block decoder's KV cache
 * of sequence b holds only its own blocks, and decode attention reads only
 * them. Decode calls then run all sequences in step (the token decoders are
 * at the same position of their blocks). bt_position reports the longest
 * (padded) sequence's position; max_seq bounds it. Every padded length must
 * be >= L_B. Errors as bt_prefill, and BT_EINVAL for lengths outside
 * [1, row_stride], unequal remainders without padding, or pad_id >= V. */
BT_API int bt_prefill_ragged(bt_model *m, const int32_t *tokens_dev, int32_t row_stride,
                             const int32_t *lengths, int32_t batch, int32_t pad_id,
                             float *logits_dev, int32_t *next_tokens_dev);

/* Decode one token per sequence. tokens_dev [batch] int32 is the token fed
 * at position t (teacher forcing); NULL feeds the model's own greedy argmax
 * from the previous call. Writes logits for token t+1 (if logits_dev) and
 * their argmax (if next_tokens_dev), as bt_prefill. When the fed token
 * completes a block the block decoder appends one entry to its cache and a
 * new token-decoder block starts from its context; otherwise the token
 * decoder appends one row to the block's local cache.
 * Errors: BT_ESTATE before a prefill, BT_ECAPACITY when t + 1 would exceed
 * max_seq.
 * Execution: each call is one CUDA-graph replay on the model's stream. For
 * bf16 models with batch <= 64 and prefix length 1 the token-decoder half of
 * the step (all token-decoder layers, the LM head, the argmax) is a single
 * persistent kernel launched cooperatively with one CTA on every SM: it
 * waits for SMs held by other work on the device, and the driver refuses it
 * if the device cannot hold one CTA per SM (the call then returns
 * BT_ECUDA). */
BT_API int bt_decode_step(bt_model *m, const int32_t *tokens_dev, float *logits_dev,
                   int32_t *next_tokens_dev);

/* Wait for the model's stream, then read and clear the device status word.
 * Returns BT_OK, BT_EDEVICE (a kernel reported a failure) or BT_ECUDA. */
BT_API int bt_sync(bt_model *m);

/* Position of the next token to be fed (the number of tokens seen per
 * sequence), or a negative status. */
BT_API int bt_position(const bt_model *m);

/* Release host-side resources (graphs, streams). Does not free the caller's
 * workspace. Waits for the model's outstanding work first. */
BT_API int bt_destroy(bt_model *m);

/* ---- measurement support ------------------------------------------------
 * Kernel kinds reported by the profiler. */
enum {
  BT_K_GEMM = 0, BT_K_ATTN_DECODE = 1, BT_K_ATTN_PREFILL = 2, BT_K_ATTN_LOCAL = 3,
  BT_K_LAYERNORM = 4, BT_K_ROPE_APPEND = 5, BT_K_EMBED = 6, BT_K_ARGMAX = 7, BT_K_OTHER = 8,
  BT_K_TOKEN_STEP = 9,  /* fused token decoder + LM head + argmax: m = B, n = vocab, k = d_model */
  BT_K_BLOCK_STEP = 10  /* the same kernel on a block step, block decoder and prefix included */
};

/* One timed kernel launch: kind, shape (GEMM: M, N, K; decode attention:
 * B*H, cached entries read, d_head; others: rows, width, 0) and its duration
 * from a pair of CUDA events recorded on the model's stream around it. */
typedef struct bt_profile_record {
  int32_t kind, m, n, k;
  float ms;
} bt_profile_record;

/* Number of this model's kernels that have been enqueued for execution so
 * far (each replay of a captured decode graph counts its kernel nodes). */
BT_API int64_t bt_kernel_launches(const bt_model *m);

/* Start recording an event pair around every kernel launch, for at most
 * `capacity` launches. While recording, decode steps are enqueued kernel by
 * kernel instead of as graph replays. Creates 2*capacity CUDA events. */
BT_API int bt_profile_begin(bt_model *m, int32_t capacity);

/* Stop recording, wait for the stream, and copy up to `capacity` records
 * into out (host array); *n_out receives the number copied. */
BT_API int bt_profile_end(bt_model *m, bt_profile_record *out, int32_t capacity,
                          int32_t *n_out);

/* Static, human-readable name of a status code. */
BT_API const char *bt_strerror(int status);

/* Text of the last CUDA error this thread saw inside the library, or "". */
BT_API const char *bt_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* BT_H_ */
