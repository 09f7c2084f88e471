// kernels.h -- host-side launchers of the Block Transformer kernels.
// Every launcher enqueues on the given stream and returns the launch's
// cudaError_t (cudaSuccess when nothing was launched).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace bt {

enum DType : int { DT_F32 = 0, DT_BF16 = 1 };
inline size_t dt_size(int dt) { return dt == DT_F32 ? 4 : 2; }

// ---- per-device one-time state ---------------------------------------------
// Kernel attributes (cudaFuncSetAttribute) and device properties apply to the
// device that is current when they are set or read, so one-time set-up is
// kept per device.
constexpr int MAX_DEVICES = 64;
// Index of the current device, or -1 if it cannot be read or is >= MAX_DEVICES
// (callers then redo their set-up on every call instead of caching it).
int current_device();
// Multiprocessor count of the current device (148 if it cannot be read).
int device_sm_count();

// ---- embedder / token ingest / step state --------------------------------
// Prompt embedder: h[b*n + i, :] = concat_j blk_emb[tokens[b, i*L_B + j]].
// Ragged batches (row_pad / row_len non-null): sequence b is the row_len[b]
// tokens at the start of its row, preceded by row_pad[b] pad ids (pad_id);
// n_blocks (>= 0) blocks per sequence are embedded (blocks past a sequence's
// end read id 0).
cudaError_t launch_embed_prompt(int dt, const int32_t* tokens, int B, int T, int L_B,
                                const void* blk_emb, int V, int D, float* h, int* status,
                                cudaStream_t s, int n_blocks = -1, const int* row_pad = nullptr,
                                const int* row_len = nullptr, int pad_id = 0);
// Trailing prompt tokens of a prompt that ends inside a block: for b < B,
// i < r, token tokens[b * T_len + col0 + i] is recorded in block_tok[b, i]
// and its token-decoder embedding tok_emb[token] (+ add[b, i] when add is
// not null: summation injection's s_{i+1}, add [B, L_B - 1, D] fp32) is
// written to row b * rows_per_seq + row_off + i of h [.., D] (fp32).
cudaError_t launch_embed_tail(int dt, const int32_t* tokens, int B, int T_len, int col0, int r,
                              int rows_per_seq, int row_off, const void* tok_emb, int V, int D, float* h,
                              int32_t* block_tok, int L_B, int* status, cudaStream_t s,
                              const int* row_col0 = nullptr,  // per-sequence col0 (ragged)
                              const float* add = nullptr);
// Decode ingest of the fed token src[b] at position t = dstate[0]:
// records it in block_tok[b, t % L_B]; block_step = 0 gathers
// h[b] = tok_emb[src[b]] (+ add[b, t % L_B] when add is not null:
// summation injection's s_{j+1} for token j of the block); block_step = 1
// (the token completes its block) gathers h[b] = concat_j blk_emb[block_tok[b, j]].
cudaError_t launch_ingest(int dt, const int32_t* src, int32_t* block_tok, const int* dstate,
                          int B, int L_B, int V, int D, int block_step, const void* blk_emb,
                          const void* tok_emb, float* h, int* status, cudaStream_t s,
                          const float* add = nullptr);
// Context rows of the token decoder for the context-injection variants
// (one CTA per sequence and row, fp32):
//   CTX_WINDOW_SHIFT  h[b * h_rows + r] = ring[b][r + P] for r < (w-1)P,
//                     proj[b][r - (w-1)P] after: the window of the last w
//                     projected context embeddings, oldest first
//   CTX_WINDOW_SAVE   ring[b][r] = h[b * h_rows + r], r < wP
//   CTX_SUM_SPLIT     h[b * h_rows] = proj[b][0]; add[b][j] = proj[b][j + 1]
// ring [B, wP, D]; proj [B, P, D] (window) or [B, L_B, D] (summation);
// add [B, L_B - 1, D].
enum CtxMode { CTX_WINDOW_SHIFT = 0, CTX_WINDOW_SAVE = 1, CTX_SUM_SPLIT = 2 };
cudaError_t launch_ctx_rows(int mode, const float* proj, float* ring, float* h, float* add, int B, int w,
                            int P, int L_B, int D, int h_rows, cudaStream_t s);
// Ingest plus the first LayerNorm(s) of the gathered row (bf16): g2 != null ->
// x[b] = [LN1 | LN2] ([B, 2D]); else x[b] = LN(h[b]) ([B, D]).
cudaError_t launch_ingest_ln(const int32_t* src, int32_t* block_tok, const int* dstate, int B,
                             int L_B, int V, int D, int block_step, const void* blk_emb,
                             const void* tok_emb, float* h, const float* g1, const float* b1,
                             const float* g2, const float* b2, float eps, void* x, int* status,
                             cudaStream_t s);
// dstate <- position t (t, t % L_B, t / L_B).
cudaError_t launch_set_state(int* dstate, int t, int L_B, cudaStream_t s);
// dstate <- dstate[0] + 1.
cudaError_t launch_advance(int* dstate, int L_B, cudaStream_t s);

// ---- LayerNorm ------------------------------------------------------------
// x1[m, 0:D] = LN(h[m]; g1, b1), x1[m, D:2D] = LN(h[m]; g2, b2) (act dtype).
cudaError_t launch_ln_dual(int dt, const float* h, int M, int D, const float* g1,
                           const float* b1, const float* g2, const float* b2, float eps,
                           void* x1, cudaStream_t s);
// out[r] = LN(h[r * row_step + row_off]; g, b) for r < R (act dtype).
// row_lag (optional): row r reads h[r * row_step + row_off - row_lag[r]].
cudaError_t launch_ln_rows(int dt, const float* h, int R, int row_step, int row_off, int D,
                           const float* g, const float* b, float eps, void* out, cudaStream_t s,
                           const int* row_lag = nullptr);

// ---- rotary + KV append ---------------------------------------------------
// Row m of qkv [M, 3D] belongs to sequence m / rows_per_seq at position
// pos_base(pos) + m % rows_per_seq. Writes rotated q to q_out [M, D] and
// rotated k, v to the caches [B][H][cap][d] at that position.
// rope_tab[p * (rot/2) + i] = (cos, sin) of p * base^(-2i/rot).
// vt (optional, may be null): also write V transposed, vt[(b*H + h)*d + e][pos].
cudaError_t launch_rope_append(int dt, const void* qkv, int M, int D, int H, int rot,
                               const float2* rope_tab, PosSpec pos, void* q_out, void* k_cache,
                               void* v_cache, int cap, cudaStream_t s, void* vt = nullptr,
                               int vt_ld = 0, int Hk = 0);  // Hk: key/value heads (0 = H)
cudaError_t launch_rope_table(float2* tab, int n_pos, int rot, float base, cudaStream_t s);

// ---- attention --------------------------------------------------------------
// Split-K flash decoding: one query per (b, h) (q row b of q [B, ldq]) over
// the first n = pos_base(kvlen) + 1 cache entries; out[b, h*d:(h+1)*d].
// part / counters: scratch of attn_decode_scratch_bytes(); counters must be
// zero before the first launch and are left zero.
size_t attn_decode_scratch_bytes(int B, int H, int d, int cap, int dt);
// The scratch layout behind it: merge counters for `pairs` (sequence, head)
// pairs (padded to 256 bytes), then two partial slots of (d + 2) floats for
// each of at most ATTN_DECODE_MAX_CTAS persistent CTAs.
constexpr int ATTN_DECODE_MAX_CTAS = 4096;
constexpr size_t attn_decode_scratch_bytes_for(long long pairs, int d) {
  return (((size_t)pairs * sizeof(int) + 255) & ~(size_t)255) +
         (size_t)2 * ATTN_DECODE_MAX_CTAS * (size_t)(d + 2) * sizeof(float);
}
// One-time setup of the decode-attention kernels (shared-memory limits).
cudaError_t attn_prepare();
int attn_decode_max_splits(int d, int cap, int dt);
// Hk: key/value heads of the caches ([B][Hk][cap][d]); query head h reads
// head h / (H / Hk) (grouped-query attention; 0 = H). Same in the attention
// launchers below.
cudaError_t launch_attn_decode(int dt, const void* q, int ldq, const void* k_cache,
                               const void* v_cache, int B, int H, int d, int cap,
                               PosSpec kvlen, void* out, int ld_out, void* scratch,
                               int* status, cudaStream_t s, int Hk = 0);
// Small causal attention: rows_per_seq queries per sequence at positions
// pos_base(qpos) + i; query at position p attends to cache entries 0..p.
cudaError_t launch_attn_small(int dt, const void* q, int ldq, const void* k_cache,
                              const void* v_cache, int B, int H, int d, int cap, PosSpec qpos,
                              void* out, int ld_out, cudaStream_t s, int Hk = 0);
// Tensor-core prefill attention (bf16, d in {64, 128}): as launch_attn_prefill
// but V is read through its transpose vt [B*H][d][vt_ld] (keys contiguous).
int attn_prefill_tc_supported(int dt, int d, int ldq, int vt_ld);
cudaError_t launch_attn_prefill_tc(const void* q, int ldq, const void* k_cache, const void* vt,
                                   int vt_ld, int B, int H, int d, int cap, int n, void* out,
                                   int ld_out, int* status, cudaStream_t s, int Hk = 0);
// Prefill causal attention over n positions 0..n-1 of every sequence:
// q rows b*n + i of q [B*n, ldq]; out rows likewise.
cudaError_t launch_attn_prefill(int dt, const void* q, int ldq, const void* k_cache,
                                const void* v_cache, int B, int H, int d, int cap, int n,
                                void* out, int ld_out, cudaStream_t s, int Hk = 0);

// ---- GEMM -----------------------------------------------------------------
enum EpiKind : int {
  EPI_QKV1 = 0,   // n < split_n: out0[m, n] = acc + bias[n] (act);
                  // n >= split_n: out1[m, D + n - split_n] = gelu(acc + bias[n]) (act)
  EPI_RESID = 1,  // out0 (fp32) [m, n] += acc + bias[n]
  EPI_F32 = 2,    // out0 (fp32) [m, n] = acc (+ bias[n] if bias)
  EPI_ACT = 3,    // out0 (act)  [m, n] = acc (+ bias[n] if bias)
  EPI_QKV1_ROPE = 4,  // as EPI_QKV1, with rotary + KV-cache append fused:
                      // q (rotated) -> out0 [m, n]; k (rotated), v -> the
                      // caches at the token's position (tensor-core decode
                      // orientation only, see gemm_rope_fusable)
  EPI_LOGITS_ARGMAX = 5,  // LM head: logits -> out0 [m, n] fp32 if out0 != null;
                          // per 128-row tile t, the (max, lowest argmax) of
                          // column m -> aux[t * M + m] (float2: value, index
                          // bits); tensor-core decode orientation only
};

struct Epi {
  int kind;
  void* out0;
  int ld0;
  void* out1;
  int ld1;
  const float* bias;
  int split_n;
  int D;
  // EPI_QKV1_ROPE only
  const float2* rope_tab;
  int rot;
  int H;
  void* kc;
  void* vc;
  int cap;
  PosSpec pos;
  // EPI_LOGITS_ARGMAX only
  void* aux;
  // Fused LayerNorm of completed rows (EPI_RESID / EPI_F32, tensor-core decode
  // orientation, N = the full row width D): the feature tile that completes
  // row m of out0 last computes LayerNorm(s) of that row. ln_g2 != null: both
  // LN1 and LN2 -> ln_out [M, 2D]; else one LN of rows m % ln_step == ln_off
  // -> ln_out row m / ln_step. ln_cnt: per-row counters, zero between launches.
  const float* ln_g1;
  const float* ln_b1;
  const float* ln_g2;
  const float* ln_b2;
  void* ln_out;
  int* ln_cnt;
  int ln_step;
  int ln_off;
  float ln_eps;
  // EPI_QKV1_ROPE: key/value heads (0 = H): output features are q (D) |
  // k (Hk d) | v (Hk d) | fc1 (4D), the caches [B][Hk][cap][d]
  int Hk;
};
// True when launch_gemm runs EPI_LOGITS_ARGMAX for this shape.
int gemm_argmax_fusable(int dt, int M, int N, int K);
// next[m] = index of the best of the n_tiles partial (value, index) pairs
// part[t * M + m] (lowest index among equal values).
// dstate (optional): advanced to the next position by the same kernel.
cudaError_t launch_argmax_reduce(const float2* part, int n_tiles, int M, int32_t* next,
                                 cudaStream_t s, int* dstate = nullptr, int L_B = 1);
// True when launch_gemm will run EPI_QKV1_ROPE fused for this shape.
int gemm_rope_fusable(int dt, int M, int N, int K, int xk_split, int xk_off, int d_head, int rot);

// out = X [M, K] (row stride ldx) . W [N, K]^T (row stride ldw), fp32
// accumulation; for output columns n >= xk_split the X columns read are
// shifted by xk_off. scratch: split-K partials (gemm_scratch_bytes).
struct GemmScratch {
  float* part;        // split-K partial tiles
  size_t part_bytes;
  int* counters;      // per output tile, zero between launches
  int n_counters;
};
size_t gemm_scratch_bytes(int max_M, int max_N);
int gemm_counter_count(int max_N);
cudaError_t launch_gemm(int dt, const void* X, int ldx, const void* W, int ldw, int M, int N,
                        int K, int xk_split, int xk_off, const Epi& e, const GemmScratch& scr,
                        int* status, cudaStream_t s);
// One-time setup of the tensor-core kernels (shared-memory limits).
cudaError_t gemm_tc_prepare();
// 0 = automatic, 1 = force the SIMT path, 2 = force the tensor-core path.
void gemm_set_path(int path);
int gemm_tc_supported(int dt, int M, int N, int K, int xk_split, int xk_off);

// ---- fused token-decoder step -------------------------------------------------
// One persistent kernel for the token-decoder half of a decode step (bf16,
// B <= 64, prefix length 1): the row of each sequence through every
// token-decoder layer (local attention over the window in the local cache,
// the new k, v appended at `pos`), the final LayerNorm, the LM head (logits
// -> `logits` when not null), the greedy argmax -> `next`, and the step state
// advanced by one position. Layer l's parameters sit at layer 0's pointers
// plus l * layer_stride bytes (weights, biases and gains alike).
struct TokenStepArgs {
  int B, D, H, dh, rot, V, Nt, L_B, l_cap;
  float eps;
  int ingest;        // 1: h = token embedding of src[b] first (block_tok updated)
  PosSpec pos;       // position of the row in the local window
  const int32_t* src;
  int32_t* block_tok;
  const bf16* tok_emb;
  int* dstate;
  const float *b_qkv1, *b_o2, *ln1_g, *ln1_b, *ln2_g, *ln2_b;
  long long layer_stride;
  bf16 *kt, *vt;     // local caches [layer][B][H][l_cap][dh]
  long long kt_layer;
  const float2* rope_tab;
  const float *lnf_g, *lnf_b;
  float* h;          // [B, D] fp32 residual rows
  bf16 *x1, *a2, *xf;
  float* logits;
  int32_t* next;
  float2* arg_part;  // [ceil(V/128), B]
  unsigned long long* arg_key;  // token_step: [B] argmax keys, zero between launches (the last CTA resets them)
  float *p1, *p2;    // split-K partials (token_step_scratch_floats)
  long long* fx;     // token_step: [B, D] int64 fixed-point split-K sums (units of 2^-32),
                     // zero between launches (each launch clears what it adds)
  unsigned* bar;     // 3 words, zero before the first launch
  int* status;
  long long wait_cycles;  // bound of every wait of the launch (SM clock cycles)
  // token_step2 only: per-(row, 128-feature tile) (mean, sum of squared
  // deviations) of h [B][D/128]. Both kernels: an L2 persisting access-policy
  // window for the launch (bytes 0 = none)
  float2* hstat;
  bf16* hb;          // token_step2: bf16 copy of h [B, D] (the G1 units' TMA source)
  void* l2_window_base;
  size_t l2_window_bytes;
  float l2_hit_ratio;
  // Block step (block = 1): the fed token completes a block. The block
  // embedding, every block-decoder layer (decode attention over the block
  // cache, the new entry appended at dstate[2]), LN_b and the prefix
  // projection run first; the token decoder then runs over the prefix row
  // (pos must be position 0) and no token is ingested. Block layer l's
  // parameters sit at block layer 0's pointers plus l * layer_stride bytes.
  int block, Nb, n_cap;
  const bf16* blk_emb;
  float* h_b;        // [B, D] fp32 block-decoder residual rows
  const float *bb_qkv1, *bb_o2, *bln1_g, *bln1_b, *bln2_g, *bln2_b;
  bf16 *kb, *vb;     // block caches [layer][B][H][n_cap][dh]
  long long kb_layer;
  const float *lnb_g, *lnb_b, *b_prefix;
  float* att_part;   // decode-attention chunk partials (token_step_scratch_floats, which = 3)
  int* att_cnt;      // [B * H] merge counters, zero between launches
};
int token_step_supported(int dt, int B, int D, int H, int rot, int V, int Nt, int P_prefix, int l_cap);
// the block-step form as well (d_head 64, at least one block layer)
int token_step_block_supported(int dt, int B, int D, int H, int rot, int V, int Nt, int Nb, int P_prefix,
                               int l_cap, int n_cap, int L_B);
// which = 1: first-GEMM partials, 2: second-GEMM partials (floats, for B rows);
// 3: block decode-attention partials for n_cap cached entries
size_t token_step_scratch_floats(int B, int D, int which, int H = 0, int n_cap = 0);
// w_qkv1_b, w_o2_b, w_prefix: block layer 0's weights and the prefix
// projection, used when a.block (may be null otherwise)
cudaError_t launch_token_step(const TokenStepArgs& a, const void* w_qkv1, const void* w_o2,
                              const void* w_lm, const void* w_qkv1_b, const void* w_o2_b,
                              const void* w_prefix, cudaStream_t s);

// The token-decoder half of a decode step as one persistent kernel with no
// grid-wide barrier (token_step.cu): bf16, B <= 64, d_head in {32, 64, 128},
// rotary on none or the first d_head/4 dims, local window <= 16 rows, any
// prefix length. a.bar: token_step2_counter_bytes(D) bytes, zero before the
// first launch (a launch leaves them zero unless a wait ran out); a.p1, a.p2,
// a.hstat, a.hb: token_step2_scratch_floats(B, D, 1 | 2 | 3 | 4) floats.
int token_step2_supported(int dt, int B, int D, int H, int rot, int V, int Nt, int l_cap);
size_t token_step2_counter_bytes(int D);
size_t token_step2_scratch_floats(int B, int D, int which);
cudaError_t launch_token_step2(const TokenStepArgs& a, const void* w_qkv1, const void* w_o2, const void* w_lm,
                               cudaStream_t s);

// ---- LM head argmax ---------------------------------------------------------
// next[b] = argmax_v logits[b, v] (lowest id among ties).
cudaError_t launch_argmax(const float* logits, int B, int V, int ld, int32_t* next,
                          cudaStream_t s);

// Record a failed CUDA call for bt_last_cuda_error (per thread).
void note_cuda_error(const char* what, cudaError_t e);

// ---- launch accounting ------------------------------------------------------
// Every kernel launch site calls note_launch(); launch_count() is the running
// total for this process (graph captures count when captured).
void note_launch();
long long launch_count();

// Programmatic dependent launch on every kernel (on unless BT_NO_PDL=1).
bool pdl_enabled();

// Launch through cudaLaunchKernelEx with the programmatic-serialization
// attribute (the kernel overlaps its prologue with the previous kernel's
// tail; see pdl_trigger / pdl_wait) and count it.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
  note_launch();
  return e;
}

#define BT_LAUNCH(...)                               \
  do {                                               \
    cudaError_t e_ = ::bt::launch_ex(__VA_ARGS__);   \
    if (e_ != cudaSuccess) return e_;                \
  } while (0)

// ---- misc -----------------------------------------------------------------
cudaError_t launch_convert_to_f32(int dt, const void* src, float* dst, size_t n, cudaStream_t s);
cudaError_t launch_add_to_f32(int dt, const void* a, const void* b, float* dst, size_t n,
                              cudaStream_t s);

}  // namespace bt
