// elementwise.cu -- embedder, decode ingest, LayerNorm, rotary + KV append,
// argmax and small conversions for the Block Transformer (sm_100a).
//
// Model: "Block Transformer: Global-to-Local Language Modeling for Fast
// Inference" (explainer page of arXiv 2406.02657). Embedder: §3.4 "The
// Embedder" [orig. §2.2] -- L_B lookups of width D/L_B concatenated, token j
// of a block in dims [j*D/L_B, (j+1)*D/L_B). Layer pieces follow the Pythia
// architecture named in §5 "Experimental setup" (LayerNorm with biased
// variance, rotate-half rotary on the first 25% of each head).
#include <stdlib.h>

#include "common.cuh"
#include "kernels.h"

namespace bt {

static long long g_launches = 0;
void note_launch() { __atomic_add_fetch(&g_launches, 1, __ATOMIC_RELAXED); }
long long launch_count() { return __atomic_load_n(&g_launches, __ATOMIC_RELAXED); }

bool pdl_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = getenv("BT_NO_PDL");
    on = (e && e[0] == '1') ? 0 : 1;
  }
  return on == 1;
}

// ---------------------------------------------------------------------------
// embedder
// ---------------------------------------------------------------------------
template <typename T>
__global__ void embed_prompt_kernel(const int32_t* __restrict__ tokens, int T_len, int n, int L_B,
                                    const T* __restrict__ table, int V, int D,
                                    float* __restrict__ h, int* status, const int* __restrict__ row_pad,
                                    const int* __restrict__ row_len, int pad_id) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x;  // row = b * n + i
  const int b = r / n, i = r % n;
  const int De = D / L_B;
  // ragged batch: sequence b is row_len[b] tokens preceded by row_pad[b]
  // pad ids; blocks past its end read id 0 (their rows are never used)
  const int pad = row_pad ? row_pad[b] : 0;
  const int len = row_len ? row_len[b] : T_len;
  for (int x = threadIdx.x; x < D; x += blockDim.x) {
    const int j = x / De, e = x - j * De;
    const int src = i * L_B + j - pad;
    int tok = src < 0 ? pad_id : (src < len ? tokens[(size_t)b * T_len + src] : 0);
    if (tok < 0 || tok >= V) {
      set_status(status, ST_BAD_TOKEN);
      tok = 0;
    }
    h[(size_t)r * D + x] = to_f(table[(size_t)tok * De + e]);
  }
}

// Trailing prompt tokens (prompt length not a multiple of L_B): token i < r
// of row b, tokens[b * T_len + col0 + i], is recorded in block_tok[b, i] and
// its token-decoder embedding becomes row b * rows_per_seq + row_off + i of h.
template <typename T>
__global__ void embed_tail_kernel(const int32_t* __restrict__ tokens, int T_len, int col0, int r,
                                  int rows_per_seq, int row_off, const T* __restrict__ tok_emb, int V,
                                  int D, float* __restrict__ h, int32_t* __restrict__ block_tok, int L_B,
                                  int* status, const int* __restrict__ row_col0,
                                  const float* __restrict__ add) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x / r, i = blockIdx.x % r;
  const int c0 = row_col0 ? row_col0[b] : col0;
  int tok = tokens[(size_t)b * T_len + c0 + i];
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) set_status(status, ST_BAD_TOKEN);
    tok = 0;
  }
  if (threadIdx.x == 0) block_tok[b * L_B + i] = tok;
  float* row = h + ((size_t)b * rows_per_seq + row_off + i) * D;
  // summation injection: token i of the block also receives s_{i+1}
  const float* ad = add ? add + ((size_t)b * (L_B - 1) + i) * D : nullptr;
  for (int x = threadIdx.x; x < D; x += blockDim.x)
    row[x] = to_f(tok_emb[(size_t)tok * D + x]) + (ad ? ad[x] : 0.f);
}

template <typename T>
__global__ void ingest_kernel(const int32_t* __restrict__ src, int32_t* __restrict__ block_tok,
                              const int* __restrict__ dstate, int L_B, int V, int D,
                              int block_step, const T* __restrict__ blk_emb,
                              const T* __restrict__ tok_emb, float* __restrict__ h,
                              int* status, const float* __restrict__ add) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  const int j = dstate[1];
  int tok = src[b];
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) set_status(status, ST_BAD_TOKEN);
    tok = 0;
  }
  if (threadIdx.x == 0) block_tok[b * L_B + j] = tok;
  if (!block_step) {
    // summation injection: token j of the block also receives s_{j+1}
    const float* ad = add ? add + ((size_t)b * (L_B - 1) + j) * D : nullptr;
    for (int x = threadIdx.x; x < D; x += blockDim.x)
      h[(size_t)b * D + x] = to_f(tok_emb[(size_t)tok * D + x]) + (ad ? ad[x] : 0.f);
  } else {
    const int De = D / L_B;
    for (int x = threadIdx.x; x < D; x += blockDim.x) {
      const int jj = x / De, e = x - jj * De;
      int t = (jj == j) ? tok : block_tok[b * L_B + jj];
      if (t < 0 || t >= V) t = 0;
      h[(size_t)b * D + x] = to_f(blk_emb[(size_t)t * De + e]);
    }
  }
}

// ingest + LayerNorm of the gathered row (one CTA of 128 threads per row)
__global__ void __launch_bounds__(128)
ingest_ln_kernel(const int32_t* __restrict__ src, int32_t* __restrict__ block_tok,
                 const int* __restrict__ dstate, int L_B, int V, int D, int block_step,
                 const bf16* __restrict__ blk_emb, const bf16* __restrict__ tok_emb,
                 float* __restrict__ h, const float* __restrict__ g1, const float* __restrict__ b1,
                 const float* __restrict__ g2, const float* __restrict__ b2, float eps,
                 bf16* __restrict__ x, int* status) {
  pdl_trigger();
  pdl_wait();
  __shared__ float row[2048];
  __shared__ float red[4];
  const int b = blockIdx.x;
  const int j = dstate[1];
  int tok = src[b];
  if (tok < 0 || tok >= V) {
    if (threadIdx.x == 0) set_status(status, ST_BAD_TOKEN);
    tok = 0;
  }
  if (threadIdx.x == 0) block_tok[b * L_B + j] = tok;
  const int De = D / L_B;
  float s1 = 0.f;
  for (int c = threadIdx.x; c < D; c += 128) {
    float v;
    if (!block_step) {
      v = __bfloat162float(tok_emb[(size_t)tok * D + c]);
    } else {
      const int jj = c / De, e = c - jj * De;
      int t = (jj == j) ? tok : block_tok[b * L_B + jj];
      if (t < 0 || t >= V) t = 0;
      v = __bfloat162float(blk_emb[(size_t)t * De + e]);
    }
    row[c] = v;
    h[(size_t)b * D + c] = v;
    s1 += v;
  }
  s1 = warp_sum(s1);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s1;
  __syncthreads();
  const float mu = ((red[0] + red[1]) + (red[2] + red[3])) / (float)D;
  __syncthreads();
  float s2 = 0.f;
  for (int c = threadIdx.x; c < D; c += 128) {
    const float d = row[c] - mu;
    s2 += d * d;
  }
  s2 = warp_sum(s2);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s2;
  __syncthreads();
  const float rstd = rsqrtf(((red[0] + red[1]) + (red[2] + red[3])) / (float)D + eps);
  const bool dual = g2 != nullptr;
  bf16* o = x + (size_t)b * (dual ? 2 * D : D);
  for (int c = threadIdx.x; c < D; c += 128) {
    const float nv = (row[c] - mu) * rstd;
    o[c] = __float2bfloat16_rn(nv * g1[c] + b1[c]);
    if (dual) o[D + c] = __float2bfloat16_rn(nv * g2[c] + b2[c]);
  }
}

cudaError_t launch_ingest_ln(const int32_t* src, int32_t* block_tok, const int* dstate, int B,
                             int L_B, int V, int D, int block_step, const void* blk_emb,
                             const void* tok_emb, float* h, const float* g1, const float* b1,
                             const float* g2, const float* b2, float eps, void* x, int* status,
                             cudaStream_t s) {
  if (D > 2048) return cudaErrorInvalidValue;
  BT_LAUNCH(ingest_ln_kernel, dim3(B), dim3(128), 0, s, src, block_tok, dstate, L_B, V, D,
            block_step, (const bf16*)blk_emb, (const bf16*)tok_emb, h, g1, b1, g2, b2, eps,
            (bf16*)x, status);
  return cudaSuccess;
}

__global__ void set_state_kernel(int* dstate, int t, int L_B) {
  pdl_trigger();
  pdl_wait();
  dstate[0] = t;
  dstate[1] = t % L_B;
  dstate[2] = t / L_B;
}

__global__ void advance_kernel(int* dstate, int L_B) {
  pdl_trigger();
  pdl_wait();
  const int t = dstate[0] + 1;
  dstate[0] = t;
  dstate[1] = t % L_B;
  dstate[2] = t / L_B;
}

cudaError_t launch_embed_prompt(int dt, const int32_t* tokens, int B, int T, int L_B,
                                const void* blk_emb, int V, int D, float* h, int* status,
                                cudaStream_t s, int n_blocks, const int* row_pad, const int* row_len,
                                int pad_id) {
  const int n = n_blocks >= 0 ? n_blocks : T / L_B;
  if (B * n == 0) return cudaSuccess;
  if (dt == DT_BF16) {
    BT_LAUNCH(embed_prompt_kernel<bf16>, dim3(B * n), dim3(256), 0, s, tokens, T, n, L_B, (const bf16*)blk_emb, V, D,
              h, status, row_pad, row_len, pad_id);
  }
  else {
    BT_LAUNCH(embed_prompt_kernel<float>, dim3(B * n), dim3(256), 0, s, tokens, T, n, L_B, (const float*)blk_emb, V,
              D, h, status, row_pad, row_len, pad_id);
  }
  return cudaGetLastError();
}

cudaError_t launch_embed_tail(int dt, const int32_t* tokens, int B, int T_len, int col0, int r,
                              int rows_per_seq, int row_off, const void* tok_emb, int V, int D, float* h,
                              int32_t* block_tok, int L_B, int* status, cudaStream_t s,
                              const int* row_col0, const float* add) {
  if (B * r == 0) return cudaSuccess;
  if (dt == DT_BF16) {
    BT_LAUNCH(embed_tail_kernel<bf16>, dim3(B * r), dim3(256), 0, s, tokens, T_len, col0, r, rows_per_seq,
              row_off, (const bf16*)tok_emb, V, D, h, block_tok, L_B, status, row_col0, add);
  } else {
    BT_LAUNCH(embed_tail_kernel<float>, dim3(B * r), dim3(256), 0, s, tokens, T_len, col0, r, rows_per_seq,
              row_off, (const float*)tok_emb, V, D, h, block_tok, L_B, status, row_col0, add);
  }
  return cudaGetLastError();
}

cudaError_t launch_ingest(int dt, const int32_t* src, int32_t* block_tok, const int* dstate,
                          int B, int L_B, int V, int D, int block_step, const void* blk_emb,
                          const void* tok_emb, float* h, int* status, cudaStream_t s, const float* add) {
  if (dt == DT_BF16) {
    BT_LAUNCH(ingest_kernel<bf16>, dim3(B), dim3(256), 0, s, src, block_tok, dstate, L_B, V, D, block_step,
                                          (const bf16*)blk_emb, (const bf16*)tok_emb, h, status, add);
  }
  else {
    BT_LAUNCH(ingest_kernel<float>, dim3(B), dim3(256), 0, s, src, block_tok, dstate, L_B, V, D, block_step,
                                           (const float*)blk_emb, (const float*)tok_emb, h,
                                           status, add);
  }
  return cudaGetLastError();
}

// Context rows of the token decoder for the context-injection variants; one
// CTA per (sequence, row), threads over the D features.
//   CTX_WINDOW_SHIFT: h[b * h_rows + r] = r < (w-1)P ? ring[b][r + P]
//                     : proj[b][r - (w-1)P], r < wP (the window moves on by
//                     one context embedding, the newest projection last)
//   CTX_WINDOW_SAVE:  ring[b][r] = h[b * h_rows + r], r < wP
//   CTX_SUM_SPLIT:    h[b * h_rows] = proj[b][0] (s_0); add[b][j] =
//                     proj[b][j + 1] (s_{j+1}), j < L_B - 1
// ring [B, wP, D], proj [B, rows, D] (rows = P, or L_B for the split), fp32.
__global__ void ctx_rows_kernel(int mode, const float* __restrict__ proj, float* __restrict__ ring,
                                float* __restrict__ h, float* __restrict__ add, int nrows, int w, int P,
                                int L_B, int D, int h_rows) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x / nrows, r = blockIdx.x % nrows;
  const float* src;
  float* dst;
  if (mode == CTX_WINDOW_SHIFT) {
    const int old = (w - 1) * P;
    src = r < old ? ring + ((size_t)b * w * P + r + P) * D : proj + ((size_t)b * P + r - old) * D;
    dst = h + ((size_t)b * h_rows + r) * D;
  } else if (mode == CTX_WINDOW_SAVE) {
    src = h + ((size_t)b * h_rows + r) * D;
    dst = ring + ((size_t)b * w * P + r) * D;
  } else {
    src = proj + ((size_t)b * L_B + r) * D;
    dst = r == 0 ? h + (size_t)b * h_rows * D : add + ((size_t)b * (L_B - 1) + r - 1) * D;
  }
  for (int x = threadIdx.x; x < D; x += blockDim.x) dst[x] = src[x];
}

cudaError_t launch_ctx_rows(int mode, const float* proj, float* ring, float* h, float* add, int B, int w,
                            int P, int L_B, int D, int h_rows, cudaStream_t s) {
  const int nrows = mode == CTX_SUM_SPLIT ? L_B : w * P;
  if (B * nrows == 0) return cudaSuccess;
  BT_LAUNCH(ctx_rows_kernel, dim3(B * nrows), dim3(256), 0, s, mode, proj, ring, h, add, nrows, w, P, L_B, D,
            h_rows);
  return cudaGetLastError();
}

cudaError_t launch_set_state(int* dstate, int t, int L_B, cudaStream_t s) {
  BT_LAUNCH(set_state_kernel, dim3(1), dim3(1), 0, s, dstate, t, L_B);
  return cudaGetLastError();
}

cudaError_t launch_advance(int* dstate, int L_B, cudaStream_t s) {
  BT_LAUNCH(advance_kernel, dim3(1), dim3(1), 0, s, dstate, L_B);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// LayerNorm: one CTA (128 threads) per row, the row held in registers;
// two-pass statistics (mean, then centred variance) in fp32.
// ---------------------------------------------------------------------------
constexpr int LN_THREADS = 128;
constexpr int LN_MAXV = 4;  // float4 per thread: D <= 2048

__device__ __forceinline__ float ln_block_sum(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = (red[0] + red[1]) + (red[2] + red[3]);
  __syncthreads();
  return v;
}

// Loads row x (D floats) into v[]; returns mean and 1/sqrt(var + eps).
__device__ __forceinline__ void ln_row(const float* __restrict__ x, int D, float eps, float4* v,
                                       float& mu, float& rstd, float* red) {
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < LN_MAXV; ++u) {
    const int i = (threadIdx.x + u * LN_THREADS) * 4;
    v[u] = (i < D) ? *reinterpret_cast<const float4*>(x + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    s += (v[u].x + v[u].y) + (v[u].z + v[u].w);
  }
  mu = ln_block_sum(s, red) / (float)D;
  float q = 0.f;
#pragma unroll
  for (int u = 0; u < LN_MAXV; ++u) {
    const int i = (threadIdx.x + u * LN_THREADS) * 4;
    if (i < D) {
      const float a = v[u].x - mu, b = v[u].y - mu, c = v[u].z - mu, d = v[u].w - mu;
      q += (a * a + b * b) + (c * c + d * d);
    }
  }
  rstd = rsqrtf(ln_block_sum(q, red) / (float)D + eps);
}

template <typename T>
__device__ __forceinline__ void store4(T* out, int i, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float* out, int i, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(out + i) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16* out, int i, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + i) = u;
}

template <typename T>
__device__ __forceinline__ void ln_store(T* o, const float4& v, int i, float mu, float rstd,
                                         const float* __restrict__ g, const float* __restrict__ b) {
  const float4 ga = *reinterpret_cast<const float4*>(g + i);
  const float4 ba = *reinterpret_cast<const float4*>(b + i);
  store4<T>(o, i, (v.x - mu) * rstd * ga.x + ba.x, (v.y - mu) * rstd * ga.y + ba.y,
            (v.z - mu) * rstd * ga.z + ba.z, (v.w - mu) * rstd * ga.w + ba.w);
}

template <typename T>
__global__ void __launch_bounds__(LN_THREADS)
ln_dual_kernel(const float* __restrict__ h, int D, const float* __restrict__ g1,
               const float* __restrict__ b1, const float* __restrict__ g2,
               const float* __restrict__ b2, float eps, T* __restrict__ x1) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[4];
  const int row = blockIdx.x;
  float4 v[LN_MAXV];
  float mu, rstd;
  ln_row(h + (size_t)row * D, D, eps, v, mu, rstd, red);
  T* o = x1 + (size_t)row * 2 * D;
#pragma unroll
  for (int u = 0; u < LN_MAXV; ++u) {
    const int i = (threadIdx.x + u * LN_THREADS) * 4;
    if (i < D) {
      ln_store<T>(o, v[u], i, mu, rstd, g1, b1);
      ln_store<T>(o + D, v[u], i, mu, rstd, g2, b2);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(LN_THREADS)
ln_rows_kernel(const float* __restrict__ h, int row_step, int row_off, int D,
               const float* __restrict__ g, const float* __restrict__ b, float eps,
               T* __restrict__ out, const int* __restrict__ row_lag) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[4];
  const int r = blockIdx.x;
  float4 v[LN_MAXV];
  float mu, rstd;
  const int off = row_lag ? row_off - row_lag[r] : row_off;
  ln_row(h + ((size_t)r * row_step + off) * D, D, eps, v, mu, rstd, red);
  T* o = out + (size_t)r * D;
#pragma unroll
  for (int u = 0; u < LN_MAXV; ++u) {
    const int i = (threadIdx.x + u * LN_THREADS) * 4;
    if (i < D) ln_store<T>(o, v[u], i, mu, rstd, g, b);
  }
}

cudaError_t launch_ln_dual(int dt, const float* h, int M, int D, const float* g1,
                           const float* b1, const float* g2, const float* b2, float eps,
                           void* x1, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  if (D > LN_THREADS * 4 * LN_MAXV || (D % 4)) return cudaErrorInvalidValue;
  if (dt == DT_BF16)
    BT_LAUNCH(ln_dual_kernel<bf16>, dim3(M), dim3(LN_THREADS), 0, s, h, D, g1, b1, g2, b2, eps, (bf16*)x1);
  else
    BT_LAUNCH(ln_dual_kernel<float>, dim3(M), dim3(LN_THREADS), 0, s, h, D, g1, b1, g2, b2, eps, (float*)x1);
  return cudaGetLastError();
}

cudaError_t launch_ln_rows(int dt, const float* h, int R, int row_step, int row_off, int D,
                           const float* g, const float* b, float eps, void* out, cudaStream_t s,
                           const int* row_lag) {
  if (R == 0) return cudaSuccess;
  if (D > LN_THREADS * 4 * LN_MAXV || (D % 4)) return cudaErrorInvalidValue;
  if (dt == DT_BF16)
    BT_LAUNCH(ln_rows_kernel<bf16>, dim3(R), dim3(LN_THREADS), 0, s, h, row_step, row_off, D, g, b, eps,
              (bf16*)out, row_lag);
  else
    BT_LAUNCH(ln_rows_kernel<float>, dim3(R), dim3(LN_THREADS), 0, s, h, row_step, row_off, D, g, b, eps,
              (float*)out, row_lag);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// rotary table + rotary/append
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(float2* tab, int n_pos, int half, double base) {
  pdl_trigger();
  pdl_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_pos * half) return;
  const int p = idx / half, i = idx - p * half;
  // angle = p * base^(-2i/rot), rot = 2*half
  const double inv = pow(base, -(double)(2 * i) / (double)(2 * half));
  double sn, cs;
  sincos((double)p * inv, &sn, &cs);
  tab[idx] = make_float2((float)cs, (float)sn);
}

cudaError_t launch_rope_table(float2* tab, int n_pos, int rot, float base, cudaStream_t s) {
  const int half = rot / 2;
  if (half == 0 || n_pos == 0) return cudaSuccess;
  const int total = n_pos * half;
  BT_LAUNCH(rope_table_kernel, dim3((total + 255) / 256), dim3(256), 0, s, tab, n_pos, half, (double)base);
  return cudaGetLastError();
}

__device__ __forceinline__ uint2 pack_bf16x4_ew(float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  return u;
}

template <typename T>
__global__ void rope_append_kernel(const T* __restrict__ qkv, int D, int H, int Hk, int rot,
                                   const float2* __restrict__ tab, PosSpec ps,
                                   T* __restrict__ q_out, T* __restrict__ kc,
                                   T* __restrict__ vc, int cap, T* __restrict__ vt, int vt_ld) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x;
  const int d = D / H;
  const int half = rot >> 1;
  const int b = m / ps.rows_per_seq;
  const int pos = pos_base(ps, b) + (m - b * ps.rows_per_seq);
  // row: q (H heads) | k (Hk heads) | v (Hk heads)
  const int Dk = Hk * d, W = D + 2 * Dk;
  const T* row = qkv + (size_t)m * W;
  for (int x = threadIdx.x; x < W; x += blockDim.x) {
    const int part = x < D ? 0 : (x < D + Dk ? 1 : 2);  // 0 q, 1 k, 2 v
    const int c = part == 0 ? x : (part == 1 ? x - D : x - D - Dk);
    const int hh = c / d, e = c - hh * d;
    float v = to_f(row[x]);
    if (part < 2 && e < rot) {
      const int i = (e < half) ? e : e - half;
      const float2 cs = tab[(size_t)pos * half + i];
      if (e < half) v = v * cs.x - to_f(row[x + half]) * cs.y;
      else v = v * cs.x + to_f(row[x - half]) * cs.y;
    }
    if (part == 0) {
      q_out[(size_t)m * D + c] = from_f<T>(v);
    } else {
      T* cache = (part == 1) ? kc : vc;
      cache[(((size_t)b * Hk + hh) * cap + pos) * d + e] = from_f<T>(v);
      if (part == 2 && vt) vt[(((size_t)b * Hk + hh) * d + e) * vt_ld + pos] = from_f<T>(v);
    }
  }
}

// The same in 16-byte pieces (bf16, d and rot / 2 multiples of 8): one
// thread per 8 consecutive features of a row, so that part, head and
// position are computed once per piece and every access is a 16-byte load
// or store; the rotate-half partner of a piece inside the rotary span is the
// aligned piece rot / 2 features away in the same head.
__global__ void rope_append_vec_kernel(const bf16* __restrict__ qkv, int M, int D, int H, int Hk, int rot,
                                       const float2* __restrict__ tab, PosSpec ps, bf16* __restrict__ q_out,
                                       bf16* __restrict__ kc, bf16* __restrict__ vc, int cap) {
  pdl_trigger();
  pdl_wait();
  const int d = D / H;
  const int half = rot >> 1;
  const int Dk = Hk * d, W = D + 2 * Dk;
  const int pieces = W / 8;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)M * pieces) return;
  const int m = (int)(idx / pieces);
  const int x = (int)(idx - (long long)m * pieces) * 8;
  const int b = m / ps.rows_per_seq;
  const int pos = pos_base(ps, b) + (m - b * ps.rows_per_seq);
  const bf16* row = qkv + (size_t)m * W;
  const int part = x < D ? 0 : (x < D + Dk ? 1 : 2);
  const int c = part == 0 ? x : (part == 1 ? x - D : x - D - Dk);
  const int hh = c / d, e = c - hh * d;
  float v[8];
  unpack16(*reinterpret_cast<const uint4*>(row + x), v, (const bf16*)nullptr);
  if (part < 2 && e < rot) {
    const bool lo = e < half;
    float pv[8];
    unpack16(*reinterpret_cast<const uint4*>(row + (lo ? x + half : x - half)), pv, (const bf16*)nullptr);
    const int i0 = lo ? e : e - half;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 cs = tab[(size_t)pos * half + i0 + j];
      v[j] = lo ? v[j] * cs.x - pv[j] * cs.y : v[j] * cs.x + pv[j] * cs.y;
    }
  }
  const uint2 lo4 = pack_bf16x4_ew(v[0], v[1], v[2], v[3]), hi4 = pack_bf16x4_ew(v[4], v[5], v[6], v[7]);
  const uint4 out = make_uint4(lo4.x, lo4.y, hi4.x, hi4.y);
  if (part == 0) {
    *reinterpret_cast<uint4*>(q_out + (size_t)m * D + c) = out;
  } else {
    bf16* cache = part == 1 ? kc : vc;
    *reinterpret_cast<uint4*>(cache + (((size_t)b * Hk + hh) * cap + pos) * d + e) = out;
  }
}

// V^T [(b*Hk + h)*d + e][pos] for positions p0 + [0, 64) of one (sequence,
// key/value head): the tile goes through shared memory so that both the
// reads (along the head dims of a row) and the writes (along positions) are
// coalesced. Rows of a sequence are consecutive, W wide, V at column voff;
// row i has position pos0 + i.
template <typename T>
__global__ void __launch_bounds__(256)
vt_write_kernel(const T* __restrict__ qkv, int W, int voff, int H, int d, int rows, int pos0,
                T* __restrict__ vt, int vt_ld) {
  pdl_trigger();
  pdl_wait();
  __shared__ float tile[64][65];
  const int bh = blockIdx.y, b = bh / H, h = bh - b * H;
  const int i0 = blockIdx.x * 64;
  const int ec = d < 64 ? d : 64;
  for (int e0 = 0; e0 < d; e0 += ec) {
    for (int x = threadIdx.x; x < 64 * ec; x += blockDim.x) {
      const int ii = x / ec, e = x - ii * ec;
      const int i = i0 + ii;
      tile[ii][e] = (i < rows) ? to_f(qkv[((size_t)b * rows + i) * W + voff + h * d + e0 + e]) : 0.f;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < 64 * ec; x += blockDim.x) {
      const int e = x / 64, ii = x - e * 64;
      const int i = i0 + ii;
      if (i < rows) vt[((size_t)bh * d + e0 + e) * vt_ld + pos0 + i] = from_f<T>(tile[ii][e]);
    }
    __syncthreads();
  }
}

cudaError_t launch_rope_append(int dt, const void* qkv, int M, int D, int H, int rot,
                               const float2* rope_tab, PosSpec pos, void* q_out, void* k_cache,
                               void* v_cache, int cap, cudaStream_t s, void* vt, int vt_ld, int Hk) {
  if (M == 0) return cudaSuccess;
  if (Hk <= 0) Hk = H;
  if (H % Hk) return cudaErrorInvalidValue;
  // V^T is written for positions known on the host (prefill) only
  if (vt && pos.mode != POS_ZERO) return cudaErrorInvalidValue;
  const int dh = D / H;
  if (dt == DT_BF16 && dh % 8 == 0 && (rot / 2) % 8 == 0) {
    const long long n = (long long)M * ((D + 2 * Hk * dh) / 8);
    BT_LAUNCH(rope_append_vec_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, (const bf16*)qkv, M, D, H,
              Hk, rot, rope_tab, pos, (bf16*)q_out, (bf16*)k_cache, (bf16*)v_cache, cap);
  } else if (dt == DT_BF16) {
    BT_LAUNCH(rope_append_kernel<bf16>, dim3(M), dim3(256), 0, s, (const bf16*)qkv, D, H, Hk, rot, rope_tab, pos,
                                               (bf16*)q_out, (bf16*)k_cache, (bf16*)v_cache, cap, (bf16*)nullptr, 0);
  }
  else {
    BT_LAUNCH(rope_append_kernel<float>, dim3(M), dim3(256), 0, s, (const float*)qkv, D, H, Hk, rot, rope_tab, pos,
                                                (float*)q_out, (float*)k_cache, (float*)v_cache,
                                                cap, (float*)nullptr, 0);
  }
  if (vt) {
    const int rows = pos.rows_per_seq, B = M / rows, d = D / H;
    const int W = D + 2 * Hk * d, voff = D + Hk * d;
    const dim3 grid((rows + 63) / 64, B * Hk);
    if (dt == DT_BF16)
      BT_LAUNCH(vt_write_kernel<bf16>, grid, dim3(256), 0, s, (const bf16*)qkv, W, voff, Hk, d, rows, pos.add,
                (bf16*)vt, vt_ld);
    else
      BT_LAUNCH(vt_write_kernel<float>, grid, dim3(256), 0, s, (const float*)qkv, W, voff, Hk, d, rows, pos.add,
                (float*)vt, vt_ld);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// argmax over the vocabulary (lowest id among ties)
// ---------------------------------------------------------------------------
__global__ void argmax_kernel(const float* __restrict__ logits, int V, int ld,
                              int32_t* __restrict__ next) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  const float* z = logits + (size_t)b * ld;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    const float x = z[v];
    if (x > best || (x == best && v < bi)) { best = x; bi = v; }
  }
  __shared__ float sv[32];
  __shared__ int si[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sv[w] = best; si[w] = bi; }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    best = lane < nw ? sv[lane] : -INFINITY;
    bi = lane < nw ? si[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
    }
    if (lane == 0) next[b] = (bi == 0x7fffffff) ? 0 : bi;
  }
}

cudaError_t launch_argmax(const float* logits, int B, int V, int ld, int32_t* next,
                          cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  BT_LAUNCH(argmax_kernel, dim3(B), dim3(1024), 0, s, logits, V, ld, next);
  return cudaGetLastError();
}

__global__ void argmax_reduce_kernel(const float2* __restrict__ part, int n_tiles, int M,
                                     int32_t* __restrict__ next, int* dstate, int L_B) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int t = threadIdx.x; t < n_tiles; t += blockDim.x) {
    const float2 p = part[(size_t)t * M + m];
    const int i = __float_as_int(p.y);
    if (p.x > best || (p.x == best && i < bi)) { best = p.x; bi = i; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
  }
  __shared__ float sv[8];
  __shared__ int si[8];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sv[w] = best; si[w] = bi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k)
      if (sv[k] > best || (sv[k] == best && si[k] < bi)) { best = sv[k]; bi = si[k]; }
    next[m] = (bi == 0x7fffffff) ? 0 : bi;
    if (dstate && m == 0) {  // the step is over: advance the position
      const int t = dstate[0] + 1;
      dstate[0] = t;
      dstate[1] = t % L_B;
      dstate[2] = t / L_B;
    }
  }
}

cudaError_t launch_argmax_reduce(const float2* part, int n_tiles, int M, int32_t* next,
                                 cudaStream_t s, int* dstate, int L_B) {
  if (M == 0) return cudaSuccess;
  BT_LAUNCH(argmax_reduce_kernel, dim3(M), dim3(256), 0, s, part, n_tiles, M, next, dstate, L_B);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// conversions used when the model is created
// ---------------------------------------------------------------------------
template <typename T>
__global__ void convert_kernel(const T* __restrict__ src, float* __restrict__ dst, size_t n) {
  pdl_trigger();
  pdl_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = to_f(src[i]);
}

template <typename T>
__global__ void add_kernel(const T* __restrict__ a, const T* __restrict__ b,
                           float* __restrict__ dst, size_t n) {
  pdl_trigger();
  pdl_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = to_f(a[i]) + to_f(b[i]);
}

cudaError_t launch_convert_to_f32(int dt, const void* src, float* dst, size_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int grid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  if (dt == DT_BF16) BT_LAUNCH(convert_kernel<bf16>, dim3(grid), dim3(256), 0, s, (const bf16*)src, dst, n);
  else BT_LAUNCH(convert_kernel<float>, dim3(grid), dim3(256), 0, s, (const float*)src, dst, n);
  return cudaGetLastError();
}

cudaError_t launch_add_to_f32(int dt, const void* a, const void* b, float* dst, size_t n,
                              cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int grid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  if (dt == DT_BF16) BT_LAUNCH(add_kernel<bf16>, dim3(grid), dim3(256), 0, s, (const bf16*)a, (const bf16*)b, dst, n);
  else BT_LAUNCH(add_kernel<float>, dim3(grid), dim3(256), 0, s, (const float*)a, (const float*)b, dst, n);
  return cudaGetLastError();
}

}  // namespace bt
