// attention.cu -- attention kernels of the Block Transformer (sm_100a).
//
// * Block-decoder decode attention: one new block per sequence attends over
//   its n cached block entries ("Block Transformer: Global-to-Local Language
//   Modeling for Fast Inference", §3.4 "The Block Decoder": the KV cache is
//   L_B times shorter and read once per L_B tokens). Split-K flash decoding:
//   each CTA streams one chunk of K and V rows of one (sequence, head) into
//   shared memory with a 1-D bulk copy, computes chunk-local softmax
//   statistics (m, l) and o, and the last CTA of a (sequence, head) merges
//   the chunks: o = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s. No CTA
//   waits for another (last-arriver merge through an atomic counter).
// * Token-decoder local attention: each new row attends over at most
//   P + L_B - 1 rows of its own block (§3.4 "The Token Decoder"); one warp per
//   (sequence, head, query row), online softmax in registers.
// * Block-decoder prefill attention: causal over the prompt's blocks.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace bt {

// ---------------------------------------------------------------------------
// split-K decode attention
// ---------------------------------------------------------------------------
template <typename T, int DH>
struct DecCfg {
  static constexpr int ROW_BYTES = DH * (int)sizeof(T);
  static constexpr int CHUNK = 16384 / ROW_BYTES;        // rows per split (16 KB of K)
  static constexpr int TPR = ROW_BYTES / 16;             // threads per row, 16 B each
  static constexpr int THREADS = 128;
  static constexpr int RPP = THREADS / TPR;              // rows per pass
  static constexpr int EPT = 16 / (int)sizeof(T);        // elements per thread
  static constexpr int SMEM = 2 * CHUNK * ROW_BYTES + CHUNK * 4 + RPP * DH * 4;
  static_assert(TPR >= 1 && TPR <= 32 && (32 % TPR) == 0, "row split");
};

__device__ __forceinline__ float block_reduce_max128(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  v = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return v;
}
__device__ __forceinline__ float block_reduce_sum128(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  v = (red[0] + red[1]) + (red[2] + red[3]);
  __syncthreads();
  return v;
}

template <typename T, int DH>
__global__ void __launch_bounds__(128)
attn_decode_kernel(const T* __restrict__ q, int ldq, const T* __restrict__ kc,
                   const T* __restrict__ vc, int H, int cap, PosSpec kvlen, T* __restrict__ out,
                   int ld_out, float* __restrict__ part, int* __restrict__ counters,
                   int max_splits, int* status, float qscale) {
  pdl_trigger();
  pdl_wait();
  using C = DecCfg<T, DH>;
  const int pair = blockIdx.x;  // b * H + h
  const int split = blockIdx.y;
  const int b = pair / H, h = pair - b * H;
  const int n = pos_base(kvlen) + 1;
  const int nsplit = (n + C::CHUNK - 1) / C::CHUNK;
  if (split >= nsplit) return;
  const int r0 = split * C::CHUNK;
  const int rows = min(C::CHUNK, n - r0);

  extern __shared__ __align__(128) uint8_t smem[];
  T* sK = reinterpret_cast<T*>(smem);
  T* sV = reinterpret_cast<T*>(smem + C::CHUNK * C::ROW_BYTES);
  float* sS = reinterpret_cast<float*>(smem + 2 * C::CHUNK * C::ROW_BYTES);
  float* sO = sS + C::CHUNK;
  __shared__ __align__(8) uint64_t bar;
  __shared__ float red[4];
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const size_t base = ((size_t)pair * cap + r0) * DH;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    const uint32_t bytes = (uint32_t)rows * C::ROW_BYTES;
    mbar_arrive_expect_tx(&bar, 2 * bytes);
    bulk_g2s(sK, kc + base, bytes, &bar);
    bulk_g2s(sV, vc + base, bytes, &bar);
  }

  // this thread's slice of q (16 bytes), scaled by log2(e)/sqrt(d)
  const int g = tid / C::TPR;
  const int e0 = (tid % C::TPR) * C::EPT;
  float qf[C::EPT];
  {
    const uint4 u = *reinterpret_cast<const uint4*>(q + (size_t)b * ldq + h * DH + e0);
    unpack16(u, qf, (const T*)nullptr);
#pragma unroll
    for (int i = 0; i < C::EPT; ++i) qf[i] *= qscale;
  }

  if (!mbar_wait_bounded(&bar, 0, status)) {
    mbar_wait_bounded(&bar, 0, status);  // second bounded wait for the copies in flight
    return;
  }

  // scores s_r = q . k_r (log2 domain). The trip count is the same for every
  // thread of the CTA (rows and RPP are uniform) so the full-warp shuffles
  // below never see a partial warp; rows past the end contribute nothing.
  for (int rb = 0; rb < rows; rb += C::RPP) {
    const int r = rb + g;
    const bool valid = r < rows;
    float s = 0.f;
    if (valid) {
      const uint4 u = *reinterpret_cast<const uint4*>(sK + r * DH + e0);
      float kf[C::EPT];
      unpack16(u, kf, (const T*)nullptr);
#pragma unroll
      for (int i = 0; i < C::EPT; ++i) s = fmaf(qf[i], kf[i], s);
    }
#pragma unroll
    for (int o = C::TPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (valid && (tid % C::TPR) == 0) sS[r] = s;
  }
  __syncthreads();
  float mx = -FLT_MAX;
  for (int r = tid; r < rows; r += C::THREADS) mx = fmaxf(mx, sS[r]);
  const float M = block_reduce_max128(mx, red);
  float l = 0.f;
  for (int r = tid; r < rows; r += C::THREADS) {
    const float p = exp2f(sS[r] - M);
    sS[r] = p;
    l += p;
  }
  const float L = block_reduce_sum128(l, red);  // contains __syncthreads: sS visible

  float of[C::EPT];
#pragma unroll
  for (int i = 0; i < C::EPT; ++i) of[i] = 0.f;
  for (int r = g; r < rows; r += C::RPP) {
    const float p = sS[r];
    const uint4 u = *reinterpret_cast<const uint4*>(sV + r * DH + e0);
    float vf[C::EPT];
    unpack16(u, vf, (const T*)nullptr);
#pragma unroll
    for (int i = 0; i < C::EPT; ++i) of[i] = fmaf(p, vf[i], of[i]);
  }
#pragma unroll
  for (int i = 0; i < C::EPT; ++i) sO[g * DH + e0 + i] = of[i];
  __syncthreads();
  float o_d = 0.f;
  if (tid < DH) {
    for (int gg = 0; gg < C::RPP; ++gg) o_d += sO[gg * DH + tid];
  }

  if (nsplit == 1) {
    if (tid < DH) out[(size_t)b * ld_out + h * DH + tid] = from_f<T>(o_d / L);
    return;
  }
  float* my = part + ((size_t)pair * max_splits + split) * (DH + 2);
  if (tid < DH) my[2 + tid] = o_d;
  if (tid == 0) { my[0] = M; my[1] = L; }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&counters[pair], 1) == nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* pp = part + (size_t)pair * max_splits * (DH + 2);
  float Mg = -FLT_MAX;
  for (int s = 0; s < nsplit; ++s) Mg = fmaxf(Mg, __ldcg(pp + (size_t)s * (DH + 2)));
  float Lg = 0.f, og = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float* ps = pp + (size_t)s * (DH + 2);
    const float w = exp2f(__ldcg(ps) - Mg);
    Lg = fmaf(w, __ldcg(ps + 1), Lg);
    if (tid < DH) og = fmaf(w, __ldcg(ps + 2 + tid), og);
  }
  if (tid < DH) out[(size_t)b * ld_out + h * DH + tid] = from_f<T>(og / Lg);
  if (tid == 0) counters[pair] = 0;
}

template <typename T>
static int dec_chunk(int d) {
  return 16384 / (d * (int)sizeof(T));
}

int attn_decode_max_splits(int d, int cap, int dt) {
  const int chunk = dt == DT_BF16 ? dec_chunk<bf16>(d) : dec_chunk<float>(d);
  return (cap + chunk - 1) / chunk;
}

size_t attn_decode_scratch_bytes(int B, int H, int d, int cap, int dt) {
  const size_t ms = (size_t)attn_decode_max_splits(d, cap, dt);
  const size_t part = (size_t)B * H * ms * (d + 2) * sizeof(float);
  const size_t part_al = (part + 255) & ~(size_t)255;
  return part_al + (size_t)B * H * sizeof(int);
}

template <typename T, int DH>
static cudaError_t launch_dec(const void* q, int ldq, const void* kc, const void* vc, int B,
                              int H, int cap, PosSpec kvlen, void* out, int ld_out,
                              void* scratch, int* status, cudaStream_t s) {
  using C = DecCfg<T, DH>;
  const int ms = (cap + C::CHUNK - 1) / C::CHUNK;
  const size_t part = (size_t)B * H * ms * (DH + 2) * sizeof(float);
  float* partp = reinterpret_cast<float*>(scratch);
  int* counters = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(scratch) +
                                         ((part + 255) & ~(size_t)255));
  dim3 grid(B * H, ms);
  const float qscale = 1.4426950408889634f / sqrtf((float)DH);
  BT_LAUNCH(attn_decode_kernel<T, DH>, dim3(grid), dim3(C::THREADS), C::SMEM, s, 
      (const T*)q, ldq, (const T*)kc, (const T*)vc, H, cap, kvlen, (T*)out, ld_out, partp,
      counters, ms, status, qscale);
  return cudaGetLastError();
}

cudaError_t launch_attn_decode(int dt, const void* q, int ldq, const void* k_cache,
                               const void* v_cache, int B, int H, int d, int cap,
                               PosSpec kvlen, void* out, int ld_out, void* scratch,
                               int* status, cudaStream_t s) {
  if (B * H == 0) return cudaSuccess;
#define BT_DEC(T, DHV) \
  return launch_dec<T, DHV>(q, ldq, k_cache, v_cache, B, H, cap, kvlen, out, ld_out, scratch, status, s)
  if (dt == DT_BF16) {
    if (d == 64) BT_DEC(bf16, 64);
    if (d == 128) BT_DEC(bf16, 128);
    if (d == 32) BT_DEC(bf16, 32);
  } else {
    if (d == 32) BT_DEC(float, 32);
    if (d == 64) BT_DEC(float, 64);
    if (d == 128) BT_DEC(float, 128);
  }
#undef BT_DEC
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// small causal attention: one warp per (sequence, head, query)
// ---------------------------------------------------------------------------
template <typename T, int DH>
__global__ void attn_small_kernel(const T* __restrict__ q, int ldq, const T* __restrict__ kc,
                                  const T* __restrict__ vc, int B, int H, int cap, PosSpec qpos,
                                  T* __restrict__ out, int ld_out, float scale) {
  pdl_trigger();
  pdl_wait();
  constexpr int EPL = DH / 32;  // elements per lane
  const int warp = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int Q = qpos.rows_per_seq;
  if (warp >= B * Q * H) return;
  const int h = warp % H;
  const int m = warp / H;  // query row = b * Q + i
  const int b = m / Q, i = m - b * Q;
  const int pos = pos_base(qpos) + i;
  float qf[EPL], of[EPL];
#pragma unroll
  for (int x = 0; x < EPL; ++x) {
    qf[x] = to_f(q[(size_t)m * ldq + h * DH + lane + 32 * x]) * scale;
    of[x] = 0.f;
  }
  const T* kb = kc + ((size_t)b * H + h) * cap * DH;
  const T* vb = vc + ((size_t)b * H + h) * cap * DH;
  float mrun = -FLT_MAX, l = 0.f;
  for (int j = 0; j <= pos; ++j) {
    float s = 0.f;
#pragma unroll
    for (int x = 0; x < EPL; ++x) s = fmaf(qf[x], to_f(kb[(size_t)j * DH + lane + 32 * x]), s);
    s = warp_sum(s);
    const float mn = fmaxf(mrun, s);
    const float c = exp2f(mrun - mn), p = exp2f(s - mn);
    l = l * c + p;
#pragma unroll
    for (int x = 0; x < EPL; ++x) of[x] = of[x] * c + p * to_f(vb[(size_t)j * DH + lane + 32 * x]);
    mrun = mn;
  }
#pragma unroll
  for (int x = 0; x < EPL; ++x) out[(size_t)m * ld_out + h * DH + lane + 32 * x] = from_f<T>(of[x] / l);
}

cudaError_t launch_attn_small(int dt, const void* q, int ldq, const void* k_cache,
                              const void* v_cache, int B, int H, int d, int cap, PosSpec qpos,
                              void* out, int ld_out, cudaStream_t s) {
  const int warps = B * qpos.rows_per_seq * H;
  if (warps == 0) return cudaSuccess;
  const int grid = (warps + 3) / 4;
  const float scale = 1.4426950408889634f / sqrtf((float)d);
#define BT_SMALL(T, DHV)                                                                      \
  BT_LAUNCH(attn_small_kernel<T, DHV>, dim3(grid), dim3(128), 0, s, (const T*)q, ldq, (const T*)k_cache,        \
                                                  (const T*)v_cache, B, H, cap, qpos, (T*)out, \
                                                  ld_out, scale);                             \
  return cudaGetLastError()
  if (dt == DT_BF16) {
    if (d == 32) { BT_SMALL(bf16, 32); }
    if (d == 64) { BT_SMALL(bf16, 64); }
    if (d == 128) { BT_SMALL(bf16, 128); }
  } else {
    if (d == 32) { BT_SMALL(float, 32); }
    if (d == 64) { BT_SMALL(float, 64); }
    if (d == 128) { BT_SMALL(float, 128); }
  }
#undef BT_SMALL
  return cudaErrorInvalidValue;
}

// Prefill causal attention (interim: the warp-per-query kernel over all n
// positions; query i of a sequence sees cache entries 0..i).
cudaError_t launch_attn_prefill(int dt, const void* q, int ldq, const void* k_cache,
                                const void* v_cache, int B, int H, int d, int cap, int n,
                                void* out, int ld_out, cudaStream_t s) {
  PosSpec p{nullptr, POS_ZERO, 0, n};
  return launch_attn_small(dt, q, ldq, k_cache, v_cache, B, H, d, cap, p, out, ld_out, s);
}

}  // namespace bt
