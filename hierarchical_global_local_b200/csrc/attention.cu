// attention.cu -- attention kernels of the Block Transformer (sm_100a).
//
// * Block-decoder decode attention: one new block per sequence attends over
//   its n cached block entries ("Block Transformer: Global-to-Local Language
//   Modeling for Fast Inference", §3.4 "The Block Decoder": the KV cache is
//   L_B times shorter and read once per L_B tokens). Flash decoding: a
//   persistent grid streams chunks of K and V rows into shared memory with
//   1-D bulk copies and keeps an online softmax (m, l, o). With enough
//   (sequence, head) pairs each CTA takes whole pairs; with few, a pair's
//   chunks are split over several CTAs and the last of them merges the
//   partials: o = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s. No CTA
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
// A work unit is one (sequence, head) pair and a contiguous range of its
// cached rows, streamed in CHUNK-row pieces (4 KB of K + 4 KB of V) through a
// STAGES-deep ring of 1-D bulk copies, with an online softmax across chunks.
// Pairs are split into several units only when there are too few pairs to
// keep every SM busy; split units are merged by the last one to finish.
template <typename T, int DH>
struct DecCfg {
  static constexpr int ROW_BYTES = DH * (int)sizeof(T);
  static constexpr int CHUNK = 4096 / ROW_BYTES;         // rows per chunk (4 KB of K)
  static constexpr int STAGES = 4;
  static constexpr int TPR = ROW_BYTES / 16;             // threads per row, 16 B each
  static constexpr int CWARPS = 4;                       // consumer warps
  static constexpr int THREADS = (CWARPS + 1) * 32;      // + one producer warp
  static constexpr int GROUPS = CWARPS * 32 / TPR;       // row groups (each owns rows)
  static constexpr int EPT = 16 / (int)sizeof(T);        // elements per thread
  static constexpr int SMEM = STAGES * 2 * CHUNK * ROW_BYTES + CWARPS * (DH + 2) * 4;
  static_assert(TPR >= 1 && TPR <= 32 && (32 % TPR) == 0, "row split");
  static_assert(DH <= CWARPS * 32, "one thread per output dim in the final reduction");
};

constexpr int DEC_UNITS_SLACK = ATTN_DECODE_MAX_CTAS;  // partial slots in the scratch (grid cap)

// resident CTAs per SM: 6 x (32 KB ring + the combine slots) of shared
// memory, 6 x 160 threads x at most 64 registers (the launch bound)
constexpr int DEC_CTAS_PER_SM = 6;

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

// Two partitions of the flattened list of (pair, chunk) work, the copy ring
// of a CTA running straight across pair boundaries:
// * whole pairs (whole = 1, when there are at least half as many pairs as
//   resident CTAs): CTA c of G handles pairs [floor(c*pairs/G),
//   floor((c+1)*pairs/G)), so no pair is split and no CTA merges partials
//   or waits on a counter at its end;
// * stream-K (whole = 0): CTA c of G handles chunks [floor(c*T/G),
//   floor((c+1)*T/G)) of the T = pairs * nch chunks. A pair whose chunks
//   span several CTAs gets one partial (m, l, o) from each; the last to
//   finish (atomic counter, no waiting) merges them in CTA order.
__device__ __forceinline__ int dec_owner(long long x, int G, long long T) {
  // the CTA whose chunk range contains chunk x
  return (int)(((x + 1) * G + T - 1) / T) - 1;
}

// barrier among the consumer warps only (the producer warp may still be
// waiting for a free stage, or gone)
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <typename T, int DH>
__global__ void __launch_bounds__(DecCfg<T, DH>::THREADS, DEC_CTAS_PER_SM)
attn_decode_kernel(const T* __restrict__ q, int ldq, const T* __restrict__ kc,
                   const T* __restrict__ vc, int pairs, int H, int cap, PosSpec kvlen,
                   T* __restrict__ out, int ld_out, float* __restrict__ part,
                   int* __restrict__ counters, int* status, float qscale, int qpk, int whole) {
  pdl_trigger();
  pdl_wait();
  using C = DecCfg<T, DH>;
  // chunks per pair from the longest sequence; a shorter sequence of a
  // ragged batch (kvlen.row_lag) has empty trailing chunks
  const int n = pos_base(kvlen) + 1;
  const int nch = (n + C::CHUNK - 1) / C::CHUNK;
  const long long Ttot = (long long)pairs * nch;
  // effective grid <= chunks (stream-K) or <= pairs (whole pairs), so that
  // every CTA's range is non-empty and the CTAs sharing a pair are consecutive
  const long long units = whole ? (long long)pairs : Ttot;
  const int G = (int)((long long)gridDim.x < units ? (long long)gridDim.x : units);
  const int c = blockIdx.x;
  if (c >= G) return;
  const long long x0 = whole ? (long long)c * pairs / G * nch : (long long)c * Ttot / G;
  const long long x1 = whole ? (long long)(c + 1) * pairs / G * nch : (long long)(c + 1) * Ttot / G;
  const int nc = (int)(x1 - x0);

  extern __shared__ __align__(128) uint8_t smem[];
  T* sKV = reinterpret_cast<T*>(smem);  // [STAGES][K chunk | V chunk]
  float* sR = reinterpret_cast<float*>(smem + C::STAGES * 2 * C::CHUNK * C::ROW_BYTES);
  __shared__ __align__(8) uint64_t full[C::STAGES], empty[C::STAGES];
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::CWARPS);
    }
    fence_mbar_init();
  }
  __syncthreads();

  bool ok = true;
  if (warp == C::CWARPS) {
    // ---- producer warp: one lane streams chunks x0 .. x1 through the ring ----
    if (lane == 0) {
      for (int i = 0; i < nc; ++i) {
        const int s = i % C::STAGES;
        if (i >= C::STAGES) mbar_wait_bounded(&empty[s], ((i / C::STAGES) + 1) & 1, status);
        const long long x = x0 + i;
        const int pr = (int)(x / nch), ci = (int)(x - (long long)pr * nch);
        const int r0 = ci * C::CHUNK;
        const int np = pos_base(kvlen, pr / H) + 1;  // this pair's entries
        const int rows = max(0, min(C::CHUNK, np - r0));
        const uint32_t bytes = (uint32_t)rows * C::ROW_BYTES;
        // key/value head of query head h: h / qpk (grouped-query attention;
        // the qpk query heads of one key/value head are consecutive pairs, so
        // their repeated reads of it come from L2)
        const int kvp = (pr / H) * (H / qpk) + (pr % H) / qpk;
        const size_t off = ((size_t)kvp * cap + r0) * DH;
        T* dk = sKV + (size_t)s * 2 * C::CHUNK * DH;
        mbar_arrive_expect_tx(&full[s], 2 * bytes);
        if (bytes) {
          bulk_g2s(dk, kc + off, bytes, &full[s]);
          bulk_g2s(dk + C::CHUNK * DH, vc + off, bytes, &full[s]);
        }
      }
    }
    return;  // the copies complete on the mbarriers; consumers sync among themselves
  }

  // ---- consumers: row group g (TPR lanes) owns rows g, g + GROUPS, ... of
  // every chunk, with its own running max, sum and output slice ----
  const int g = tid / C::TPR;  // valid for consumer warps
  const int e0 = (tid % C::TPR) * C::EPT;
  const int first_pair = (int)(x0 / nch);
  // q of the CTA's first pair; the next pair's q is loaded while the current
  // pair is combined
  uint4 qn;
  {
    const int b = first_pair / H, h = first_pair - b * H;
    qn = *reinterpret_cast<const uint4*>(q + (size_t)b * ldq + h * DH + e0);
  }
  int i = 0;
  for (int pr = first_pair; i < nc; ++pr) {
    const long long pend = (long long)(pr + 1) * nch;
    const int cnt = (int)((pend < x1 ? pend : x1) - (x0 + i));
    const int b = pr / H, h = pr - b * H;
    const int np = pos_base(kvlen, b) + 1;  // this pair's entries (<= n)
    float M = -FLT_MAX, l = 0.f;
    float of[C::EPT];
#pragma unroll
    for (int e = 0; e < C::EPT; ++e) of[e] = 0.f;
    {
      float qf[C::EPT];
      unpack16(qn, qf, (const T*)nullptr);
#pragma unroll
      for (int e = 0; e < C::EPT; ++e) qf[e] *= qscale;
      for (int k = 0; k < cnt; ++k) {
        const int ii = i + k;
        const int s = ii % C::STAGES;
        if (!mbar_wait_bounded(&full[s], (ii / C::STAGES) & 1, status)) ok = false;
        const T* sK = sKV + (size_t)s * 2 * C::CHUNK * DH;
        const T* sV = sK + C::CHUNK * DH;
        const long long x = x0 + ii;
        const int rows = min(C::CHUNK, np - (int)(x - (long long)pr * nch) * C::CHUNK);
        // a chunk holds 2 * GROUPS rows: row group g takes rows g and
        // g + GROUPS and folds both into its softmax with one rescale. All
        // lanes run the shuffles (an empty row scores -FLT_MAX, weight 0).
        static_assert(C::CHUNK == 2 * C::GROUPS, "two rows per row group and chunk");
        {
          const int r0 = g, r1 = g + C::GROUPS;
          const bool v0 = r0 < rows, v1 = r1 < rows;
          float s0 = 0.f, s1 = 0.f;
          float vf0[C::EPT], vf1[C::EPT];
          if (v0) {
            float kf[C::EPT];
            unpack16(*reinterpret_cast<const uint4*>(sK + r0 * DH + e0), kf, (const T*)nullptr);
            unpack16(*reinterpret_cast<const uint4*>(sV + r0 * DH + e0), vf0, (const T*)nullptr);
#pragma unroll
            for (int e = 0; e < C::EPT; ++e) s0 = fmaf(qf[e], kf[e], s0);
          }
          if (v1) {
            float kf[C::EPT];
            unpack16(*reinterpret_cast<const uint4*>(sK + r1 * DH + e0), kf, (const T*)nullptr);
            unpack16(*reinterpret_cast<const uint4*>(sV + r1 * DH + e0), vf1, (const T*)nullptr);
#pragma unroll
            for (int e = 0; e < C::EPT; ++e) s1 = fmaf(qf[e], kf[e], s1);
          }
#pragma unroll
          for (int o = C::TPR / 2; o > 0; o >>= 1) {
            s0 += __shfl_xor_sync(0xffffffffu, s0, o);
            s1 += __shfl_xor_sync(0xffffffffu, s1, o);
          }
          if (v0) {
            if (!v1) s1 = -FLT_MAX;
            const float Mn = fmaxf(M, fmaxf(s0, s1));
            const float cs = exp2f(M - Mn), p0 = exp2f(s0 - Mn), p1 = v1 ? exp2f(s1 - Mn) : 0.f;
            l = l * cs + (p0 + p1);
#pragma unroll
            for (int e = 0; e < C::EPT; ++e) {
              float t = of[e] * cs;
              t = fmaf(p0, vf0[e], t);
              of[e] = v1 ? fmaf(p1, vf1[e], t) : t;
            }
            M = Mn;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with stage s
      }
    }
    i += cnt;
    if (i < nc) {
      const int b1 = (pr + 1) / H, h1 = (pr + 1) - b1 * H;
      qn = *reinterpret_cast<const uint4*>(q + (size_t)b1 * ldq + h1 * DH + e0);
    }
    // the warp's row groups merged by shuffles: lanes t, t + TPR, ... hold
    // the same output slice (a group without rows has M = -FLT_MAX, l = 0)
#pragma unroll
    for (int o = C::TPR; o < 32; o <<= 1) {
      const float Mo = __shfl_xor_sync(0xffffffffu, M, o);
      const float lo = __shfl_xor_sync(0xffffffffu, l, o);
      const float Mn = fmaxf(M, Mo);
      const float wa = exp2f(M - Mn), wb = exp2f(Mo - Mn);
      l = l * wa + lo * wb;
#pragma unroll
      for (int e = 0; e < C::EPT; ++e) of[e] = of[e] * wa + __shfl_xor_sync(0xffffffffu, of[e], o) * wb;
      M = Mn;
    }
    // park each warp's (M, l, o) for the combination across warps
    if (lane < C::TPR) {
      float* gr = sR + (size_t)warp * (DH + 2);
#pragma unroll
      for (int e = 0; e < C::EPT; ++e) gr[2 + e0 + e] = of[e];
      if (lane == 0) { gr[0] = M; gr[1] = l; }
    }
    cons_sync();
    // combine the warps: thread t < DH owns output dim t
    float Mg = -FLT_MAX, Lg = 0.f, og = 0.f;
    if (tid < DH) {
#pragma unroll
      for (int w = 0; w < C::CWARPS; ++w) Mg = fmaxf(Mg, sR[(size_t)w * (DH + 2)]);
#pragma unroll
      for (int w = 0; w < C::CWARPS; ++w) {
        const float* gr = sR + (size_t)w * (DH + 2);
        const float wt = exp2f(gr[0] - Mg);
        Lg = fmaf(wt, gr[1], Lg);
        og = fmaf(wt, gr[2 + tid], og);
      }
    }
    const long long pbeg = (long long)pr * nch;
    const int first = whole ? c : dec_owner(pbeg, G, Ttot);
    const int last = whole ? c : dec_owner(pbeg + nch - 1, G, Ttot);
    if (first == last) {
      if (ok && tid < DH) out[(size_t)b * ld_out + h * DH + tid] = from_f<T>(og / Lg);
    } else {
      // partial slot: 2c if pair pr is where this CTA's range starts, else 2c + 1
      float* my = part + ((size_t)2 * c + (pr == first_pair ? 0 : 1)) * (DH + 2);
      if (tid < DH) my[2 + tid] = og;
      if (tid == 0) { my[0] = Mg; my[1] = Lg; }
      // the consumers' barrier orders their partial writes before thread 0's
      // gpu-scope fence and counter update (release); the fence after the
      // update orders the last arriver's reads of the other partials after
      // it (acquire)
      cons_sync();
      if (tid == 0) {
        __threadfence();
        s_last = (atomicAdd(&counters[pr], 1) == last - first);
        __threadfence();
      }
      cons_sync();
      if (s_last) {
        float M2 = -FLT_MAX;
        for (int cc = first; cc <= last; ++cc) {
          const int first_of_cc = (int)(((long long)cc * Ttot / G) / nch);
          const float* ps = part + ((size_t)2 * cc + (pr == first_of_cc ? 0 : 1)) * (DH + 2);
          M2 = fmaxf(M2, __ldcg(ps));
        }
        float L2 = 0.f, o2 = 0.f;
        for (int cc = first; cc <= last; ++cc) {
          const int first_of_cc = (int)(((long long)cc * Ttot / G) / nch);
          const float* ps = part + ((size_t)2 * cc + (pr == first_of_cc ? 0 : 1)) * (DH + 2);
          const float w = exp2f(__ldcg(ps) - M2);
          L2 = fmaf(w, __ldcg(ps + 1), L2);
          if (tid < DH) o2 = fmaf(w, __ldcg(ps + 2 + tid), o2);
        }
        if (ok && tid < DH) out[(size_t)b * ld_out + h * DH + tid] = from_f<T>(o2 / L2);
        if (tid == 0) counters[pr] = 0;
      }
    }
    cons_sync();  // sR / s_last reused for the next pair
  }
}

static int dec_sm_count() { return device_sm_count(); }

template <typename T>
static int dec_chunk(int d) {
  return 4096 / (d * (int)sizeof(T));
}


// Persistent grid, at most DEC_CTAS_PER_SM CTAs per SM. With at least half as
// many (sequence, head) pairs as resident CTAs each CTA takes whole pairs,
// k or k - 1 of them for k = ceil(pairs / resident) (*whole = 1); with fewer
// pairs the chunks are spread over every resident CTA (stream-K, never more
// CTAs than chunks at the capacity).
static int dec_grid(int pairs, int d, int cap, int dt, int* whole) {
  const int chunk = dt == DT_BF16 ? dec_chunk<bf16>(d) : dec_chunk<float>(d);
  const long long slots = (long long)DEC_CTAS_PER_SM * dec_sm_count();
  if (2LL * pairs >= slots) {
    *whole = 1;
    const long long k = (pairs + slots - 1) / slots;
    return (int)((pairs + k - 1) / k);
  }
  *whole = 0;
  const long long max_chunks = (long long)pairs * ((cap + chunk - 1) / chunk);
  return (int)(slots < max_chunks ? slots : max_chunks);
}

int attn_decode_max_splits(int d, int cap, int dt) {
  int whole;
  return dec_grid(1, d, cap, dt, &whole);
}

// scratch layout: [merge counters: B*H ints, 256-aligned][partials: two
// slots of (d + 2) floats per CTA of the grid]; counters sit at offset 0.
size_t attn_decode_scratch_bytes(int B, int H, int d, int cap, int dt) {
  return attn_decode_scratch_bytes_for((long long)B * H, d);
}

template <typename T, int DH>
static cudaError_t dec_prepare() {
  // the attribute applies to the current device only
  static bool done[MAX_DEVICES] = {};
  const int dev = current_device();
  if (dev >= 0 && done[dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(attn_decode_kernel<T, DH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DecCfg<T, DH>::SMEM);
  if (e == cudaSuccess && dev >= 0) done[dev] = true;
  return e;
}

cudaError_t attn_prepare() {
  cudaError_t e;
  if ((e = dec_prepare<bf16, 32>()) != cudaSuccess) return e;
  if ((e = dec_prepare<bf16, 64>()) != cudaSuccess) return e;
  if ((e = dec_prepare<bf16, 128>()) != cudaSuccess) return e;
  if ((e = dec_prepare<float, 32>()) != cudaSuccess) return e;
  if ((e = dec_prepare<float, 64>()) != cudaSuccess) return e;
  return dec_prepare<float, 128>();
}

template <typename T, int DH>
static cudaError_t launch_dec(const void* q, int ldq, const void* kc, const void* vc, int B,
                              int H, int cap, PosSpec kvlen, void* out, int ld_out,
                              void* scratch, int* status, cudaStream_t s, int g) {
  using C = DecCfg<T, DH>;
  cudaError_t e = dec_prepare<T, DH>();
  if (e != cudaSuccess) return e;
  const int pairs = B * H;
  int whole = 0;
  int G = dec_grid(pairs, DH, cap, sizeof(T) == 2 ? DT_BF16 : DT_F32, &whole);
  if (G > DEC_UNITS_SLACK) G = DEC_UNITS_SLACK;  // partial slots in the scratch
  int* counters = reinterpret_cast<int*>(scratch);
  float* partp = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(scratch) +
                                          (((size_t)pairs * sizeof(int) + 255) & ~(size_t)255));
  const float qscale = 1.4426950408889634f / sqrtf((float)DH);
  BT_LAUNCH(attn_decode_kernel<T, DH>, dim3(G), dim3(C::THREADS), C::SMEM, s, (const T*)q, ldq,
            (const T*)kc, (const T*)vc, pairs, H, cap, kvlen, (T*)out, ld_out, partp, counters,
            status, qscale, g, whole);
  return cudaSuccess;
}

cudaError_t launch_attn_decode(int dt, const void* q, int ldq, const void* k_cache,
                               const void* v_cache, int B, int H, int d, int cap,
                               PosSpec kvlen, void* out, int ld_out, void* scratch,
                               int* status, cudaStream_t s, int Hk) {
  if (B * H == 0) return cudaSuccess;
  if (Hk <= 0) Hk = H;
  if (H % Hk) return cudaErrorInvalidValue;
  const int g = H / Hk;
#define BT_DEC(T, DHV) \
  return launch_dec<T, DHV>(q, ldq, k_cache, v_cache, B, H, cap, kvlen, out, ld_out, scratch, status, s, g)
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
                                  T* __restrict__ out, int ld_out, float scale, int g) {
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
  // key/value head h / g of H / g (grouped-query attention)
  const T* kb = kc + ((size_t)b * (H / g) + h / g) * cap * DH;
  const T* vb = vc + ((size_t)b * (H / g) + h / g) * cap * DH;
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
                              void* out, int ld_out, cudaStream_t s, int Hk) {
  const int warps = B * qpos.rows_per_seq * H;
  if (warps == 0) return cudaSuccess;
  if (Hk <= 0) Hk = H;
  if (H % Hk) return cudaErrorInvalidValue;
  const int g = H / Hk;
  const int grid = (warps + 3) / 4;
  const float scale = 1.4426950408889634f / sqrtf((float)d);
#define BT_SMALL(T, DHV)                                                                      \
  BT_LAUNCH(attn_small_kernel<T, DHV>, dim3(grid), dim3(128), 0, s, (const T*)q, ldq, (const T*)k_cache,        \
                                                  (const T*)v_cache, B, H, cap, qpos, (T*)out, \
                                                  ld_out, scale, g);                          \
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
                                void* out, int ld_out, cudaStream_t s, int Hk) {
  PosSpec p{nullptr, POS_ZERO, 0, n};
  return launch_attn_small(dt, q, ldq, k_cache, v_cache, B, H, d, cap, p, out, ld_out, s, Hk);
}

}  // namespace bt
