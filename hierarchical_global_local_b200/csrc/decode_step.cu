// decode_step.cu -- the token-decoder half of a decode step as one persistent
// kernel (bf16, at most 64 sequences): every token-decoder layer, the final
// LayerNorm, the LM head and the greedy argmax. A second instance of the same
// kernel (BLOCK = true, opt-in) runs a whole block step: the block embedding,
// every block-decoder layer with its decode attention as a phase, LN_b and the
// prefix projection, then the token-decoder program over the prefix row.
//
// Block Transformer (Ho et al., "Block Transformer: Global-to-Local Language
// Modeling for Fast Inference"), section 2.3 (token decoder) and the Pythia
// layer it is built from (parallel attention + MLP residual, partial rotary,
// GELU MLP). The token decoder of one decode step reads every one of its
// weights once for a single row per sequence: the step is a chain of small
// weight-streaming GEMMs whose cost, launched as separate kernels, is
// launch and pipeline-fill latency rather than bytes.
//
// Here one CTA per SM runs the whole chain. A producer warp streams every
// weight tile the CTA will use, in program order, through a shared-memory
// ring with TMA (weights do not depend on the activations, so the stream
// runs ahead across layer boundaries and grid barriers); an MMA warp issues
// the tensor-core work of every unit as soon as its activations are staged
// and an accumulator is free; the four worker warps stage activations, drain
// the accumulators and run the phases below, separated by grid-wide barriers:
//   I   (row b per CTA)  embed the fed token (token steps), LayerNorm 1/2 of
//                        layer 0 -> x1 = [LN1(h) | LN2(h)] bf16
//   per layer l:
//   G1  (tile x K-split) partial sums of x1 W_qkv1^T (q | k | v | fc1) on
//                        tcgen05 (activation boxes by TMA), fp32 partial
//                        tiles to L2
//   R1                   sum the splits + bias; q, k rotary; k, v into the
//                        local cache; attention over the local window (16
//                        lanes per sequence and head); GELU(fc1) -> a2
//   G2  (tile x K-split) partial sums of a2 W_o2^T ([W_o | W_2])
//   R2  (row b per CTA)  h += splits + b_o + b_2; LayerNorm of the new row
//                        for the next layer, or the final LayerNorm -> xf
//   GL  (vocab tiles)    LM head on tcgen05 (two TMEM accumulators: the MMAs
//                        of one tile overlap the epilogue of the previous);
//                        logits (optional) and per-tile argmax partials
//   AR                   greedy argmax per row (lowest id on ties), advance
//                        the step state
// The MMA orientation is "weights as A": M = 128 output features per tile,
// N = the batch padded to a multiple of 16, K in 64-wide swizzled blocks.
//
// Block-step phases before the token-decoder program (BLOCK = true):
//   I_b (row b per CTA)  block row = the L_B token embeddings of the completed
//                        block; LN1 | LN2 of block layer 0 -> x1
//   per block layer: G1, then A (decode attention over the block cache, see
//   block_attention_phase; GELU(fc1) -> a2), G2, then R2 into the block
//   residual rows with the next block layer's LayerNorms or LN_b -> xf
//   Gp / Rp              prefix projection W_p xf + b_p -> the token rows,
//                        LN1 | LN2 of token layer 0 -> x1
//
// Grid barriers are a counter in global memory (release by a red.release
// add, acquire by polling with ld.acquire). All CTAs must be resident at
// once: one CTA per SM, grid = number of SMs, launched cooperatively so that
// the driver guarantees it. Every wait is bounded: a barrier that runs out
// sets ST_WAIT_TIMEOUT and an abort word that makes every CTA skip the rest
// of the step; the producer then waits (bounded) for its copies in flight,
// TMEM is freed and the kernel returns.
#include <cuda.h>
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "gridsync.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace bt {

namespace {

constexpr int WORKERS = 128;                 // warps 0-3 (TMEM lanes 0-127)
constexpr int THREADS = WORKERS + 64;        // warp 4: TMA producer, warp 5: MMA issuer
constexpr int TILE_BYTES = 128 * 64 * 2;     // one weight box: 128 rows x 64 K (bf16)
constexpr int MAX_STAGES = 12;
// K splits: as many as fill the SMs up to these caps. q|k|v|fc1: fewer splits
// mean fewer partial sums for the reduction phase (B200, D = 768: 2 beats 1
// and 3). [W_o | W_2]: the token layers add their splits into fixed-point
// accumulators by L2 reductions, so more splits only add reductions (D = 768:
// 20 splits 178.6 us per token step, 15: 178.7, 12: 180.6, 10: 182.6).
constexpr int MAX_S1 = 2;                    // K splits of the q|k|v|fc1 GEMM
constexpr int MAX_S2 = 24;                   // K splits of the [W_o | W_2] GEMM
constexpr int MAX_B = 64;
constexpr int MAX_WIN = 8;                   // local-window slots (P + L_B - 1)
constexpr int TMEM_COLS = 128;               // two accumulators of up to 64 columns
// block-step decode attention: units of ATT_CH cache entries of one
// (sequence, head), d_head 64; each worker warp streams its units' K and V
// rows through ATT_SLOTS bulk-copy slots in the (then idle) activation buffer
constexpr int ATT_CH = 32;
constexpr int ATT_SLOTS = 3;
constexpr int ATT_SLOT_BYTES = 2 * ATT_CH * 64 * 2;              // K and V rows
constexpr int ATT_BYTES = 4 * ATT_SLOTS * ATT_SLOT_BYTES;        // 96 KB
constexpr int ATT_PART = 68;                                     // m, l, o[64], pad
constexpr int ATT_MAX_CHUNKS = 32;                               // n_cap <= 1024
constexpr int PRODUCER_SLEEP_NS = 128;  // back-off of the weight producer's slot waits
constexpr int MMA_SLEEP_NS = 32;        // back-off of the MMA warp's waits (on the critical path)

struct Plan {
  int Bp;            // batch padded to a multiple of 16 (MMA N)
  int S1, S2;        // K splits
  int T1, T2, TL;    // feature tiles: 7D/128, D/128, ceil(V/128)
  int nkb1, nkb2;    // 64-wide K blocks per split
  int nkbL;          // K blocks of the LM head (D/64)
  int Sp, nkbp;      // prefix projection (block steps): K splits, K blocks per split
  int stages;
  float scale;       // log2(e) / sqrt(d_head)
};

__device__ __forceinline__ void wsync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }


template <typename T>
__device__ __forceinline__ const T* layer_ptr(const T* base, int l, long long stride) {
  return reinterpret_cast<const T*>(reinterpret_cast<const uint8_t*>(base) + (long long)l * stride);
}

// mbarrier wait of the producer and MMA warps: backs off between polls so
// that the worker warps sharing their SM sub-partitions keep the issue
// slots; gives up when the CTA has aborted
__device__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* status, volatile int* s_abort,
                              int sleep_ns, long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  int n = 0;
  while (!mbar_try_wait(bar, parity)) {
    __nanosleep(sleep_ns);
    if ((++n & 63) == 0) {
      if (*s_abort) return false;
      if (clock64() - t0 > limit) {
        set_status(status, ST_WAIT_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

// Grid-wide barrier for the 128 worker threads of every CTA (named barrier
// 1), bounded by the launch's wait limit (gridsync.cuh).
__device__ __forceinline__ bool grid_sync(const TokenStepArgs& a, unsigned target, volatile int* s_abort) {
  return grid_barrier(a.bar, target, a.wait_cycles, a.status, s_abort, 1, 128);
}

// sum over the four worker warps (all 128 workers call it)
__device__ __forceinline__ float worker_sum(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  wsync();
  v = (red[0] + red[1]) + (red[2] + red[3]);
  wsync();
  return v;
}

__device__ __forceinline__ void store_bf16x4(bf16* o, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(o) = u;
}

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// LayerNorm gains / biases of the features this thread holds (float4 q =
// tid + 128u covers features 4q..4q+3), loaded with the row's other inputs
struct LnParams {
  float4 g1[4], b1[4], g2[4], b2[4];
};
__device__ __forceinline__ void ln_load(LnParams& p, int D, const float* g1, const float* b1,
                                        const float* g2, const float* b2) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int f = (threadIdx.x + u * WORKERS) * 4;
    if (f < D) {
      p.g1[u] = *reinterpret_cast<const float4*>(g1 + f);
      p.b1[u] = *reinterpret_cast<const float4*>(b1 + f);
      if (g2) {
        p.g2[u] = *reinterpret_cast<const float4*>(g2 + f);
        p.b2[u] = *reinterpret_cast<const float4*>(b2 + f);
      }
    }
  }
}

// LayerNorm of the row held in v[] (same layout), written as bf16 with
// (g1, b1) to out1 and, if out2, (g2, b2) to out2. Two-pass statistics in fp32.
__device__ void ln_out(const float4* v, int D, float eps, const LnParams& p, bf16* out1, bf16* out2,
                       float* red) {
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int f = (threadIdx.x + u * WORKERS) * 4;
    if (f < D) s += (v[u].x + v[u].y) + (v[u].z + v[u].w);
  }
  const float mu = worker_sum(s, red) / (float)D;
  float q = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int f = (threadIdx.x + u * WORKERS) * 4;
    if (f < D) {
      const float a = v[u].x - mu, b = v[u].y - mu, c = v[u].z - mu, d = v[u].w - mu;
      q += (a * a + b * b) + (c * c + d * d);
    }
  }
  const float rstd = rsqrtf(worker_sum(q, red) / (float)D + eps);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int f = (threadIdx.x + u * WORKERS) * 4;
    if (f < D) {
      const float n0 = (v[u].x - mu) * rstd, n1 = (v[u].y - mu) * rstd;
      const float n2 = (v[u].z - mu) * rstd, n3 = (v[u].w - mu) * rstd;
      const float4 ga = p.g1[u], ba = p.b1[u];
      store_bf16x4(out1 + f, n0 * ga.x + ba.x, n1 * ga.y + ba.y, n2 * ga.z + ba.z, n3 * ga.w + ba.w);
      if (out2) {
        const float4 gb = p.g2[u], bb = p.b2[u];
        store_bf16x4(out2 + f, n0 * gb.x + bb.x, n1 * gb.y + bb.y, n2 * gb.z + bb.z, n3 * gb.w + bb.w);
      }
    }
  }
}

// ---- TMA producer (warp 4, one thread) ----------------------------------------
// Walks exactly the (phase, unit, K block) sequence the MMA issuer consumes.
__device__ void producer(const CUtensorMap* mq, const CUtensorMap* mo, const CUtensorMap* ml,
                         const CUtensorMap* mqb, const CUtensorMap* mob, const CUtensorMap* mp,
                         const Plan& P, int Nt, int Nb, uint8_t* ring, uint64_t* full, uint64_t* empty,
                         int* status, volatile int* s_abort, long long limit) {
  const int G = gridDim.x, c = blockIdx.x;
  int it = 0;
  bool stop = false;
  // weights are read once per step: keep them from evicting the activations
  // and partial sums that the phases exchange through L2
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  auto load = [&](const CUtensorMap* m, int x, int y, int z, bool three) {
    if (stop) return;
    const int s = it % P.stages;
    if (it >= P.stages && !wait_or_abort(&empty[s], ((it / P.stages) + 1) & 1, status, s_abort, PRODUCER_SLEEP_NS, limit)) {
      stop = true;
      return;
    }
    mbar_arrive_expect_tx(&full[s], TILE_BYTES);
    if (three) tc::tma_load_3d_hint(ring + (size_t)s * TILE_BYTES, m, x, y, z, &full[s], policy);
    else tc::tma_load_2d_hint(ring + (size_t)s * TILE_BYTES, m, x, y, &full[s], policy);
    ++it;
  };
  // block step: block-decoder layers and the prefix projection first
  for (int l = 0; l < Nb && !stop; ++l) {
    for (int u = c; u < P.T1 * P.S1 && !stop; u += G) {
      const int t = u % P.T1, sp = u / P.T1;
      for (int kb = 0; kb < P.nkb1; ++kb) load(mqb, (sp * P.nkb1 + kb) * 64, t * 128, l, true);
    }
    for (int u = c; u < P.T2 * P.S2 && !stop; u += G) {
      const int t = u % P.T2, sp = u / P.T2;
      for (int kb = 0; kb < P.nkb2; ++kb) load(mob, (sp * P.nkb2 + kb) * 64, t * 128, l, true);
    }
  }
  if (Nb > 0)
    for (int u = c; u < P.T2 * P.Sp && !stop; u += G) {
      const int t = u % P.T2, sp = u / P.T2;
      for (int kb = 0; kb < P.nkbp; ++kb) load(mp, (sp * P.nkbp + kb) * 64, t * 128, 0, false);
    }
  // (Prefetching the LM head into L2 while the layers run, with an
  // evict-last policy, measured ~10 us slower per token step on B200 at
  // D = 768: the LM head streams from HBM with the other weights.)
  for (int l = 0; l < Nt && !stop; ++l) {
    for (int u = c; u < P.T1 * P.S1 && !stop; u += G) {
      const int t = u % P.T1, sp = u / P.T1;
      for (int kb = 0; kb < P.nkb1; ++kb) load(mq, (sp * P.nkb1 + kb) * 64, t * 128, l, true);
    }
    for (int u = c; u < P.T2 * P.S2 && !stop; u += G) {
      const int t = u % P.T2, sp = u / P.T2;
      for (int kb = 0; kb < P.nkb2; ++kb) load(mo, (sp * P.nkb2 + kb) * 64, t * 128, l, true);
    }
  }
  for (int t = c; t < P.TL && !stop; t += G)
    for (int kb = 0; kb < P.nkbL; ++kb) load(ml, kb * 64, t * 128, 0, false);
  // copies still in flight (none on a normal run: the issuer consumed them all)
  const int first = it > P.stages ? it - P.stages : 0;
  for (int j = first; j < it; ++j) mbar_wait_bounded(&full[j % P.stages], (j / P.stages) & 1, status);
}

// ---- worker-side pieces ------------------------------------------------------
// Activations for one unit: nkb boxes of Bp rows x 64 columns of a bf16
// matrix (rows >= B read as zero), columns col0 + 64*kb, by TMA into `act`
// (swizzled K-major blocks of Bp x 128 bytes) with completion on `bar`. One
// thread. The rows were written by other CTAs of this kernel through the
// generic proxy before the grid barrier; the proxy fence orders those writes
// before this thread's asynchronous-proxy reads.
__device__ void load_act(const CUtensorMap* map, uint8_t* act, int col0, int nkb, int Bp, uint64_t* bar) {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  mbar_arrive_expect_tx(bar, (uint32_t)(nkb * Bp * 128));
  for (int kb = 0; kb < nkb; ++kb)
    tc::tma_load_2d(act + (size_t)kb * Bp * 128, map, col0 + kb * 64, 0, bar);
}

// One thread: the MMAs of one unit (nkb K blocks from the ring, activations
// from `act`) into TMEM columns at tmem_d, then a commit to `done`.
__device__ void issue_unit(const Plan& P, int nkb, uint8_t* ring, const uint8_t* act, uint32_t tmem_d,
                           uint64_t* full, uint64_t* empty, uint64_t* done, int& it, int* status) {
  const uint32_t idesc = tc::idesc_bf16_m128(P.Bp);
  for (int kb = 0; kb < nkb; ++kb, ++it) {
    const int s = it % P.stages;
    mbar_wait_bounded(&full[s], (it / P.stages) & 1, status);
    tc::fence_after();
    const uint64_t da = tc::desc_sw128(smem_u32(ring + (size_t)s * TILE_BYTES));
    const uint64_t db = tc::desc_sw128(smem_u32(act + (size_t)kb * P.Bp * 128));
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)  // 16-wide K slices: +32 bytes = +2 in descriptor units
      tc::mma_bf16(tmem_d, da + 2 * kk, db + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
    tc::commit(&empty[s]);
  }
  tc::commit(done);
}

// fp32 partial tile (128 features x B rows) from TMEM to part[u][row][128]
__device__ void store_partial(uint32_t tbuf, float* part, int u, int B, int Bp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t trow = tbuf + ((uint32_t)(warp * 32) << 16);
  float* dst = part + (size_t)u * B * 128 + warp * 32 + lane;
  for (int c0 = 0; c0 < Bp; c0 += 16) {
    float v[16];
    tc::tmem_ld16(trow + c0, v);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (c0 + j < B) __stcg(dst + (size_t)(c0 + j) * 128, v[j]);
  }
}

// Fixed-point scale of the split-K sums: a partial v is added as the
// 64-bit integer round(v * 2^32). Integer addition is associative, so the
// sum does not depend on the order in which the splits arrive, and the
// result is the same bit for bit from run to run (which fp32 additions in
// arrival order are not). Resolution 2^-32; |sums| below 2^31.
constexpr float FX_ONE = 4294967296.0f;            // 2^32
constexpr float FX_INV = 2.3283064365386963e-10f;  // 2^-32

// The same accumulator added into the int64 accumulators fx [B][D]
// (features t*128 .. t*128+127) with L2 reductions: the phase after the
// next grid barrier reads one value per element instead of one per split,
// and stores zero back.
__device__ void red_partial(uint32_t tbuf, long long* fx, int t, int B, int Bp, int D) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t trow = tbuf + ((uint32_t)(warp * 32) << 16);
  unsigned long long* dst = reinterpret_cast<unsigned long long*>(fx) + (size_t)t * 128 + warp * 32 + lane;
  for (int c0 = 0; c0 < Bp; c0 += 16) {
    float v[16];
    tc::tmem_ld16(trow + c0, v);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (c0 + j < B) atomicAdd(dst + (size_t)(c0 + j) * D, (unsigned long long)__float2ll_rn(v[j] * FX_ONE));
  }
}

// four consecutive fixed-point sums as floats; the accumulators are cleared
__device__ __forceinline__ float4 fx_take4(long long* p) {
  longlong2* q = reinterpret_cast<longlong2*>(p);
  const longlong2 a = __ldcg(q), b = __ldcg(q + 1);
  __stcg(q, make_longlong2(0, 0));
  __stcg(q + 1, make_longlong2(0, 0));
  return make_float4(__ll2float_rn(a.x) * FX_INV, __ll2float_rn(a.y) * FX_INV, __ll2float_rn(b.x) * FX_INV,
                     __ll2float_rn(b.y) * FX_INV);
}

// Shared-memory barriers of the worker / MMA hand-off.
struct Sync {
  uint64_t* full;       // [stages] weight tile landed
  uint64_t* empty;      // [stages] weight tile consumed
  uint64_t* act_full;   // activations landed (TMA transaction count)
  uint64_t* acc_full;   // [2] accumulator ready (tcgen05.commit)
  uint64_t* acc_empty;  // [2] accumulator drained (128 worker arrivals)
};

// Split-K GEMM phase, worker side: units u = blockIdx.x + i*gridDim.x of T
// tiles x S splits, each nkb K blocks; activations through `map`, columns
// col_of(tile) + split*nkb*64. `na` counts activation loads, `nu` accumulator
// uses (both in the MMA warp's order).
template <typename ColOf>
__device__ void gemm_phase(const Plan& P, int T, int S, int nkb, const CUtensorMap* map, ColOf col_of,
                           int B, float* part, uint8_t* act, uint32_t tmem, const Sync& y, int& na,
                           int& nu, int* status, long long* red_fx = nullptr, int D = 0) {
  for (int u = blockIdx.x; u < T * S; u += gridDim.x) {
    const int t = u % T, sp = u / T;
    // act is free: the previous unit's MMAs (its last readers) completed
    // before that unit's accumulator was drained below
    if (threadIdx.x == 0) load_act(map, act, col_of(t) + sp * nkb * 64, nkb, P.Bp, y.act_full);
    ++na;
    const int buf = nu & 1;
    mbar_wait_bounded(&y.acc_full[buf], (nu >> 1) & 1, status);
    tc::fence_after();
    if (red_fx) red_partial(tmem + (uint32_t)(buf * 64), red_fx, t, B, P.Bp, D);
    else store_partial(tmem + (uint32_t)(buf * 64), part, u, B, P.Bp);
    tc::fence_before();
    mbar_arrive(&y.acc_empty[buf]);
    ++nu;
  }
}

// MMA warp (one thread): the same unit sequence as the workers and the
// producer. Waits for staged activations and a drained accumulator.
__device__ void mma_issuer(const Plan& P, int Nt, int Nb, uint8_t* ring, const uint8_t* act, uint32_t tmem,
                           const Sync& y, int* status, volatile int* s_abort, long long limit) {
  const int G = gridDim.x, c = blockIdx.x;
  int it = 0, na = 0, nu = 0;
  auto unit = [&](int nkb, bool need_act) -> bool {
    if (need_act) {
      if (!wait_or_abort(y.act_full, na & 1, status, s_abort, MMA_SLEEP_NS, limit)) return false;
      ++na;
    }
    const int buf = nu & 1;
    if (nu >= 2 && !wait_or_abort(&y.acc_empty[buf], ((nu >> 1) + 1) & 1, status, s_abort, MMA_SLEEP_NS, limit))
      return false;
    tc::fence_after();
    issue_unit(P, nkb, ring, act, tmem + (uint32_t)(buf * 64), y.full, y.empty, &y.acc_full[buf], it, status);
    ++nu;
    return true;
  };
  for (int l = 0; l < Nb; ++l) {
    for (int u = c; u < P.T1 * P.S1; u += G)
      if (!unit(P.nkb1, true)) return;
    for (int u = c; u < P.T2 * P.S2; u += G)
      if (!unit(P.nkb2, true)) return;
  }
  if (Nb > 0)
    for (int u = c; u < P.T2 * P.Sp; u += G)
      if (!unit(P.nkbp, true)) return;
  for (int l = 0; l < Nt; ++l) {
    for (int u = c; u < P.T1 * P.S1; u += G)
      if (!unit(P.nkb1, true)) return;
    for (int u = c; u < P.T2 * P.S2; u += G)
      if (!unit(P.nkb2, true)) return;
  }
  bool first = true;
  for (int t = c; t < P.TL; t += G) {
    if (!unit(P.nkbL, first)) return;  // every vocab tile reads the same staged input
    first = false;
  }
}

// R1, one half-warp (16 lanes) per (sequence, head): q|k|v from the K
// splits + bias, rotary on q and k, k and v appended to the local cache at
// `pos`, attention of the query over cache slots 0..pos. Lane l of the group
// holds head dims l + 16x.
template <int DH>
__device__ void attend_item(const TokenStepArgs& a, const Plan& P, const float* bq, bf16* kc, bf16* vc,
                            int b, int h, int pos, bool active) {
  constexpr int EPL = DH / 16;
  const int l16 = threadIdx.x & 15;
  const int D = a.D, B = a.B;
  const size_t split_stride = (size_t)P.T1 * B * 128;
  float q[EPL], k[EPL], v[EPL];
  float kw[MAX_WIN][EPL], vw[MAX_WIN][EPL];
  const size_t base = ((size_t)b * a.H + h) * a.l_cap * DH;
  // every load of the item in one batch: partial sums, biases, the window
#pragma unroll
  for (int x = 0; x < EPL; ++x) {
    const int nq = h * DH + l16 + 16 * x, nk = D + nq, nv = 2 * D + nq;
    float sq = 0.f, sk = 0.f, sv = 0.f;
    if (active) {
      sq = bq[nq]; sk = bq[nk]; sv = bq[nv];
      const float* pq = a.p1 + ((size_t)(nq >> 7) * B + b) * 128 + (nq & 127);
      const float* pk = a.p1 + ((size_t)(nk >> 7) * B + b) * 128 + (nk & 127);
      const float* pv = a.p1 + ((size_t)(nv >> 7) * B + b) * 128 + (nv & 127);
#pragma unroll
      for (int s = 0; s < MAX_S1; ++s) {
        if (s < P.S1) {
          sq += __ldcg(pq + s * split_stride);
          sk += __ldcg(pk + s * split_stride);
          sv += __ldcg(pv + s * split_stride);
        }
      }
    }
    q[x] = sq; k[x] = sk; v[x] = sv;
#pragma unroll
    for (int j = 0; j < MAX_WIN; ++j) {
      const int e = l16 + 16 * x;
      kw[j][x] = (active && j < pos) ? __bfloat162float(kc[base + (size_t)j * DH + e]) : 0.f;
      vw[j][x] = (active && j < pos) ? __bfloat162float(vc[base + (size_t)j * DH + e]) : 0.f;
    }
  }
  if (a.rot > 0) {
    // rotate-half pairs (e, e ^ half), e < rot: for half < 16 the pair is in
    // lane l16 ^ half of the group, for half = 16 in this lane's register x ^ 1
    const int half = a.rot >> 1;
    float qp[EPL], kp[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) {
      const float qs = __shfl_xor_sync(0xffffffffu, q[x], half < 16 ? half : 0);
      const float ks = __shfl_xor_sync(0xffffffffu, k[x], half < 16 ? half : 0);
      qp[x] = (half < 16) ? qs : q[x ^ 1];
      kp[x] = (half < 16) ? ks : k[x ^ 1];
    }
#pragma unroll
    for (int x = 0; x < EPL; ++x) {
      const int e = l16 + 16 * x;
      if (e < a.rot) {
        const float2 cs = a.rope_tab[(size_t)pos * half + (e & (half - 1))];
        if (e & half) {
          q[x] = q[x] * cs.x + qp[x] * cs.y;
          k[x] = k[x] * cs.x + kp[x] * cs.y;
        } else {
          q[x] = q[x] * cs.x - qp[x] * cs.y;
          k[x] = k[x] * cs.x - kp[x] * cs.y;
        }
      }
    }
  }
#pragma unroll
  for (int x = 0; x < EPL; ++x) {
    const int e = l16 + 16 * x;
    const bf16 kb = __float2bfloat16_rn(k[x]), vb = __float2bfloat16_rn(v[x]);
    if (active) {
      kc[base + (size_t)pos * DH + e] = kb;
      vc[base + (size_t)pos * DH + e] = vb;
    }
    k[x] = __bfloat162float(kb);  // attention reads what the cache holds
    v[x] = __bfloat162float(vb);
  }
  float mrun = -FLT_MAX, lsum = 0.f, o[EPL];
#pragma unroll
  for (int x = 0; x < EPL; ++x) o[x] = 0.f;
#pragma unroll
  for (int j = 0; j < MAX_WIN; ++j) {
    if (j > pos) break;
    float s = 0.f;
#pragma unroll
    for (int x = 0; x < EPL; ++x) s = fmaf(q[x], j < pos ? kw[j][x] : k[x], s);
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);  // 16-lane group
    s *= P.scale;
    const float mn = fmaxf(mrun, s);
    const float cf = exp2f(mrun - mn), p = exp2f(s - mn);
    lsum = lsum * cf + p;
#pragma unroll
    for (int x = 0; x < EPL; ++x) o[x] = o[x] * cf + p * (j < pos ? vw[j][x] : v[x]);
    mrun = mn;
  }
  if (active) {
    bf16* out = a.a2 + (size_t)b * 5 * D + h * DH;
#pragma unroll
    for (int x = 0; x < EPL; ++x) out[l16 + 16 * x] = __float2bfloat16_rn(o[x] / lsum);
  }
}

__device__ void gelu_fc1(const TokenStepArgs& a, const Plan& P, const float* bq, int c0 = 0, int nc = 0);

__device__ void r1_phase(const TokenStepArgs& a, const Plan& P, int l, int pos) {
  const int B = a.B;
  const float* bq = layer_ptr(a.b_qkv1, l, a.layer_stride);
  bf16* kc = a.kt + (size_t)l * a.kt_layer;
  bf16* vc = a.vt + (size_t)l * a.kt_layer;
  // (sequence, head) items over the half-warps of the first CA CTAs; both
  // halves of a warp run the shuffles together, an idle half with
  // active = false. When one item per half-warp leaves CTAs without items,
  // and those can take GELU(fc1) in at most two batches of four float4 per
  // thread, they do it meanwhile (two latency chains side by side instead
  // of one after the other); else every CTA does GELU after its items.
  const int G = gridDim.x;
  const int hw = threadIdx.x >> 4;
  const int n_items = B * a.H;
  const int A = min(G, (n_items + 7) / 8);
  const bool split = A < G && (long long)B * a.D <= (long long)(G - A) * WORKERS * 8;
  const int CA = split ? A : G;
  if ((int)blockIdx.x < CA) {
    for (int i0 = blockIdx.x * 8 + (hw & ~1); i0 < n_items; i0 += 8 * CA) {
      const int i = i0 + (hw & 1);
      const bool active = i < n_items;
      const int b = active ? i / a.H : 0, h = active ? i - b * a.H : 0;
      if (a.dh == 32) attend_item<32>(a, P, bq, kc, vc, b, h, pos, active);
      else if (a.dh == 64) attend_item<64>(a, P, bq, kc, vc, b, h, pos, active);
      else attend_item<128>(a, P, bq, kc, vc, b, h, pos, active);
    }
  }
  gelu_fc1(a, P, bq, split ? A : 0, split ? G - A : 0);
}

// GELU(fc1): features 3D + c, c < 4D, of the first GEMM (its K splits + the
// bias) -> a2[:, D + c], four at a time (a group never crosses a 128-feature
// tile), over the nc CTAs c0 .. c0 + nc - 1 (nc = 0: the whole grid)
__device__ void gelu_fc1(const TokenStepArgs& a, const Plan& P, const float* bq, int c0, int nc) {
  if (nc <= 0) {
    c0 = 0;
    nc = gridDim.x;
  }
  const int rank = (int)blockIdx.x - c0;
  if (rank < 0 || rank >= nc) return;
  const int D = a.D, B = a.B;
  const int W4 = D;  // float4 groups per row
  const int E = B * W4;
  const int nthr = nc * WORKERS;
  constexpr int BATCH = 4;
  for (int e0 = rank * WORKERS + threadIdx.x; e0 < E; e0 += BATCH * nthr) {
    float4 acc[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int e = e0 + j * nthr;
      if (e < E) {
        const int b = e / W4, n = 3 * D + 4 * (e - b * W4);
        float4 sum = *reinterpret_cast<const float4*>(bq + n);
        const float* src = a.p1 + ((size_t)(n >> 7) * B + b) * 128 + (n & 127);
        const size_t split_stride = (size_t)P.T1 * B * 128;
#pragma unroll
        for (int sp = 0; sp < MAX_S1; ++sp)
          if (sp < P.S1) sum = f4add(sum, __ldcg(reinterpret_cast<const float4*>(src + sp * split_stride)));
        acc[j] = sum;
      }
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int e = e0 + j * nthr;
      if (e < E) {
        const int b = e / W4, c = 4 * (e - b * W4);
        store_bf16x4(a.a2 + (size_t)b * 5 * D + D + c, gelu_erf(acc[j].x), gelu_erf(acc[j].y),
                     gelu_erf(acc[j].z), gelu_erf(acc[j].w));
      }
    }
  }
}

// R2: h += (the out|fc2 units' K-split sum, from the fixed-point
// accumulators) + (b_o + b_2), then the LayerNorm of the new row for layer l + 1
// (LN1 | LN2 -> x1) or the final LayerNorm (-> xf).
__device__ void r2_phase(const TokenStepArgs& a, const Plan& P, int l, float* red) {
  const int D = a.D, B = a.B;
  const float* bo = layer_ptr(a.b_o2, l, a.layer_stride);
  // the next LayerNorm's parameters: layer l + 1's LN1 | LN2, or the final one
  LnParams lp;
  if (blockIdx.x < B) {
    if (l + 1 < a.Nt)
      ln_load(lp, D, layer_ptr(a.ln1_g, l + 1, a.layer_stride), layer_ptr(a.ln1_b, l + 1, a.layer_stride),
              layer_ptr(a.ln2_g, l + 1, a.layer_stride), layer_ptr(a.ln2_b, l + 1, a.layer_stride));
    else
      ln_load(lp, D, a.lnf_g, a.lnf_b, nullptr, nullptr);
  }
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    float4 hv[4];
    float* hrow = a.h + (size_t)b * D;
    long long* frow = a.fx + (size_t)b * D;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int f = (threadIdx.x + u * WORKERS) * 4;
      hv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (f < D) {
        const float4 acc = f4add(f4add(__ldcg(reinterpret_cast<const float4*>(hrow + f)), fx_take4(frow + f)),
                                 *reinterpret_cast<const float4*>(bo + f));
        hv[u] = acc;
        __stcg(reinterpret_cast<float4*>(hrow + f), acc);
      }
    }
    if (l + 1 < a.Nt) {
      bf16* o = a.x1 + (size_t)b * 2 * D;
      ln_out(hv, D, a.eps, lp, o, o + D, red);
    } else {
      ln_out(hv, D, a.eps, lp, a.xf + (size_t)b * D, nullptr, red);
    }
  }
}

// phase I: the row of each sequence (the fed token's embedding on token
// steps; the prefix row already in h on block steps) -> LN1 | LN2 of layer 0
__device__ void ingest_phase(const TokenStepArgs& a, int jb, float* red) {
  const int D = a.D;
  LnParams lp;
  if (blockIdx.x < a.B) ln_load(lp, D, a.ln1_g, a.ln1_b, a.ln2_g, a.ln2_b);
  for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
    float4 hv[4];
    float* hrow = a.h + (size_t)b * D;
    int tok = 0;
    if (a.ingest) {
      tok = a.src[b];
      if (tok < 0 || tok >= a.V) {
        if (threadIdx.x == 0) set_status(a.status, ST_BAD_TOKEN);
        tok = 0;
      }
      if (threadIdx.x == 0) a.block_tok[b * a.L_B + jb] = tok;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int f = (threadIdx.x + u * WORKERS) * 4;
      hv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (f < D) {
        if (a.ingest) {
          const uint2 w = *reinterpret_cast<const uint2*>(a.tok_emb + (size_t)tok * D + f);
          const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
          const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
          hv[u] = make_float4(lo.x, lo.y, hi.x, hi.y);
          __stcg(reinterpret_cast<float4*>(hrow + f), hv[u]);
        } else {
          hv[u] = __ldcg(reinterpret_cast<const float4*>(hrow + f));
        }
      }
    }
    bf16* o = a.x1 + (size_t)b * 2 * D;
    ln_out(hv, D, a.eps, lp, o, o + D, red);
  }
}

// Row reduction for the out|fc2 and prefix GEMMs: h[b] = (residual ? h[b] : 0)
// + bias + the S K-split partials (T tiles) or, with S = 0, the fixed-point
// sums in a.fx (cleared as they are read), then a LayerNorm of the new row:
// LN1 | LN2 -> out (row stride 2D) when lp holds two, else one LN -> out
// (row stride D). One CTA per row.
__device__ void reduce_ln(const TokenStepArgs& a, const Plan& P, float* h, const float* bias, int S,
                          bool residual, const float* g1, const float* b1, const float* g2,
                          const float* b2, bf16* out, float* red) {
  const int D = a.D, B = a.B;
  LnParams lp;
  if (blockIdx.x < B) ln_load(lp, D, g1, b1, g2, b2);
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    float4 hv[4];
    float* hrow = h + (size_t)b * D;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int f = (threadIdx.x + u * WORKERS) * 4;
      hv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (f < D) {
        float4 acc = *reinterpret_cast<const float4*>(bias + f);
        if (residual) acc = f4add(acc, __ldcg(reinterpret_cast<const float4*>(hrow + f)));
        if (S == 0) acc = f4add(acc, fx_take4(a.fx + (size_t)b * D + f));
        const int t = f >> 7, off = f & 127;
#pragma unroll
        for (int sp = 0; sp < MAX_S2; ++sp)
          if (sp < S)
            acc = f4add(acc, __ldcg(reinterpret_cast<const float4*>(
                                 a.p2 + ((size_t)(sp * P.T2 + t) * B + b) * 128 + off)));
        hv[u] = acc;
        __stcg(reinterpret_cast<float4*>(hrow + f), acc);
      }
    }
    if (g2) ln_out(hv, D, a.eps, lp, out + (size_t)b * 2 * D, out + (size_t)b * 2 * D + D, red);
    else ln_out(hv, D, a.eps, lp, out + (size_t)b * D, nullptr, red);
  }
}

// Block step, phase I: block row of each sequence = the L_B token embeddings
// of the completed block concatenated (the fed token is its last), then
// LN1 | LN2 of block layer 0 -> x1.
__device__ void block_ingest_phase(const TokenStepArgs& a, int jb, float* red) {
  const int D = a.D, De = D / a.L_B;
  LnParams lp;
  if (blockIdx.x < a.B) ln_load(lp, D, a.bln1_g, a.bln1_b, a.bln2_g, a.bln2_b);
  for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
    int tok = a.src[b];
    if (tok < 0 || tok >= a.V) {
      if (threadIdx.x == 0) set_status(a.status, ST_BAD_TOKEN);
      tok = 0;
    }
    if (threadIdx.x == 0) a.block_tok[b * a.L_B + jb] = tok;
    float4 hv[4];
    float* hrow = a.h_b + (size_t)b * D;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int f = (threadIdx.x + u * WORKERS) * 4;
      hv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (f < D) {
        // 4 | De: a float4 group never straddles two tokens' pieces
        const int j = f / De, e = f - j * De;
        int t = (j == jb) ? tok : a.block_tok[b * a.L_B + j];
        if (t < 0 || t >= a.V) t = 0;
        const uint2 w = *reinterpret_cast<const uint2*>(a.blk_emb + (size_t)t * De + e);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
        hv[u] = make_float4(lo.x, lo.y, hi.x, hi.y);
        __stcg(reinterpret_cast<float4*>(hrow + f), hv[u]);
      }
    }
    bf16* o = a.x1 + (size_t)b * 2 * D;
    ln_out(hv, D, a.eps, lp, o, o + D, red);
  }
}

// q, k or v (part 0, 1, 2) of head h of row b, head dims lane and lane + 32
// (d_head 64): the K splits of the first GEMM + the bias, rotary on q and k.
__device__ __forceinline__ void head_dims64(const TokenStepArgs& a, const Plan& P, const float* bq, int b,
                                            int h, int part, int pos, float& x0, float& x1) {
  const int lane = threadIdx.x & 31;
  const size_t split_stride = (size_t)P.T1 * a.B * 128;
  const int n0 = part * a.D + h * 64 + lane, n1 = n0 + 32;
  float s0 = bq[n0], s1 = bq[n1];
  const float* p0 = a.p1 + ((size_t)(n0 >> 7) * a.B + b) * 128 + (n0 & 127);
  const float* p1 = a.p1 + ((size_t)(n1 >> 7) * a.B + b) * 128 + (n1 & 127);
#pragma unroll
  for (int sp = 0; sp < MAX_S1; ++sp)
    if (sp < P.S1) {
      s0 += __ldcg(p0 + sp * split_stride);
      s1 += __ldcg(p1 + sp * split_stride);
    }
  if (part < 2 && a.rot > 0) {
    // rotate-half pairs (e, e ^ half), e < rot <= 32: the pair of dim lane
    // is in lane ^ half of the same register
    const int half = a.rot >> 1;
    const float r0 = __shfl_xor_sync(0xffffffffu, s0, half < 32 ? half : 0);
    const float r1 = __shfl_xor_sync(0xffffffffu, s1, half < 32 ? half : 0);
    const int e0 = lane, e1 = lane + 32;
    if (e0 < a.rot) {
      const float2 cs = a.rope_tab[(size_t)pos * half + (e0 & (half - 1))];
      s0 = (e0 & half) ? s0 * cs.x + r0 * cs.y : s0 * cs.x - r0 * cs.y;
    }
    if (e1 < a.rot) {
      const float2 cs = a.rope_tab[(size_t)pos * half + (e1 & (half - 1))];
      s1 = (e1 & half) ? s1 * cs.x + r1 * cs.y : s1 * cs.x - r1 * cs.y;
    }
  }
  x0 = s0;
  x1 = s1;
}

// Block step, phase R1 of block layer l: decode attention of each
// (sequence, head) over its n = pos + 1 block-cache entries, split into
// units of ATT_CH entries spread evenly over the grid: a CTA takes a
// contiguous range of units and each of its warps a contiguous quarter, so a
// warp's units are mostly consecutive chunks of one (sequence, head). A warp
// streams its units' K and V rows with 1-D bulk copies into its ATT_SLOTS
// slots, scores one entry per lane and folds each unit into a running
// (max, sum, weighted V) per (sequence, head); at the end of each run it
// writes one partial and counts the run's units on the (sequence, head)'s
// counter. The warp that completes the count merges the partials into a2.
// The unit holding the newest entry (position pos) computes its k and v from
// the first GEMM's partial sums, appends them to the cache and scores them
// from shared memory. `katt` counts this warp's units over the launch (slot
// and parity bookkeeping). Then GELU(fc1) as in the token layers.
__device__ void block_attention_phase(const TokenStepArgs& a, const Plan& P, int l, int pos, uint8_t* att,
                                      uint64_t* att_bar, float* q_s, int& katt) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int H = a.H, D = a.D;
  const float* bq = layer_ptr(a.bb_qkv1, l, a.layer_stride);
  bf16* kc = a.kb + (size_t)l * a.kb_layer;
  bf16* vc = a.vb + (size_t)l * a.kb_layer;
  const int n = pos + 1;
  const int C = (n + ATT_CH - 1) / ATT_CH;
  const long long U = (long long)a.B * H * C;
  const long long c0 = U * blockIdx.x / gridDim.x, c1 = U * (blockIdx.x + 1) / gridDim.x;
  const long long per_w = (c1 - c0 + 3) / 4;
  const long long wb = c0 + warp * per_w;
  const long long we = (wb + per_w < c1) ? wb + per_w : c1;
  const int nm = we > wb ? (int)(we - wb) : 0;
  uint8_t* wslot = att + (size_t)warp * ATT_SLOTS * ATT_SLOT_BYTES;
  uint64_t* wbar = att_bar + warp * ATT_SLOTS;
  float* qs = q_s + warp * 64;
  auto issue = [&](int i) {  // lane 0
    const long long u = wb + i;
    const int pr = (int)(u / C), j = (int)(u - (long long)pr * C);
    const int e0 = j * ATT_CH;
    const int rows = min(ATT_CH, n - e0);
    const int rc = (e0 + rows == n) ? rows - 1 : rows;  // the newest entry is not in the cache yet
    const int slot = (katt + i) % ATT_SLOTS;
    uint8_t* ks = wslot + (size_t)slot * ATT_SLOT_BYTES;
    const uint32_t bytes = (uint32_t)rc * 128;
    mbar_arrive_expect_tx(&wbar[slot], 2 * bytes);
    if (bytes) {
      const size_t off = ((size_t)pr * a.n_cap + e0) * 64;
      bulk_g2s(ks, kc + off, bytes, &wbar[slot]);
      bulk_g2s(ks + ATT_CH * 128, vc + off, bytes, &wbar[slot]);
    }
  };
  if (lane == 0)
    for (int i = 0; i < nm && i < ATT_SLOTS; ++i) issue(i);

  // the (sequence, head) run in progress
  int cur = -1, run_first = 0, run_len = 0;
  float mr = -INFINITY, lr = 0.f, or0 = 0.f, or1 = 0.f;
  auto flush = [&]() {
    float* part = a.att_part + ((size_t)cur * C + run_first) * ATT_PART;
    if (lane == 0) {
      __stcg(part, mr);
      __stcg(part + 1, lr);
    }
    __stcg(reinterpret_cast<float2*>(part + 2) + lane, make_float2(or0, or1));
    __threadfence();
    int old = 0;
    if (lane == 0) old = atomicAdd(&a.att_cnt[cur], run_len);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old + run_len == C) {
      // every unit of (b, h) is in: merge the runs' partials (slots of units
      // that were not the first of a run hold m = -inf and are skipped)
      __threadfence();
      const int b = cur / H, h = cur - b * H;
      const float* pp = a.att_part + (size_t)cur * C * ATT_PART;
      const float mc = (lane < C) ? __ldcg(pp + (size_t)lane * ATT_PART) : -INFINITY;
      const float lc = (lane < C && mc != -INFINITY) ? __ldcg(pp + (size_t)lane * ATT_PART + 1) : 0.f;
      const float M = warp_max(mc);
      const float wc = (lane < C && mc != -INFINITY) ? exp2f(mc - M) : 0.f;
      const float L = warp_sum(lc * wc);
      float O0 = 0.f, O1 = 0.f;
      for (int c = 0; c < C; ++c) {
        const float w = __shfl_sync(0xffffffffu, wc, c);
        if (w != 0.f) {
          const float2 oc = __ldcg(reinterpret_cast<const float2*>(pp + (size_t)c * ATT_PART + 2) + lane);
          O0 = fmaf(w, oc.x, O0);
          O1 = fmaf(w, oc.y, O1);
        }
      }
      const float inv = 1.f / L;
      *reinterpret_cast<__nv_bfloat162*>(a.a2 + (size_t)b * 5 * D + h * 64 + 2 * lane) =
          __floats2bfloat162_rn(O0 * inv, O1 * inv);
      if (lane == 0) a.att_cnt[cur] = 0;  // ready for the next layer / step
    }
  };

  for (int i = 0; i < nm; ++i) {
    const long long u = wb + i;
    const int pr = (int)(u / C), j = (int)(u - (long long)pr * C);
    if (pr != cur) {
      if (cur >= 0) flush();
      cur = pr;
      run_first = j;
      run_len = 0;
      mr = -INFINITY;
      lr = or0 = or1 = 0.f;
      float q0, q1;
      head_dims64(a, P, bq, pr / H, pr % H, 0, pos, q0, q1);
      __syncwarp();
      qs[lane] = q0 * P.scale;
      qs[lane + 32] = q1 * P.scale;
    } else if (lane == 0) {
      __stcg(a.att_part + ((size_t)pr * C + j) * ATT_PART, -INFINITY);  // not a run's first unit
    }
    const int e0 = j * ATT_CH;
    const int rows = min(ATT_CH, n - e0);
    const bool newest = (e0 + rows == n);
    const int slot = (katt + i) % ATT_SLOTS;
    uint8_t* ks = wslot + (size_t)slot * ATT_SLOT_BYTES;
    uint8_t* vs = ks + ATT_CH * 128;
    float k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
    if (newest) {
      head_dims64(a, P, bq, pr / H, pr % H, 1, pos, k0, k1);
      head_dims64(a, P, bq, pr / H, pr % H, 2, pos, v0, v1);
    }
    mbar_wait_bounded(&wbar[slot], ((katt + i) / ATT_SLOTS) & 1, a.status);
    if (newest) {
      const bf16 kb0 = __float2bfloat16_rn(k0), kb1 = __float2bfloat16_rn(k1);
      const bf16 vb0 = __float2bfloat16_rn(v0), vb1 = __float2bfloat16_rn(v1);
      const size_t off = ((size_t)pr * a.n_cap + pos) * 64;
      kc[off + lane] = kb0;
      kc[off + lane + 32] = kb1;
      vc[off + lane] = vb0;
      vc[off + lane + 32] = vb1;
      bf16* kr = reinterpret_cast<bf16*>(ks + (size_t)(rows - 1) * 128);
      bf16* vr = reinterpret_cast<bf16*>(vs + (size_t)(rows - 1) * 128);
      kr[lane] = kb0;
      kr[lane + 32] = kb1;
      vr[lane] = vb0;
      vr[lane + 32] = vb1;
    }
    __syncwarp();
    // scores, one entry per lane; the word order is rotated per lane so that
    // the 32 lanes read 32 different banks
    float sc = -INFINITY;
    if (lane < rows) {
      const uint32_t* kr = reinterpret_cast<const uint32_t*>(ks + (size_t)lane * 128);
      float acc = 0.f;
#pragma unroll 8
      for (int w = 0; w < 32; ++w) {
        const int ww = (w + lane) & 31;
        const uint32_t kw = kr[ww];
        const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw));
        acc = fmaf(qs[2 * ww], kf.x, acc);
        acc = fmaf(qs[2 * ww + 1], kf.y, acc);
      }
      sc = acc;
    }
    const float mx = fmaxf(warp_max(sc), mr);
    const float pj = (lane < rows) ? exp2f(sc - mx) : 0.f;
    const float cf = exp2f(mr - mx);
    lr = lr * cf + warp_sum(pj);
    or0 *= cf;
    or1 *= cf;
    mr = mx;
    // weighted V for head dims 2*lane, 2*lane + 1
    for (int jj = 0; jj < rows; ++jj) {
      const float pw = __shfl_sync(0xffffffffu, pj, jj);
      const uint32_t vw = reinterpret_cast<const uint32_t*>(vs + (size_t)jj * 128)[lane];
      const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vw));
      or0 = fmaf(pw, vf.x, or0);
      or1 = fmaf(pw, vf.y, or1);
    }
    ++run_len;
    // this slot's generic reads are done before the next bulk copy into it
    fence_proxy_async();
    __syncwarp();
    if (lane == 0 && i + ATT_SLOTS < nm) issue(i + ATT_SLOTS);
  }
  if (cur >= 0) flush();
  katt += nm;
  gelu_fc1(a, P, bq);
}

__device__ __forceinline__ void better(float& v, int& i, float ov, int oi) {
  if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
}

// Per-row argmax over the warp's 32 features for 32 rows held one per
// register (v[r], index idx for all): a transposing butterfly -- at each of
// the 5 levels a lane keeps half of its rows and trades the other half with
// its partner -- leaves row `lane` reduced over the 32 lanes in 31 exchanges.
__device__ __forceinline__ void warp_argmax32(float* v, int* ix) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16, h = 16; o > 0; o >>= 1, h >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float sv = up ? v[i] : v[i + h];
      const int si = up ? ix[i] : ix[i + h];
      const float rv = __shfl_xor_sync(0xffffffffu, sv, o);
      const int ri = __shfl_xor_sync(0xffffffffu, si, o);
      float kv = up ? v[i + h] : v[i];
      int ki = up ? ix[i + h] : ix[i];
      better(kv, ki, rv, ri);
      v[i] = kv;
      ix[i] = ki;
    }
  }
}

// GL epilogue of vocab tile t: logits (optional) and the tile's argmax per row
// Greedy argmax through one 64-bit atomicMax per row and vocabulary tile: the
// logit's order-preserving bits above (-0 counted as +0), 2^32 - 1 - id below,
// so the largest logit wins and the lowest id among equal ones.
__device__ __forceinline__ unsigned long long argmax_key(float v, int id) {
  const unsigned u = __float_as_uint(v + 0.0f);
  const unsigned ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)ord << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)id);
}

__device__ void lm_epilogue(uint32_t tbuf, int t, const TokenStepArgs& a, int Bp, float2 (*s_arg)[MAX_B]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t trow = tbuf + ((uint32_t)(warp * 32) << 16);
  const int n = t * 128 + warp * 32 + lane;
  for (int c0 = 0; c0 < Bp; c0 += 32) {
    float v[32];
    int ix[32];
    tc::tmem_ld16(trow + c0, v);
    if (c0 + 16 < Bp) tc::tmem_ld16(trow + c0 + 16, v + 16);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int m = c0 + j;
      if (a.logits && m < a.B && n < a.V) a.logits[(size_t)m * a.V + n] = v[j];
      if (n >= a.V || m >= a.B) v[j] = -INFINITY;
      ix[j] = n;
    }
    warp_argmax32(v, ix);
    if (c0 + lane < a.B) s_arg[warp][c0 + lane] = make_float2(v[0], __int_as_float(ix[0]));
  }
  tc::fence_before();
  wsync();
  if (threadIdx.x < a.B) {
    const int r = threadIdx.x;
    float2 best = s_arg[0][r];
#pragma unroll
    for (int w = 1; w < 4; ++w) {
      const float2 o = s_arg[w][r];
      if (o.x > best.x || (o.x == best.x && __float_as_int(o.y) < __float_as_int(best.y))) best = o;
    }
    atomicMax(a.arg_key + r, argmax_key(best.x, __float_as_int(best.y)));
  }
  wsync();  // s_arg is reused by the next tile
}

__device__ void lm_phase(const TokenStepArgs& a, const Plan& P, const CUtensorMap* mxf, uint8_t* act,
                         uint32_t tmem, const Sync& y, int& na, int& nu, float2 (*s_arg)[MAX_B]) {
  const int G = gridDim.x;
  if ((int)blockIdx.x >= P.TL) return;
  if (threadIdx.x == 0) load_act(mxf, act, 0, P.nkbL, P.Bp, y.act_full);
  ++na;
  for (int t = blockIdx.x; t < P.TL; t += G) {
    const int buf = nu & 1;
    mbar_wait_bounded(&y.acc_full[buf], (nu >> 1) & 1, a.status);
    tc::fence_after();
    lm_epilogue(tmem + (uint32_t)(buf * 64), t, a, P.Bp, s_arg);
    mbar_arrive(&y.acc_empty[buf]);  // lm_epilogue ended with the tcgen05 fence + barrier
    ++nu;
  }
}

// AR: greedy id per row from the tile partials (lowest id on ties)
// The last CTA out of a completed step: each row's id from its argmax key (the
// keys reset for the next launch), then the position advances. After an abort
// only the keys are reset.
__device__ void finish_step(const TokenStepArgs& a) {
  const bool aborted = *reinterpret_cast<volatile unsigned*>(&a.bar[2]) != 0u;
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    const unsigned long long k = atomicExch(a.arg_key + b, 0ull);
    if (!aborted) a.next[b] = (int)(0xFFFFFFFFu - (unsigned)(k & 0xFFFFFFFFull));
  }
  if (threadIdx.x == 0 && !aborted) {
    const int t = a.dstate[0] + 1;
    a.dstate[0] = t;
    a.dstate[1] = t % a.L_B;
    a.dstate[2] = t / a.L_B;
  }
}

// BLOCK = false: token steps only (no block-step code, fewer registers)
template <bool BLOCK>
__global__ void __launch_bounds__(THREADS, 1)
token_step_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mo,
                  const __grid_constant__ CUtensorMap ml, const __grid_constant__ CUtensorMap mx1,
                  const __grid_constant__ CUtensorMap ma2, const __grid_constant__ CUtensorMap mxf,
                  const __grid_constant__ CUtensorMap mqb, const __grid_constant__ CUtensorMap mob,
                  const __grid_constant__ CUtensorMap mp, const TokenStepArgs a, const Plan P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint8_t* ring = smem;
  uint8_t* act = smem + (size_t)P.stages * TILE_BYTES;
  __shared__ __align__(8) uint64_t full[MAX_STAGES], empty[MAX_STAGES], act_full, acc_full[2], acc_empty[2];
  __shared__ uint32_t tmem_slot;
  __shared__ float red[4];
  __shared__ float2 s_arg[4][MAX_B];
  __shared__ volatile int s_abort;
  __shared__ int s_last;
  __shared__ __align__(8) uint64_t att_bar[4 * ATT_SLOTS];  // block-step attention slots
  __shared__ float q_s[4 * 64];

  const int warp = threadIdx.x >> 5;
  const int Nb = (BLOCK && a.block) ? a.Nb : 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < P.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 4 * ATT_SLOTS; ++i) mbar_init(&att_bar[i], 1);
    mbar_init(&act_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], WORKERS);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, TMEM_COLS);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_slot;
  const Sync y{full, empty, &act_full, acc_full, acc_empty};
  pdl_trigger();

  if (warp == 4) {
    // weights do not depend on earlier kernels: no wait before streaming them
    if ((threadIdx.x & 31) == 0)
      producer(&mq, &mo, &ml, &mqb, &mob, &mp, P, a.Nt, Nb, ring, full, empty, a.status, &s_abort,
               a.wait_cycles);
  } else if (warp == 5) {
    if ((threadIdx.x & 31) == 0) mma_issuer(P, a.Nt, Nb, ring, act, tmem, y, a.status, &s_abort, a.wait_cycles);
  } else {
    pdl_wait();
    const int G = gridDim.x;
    const int pos = pos_base(a.pos);  // read before the first barrier: the last phase advances it
    const int jb = a.dstate[1];
    unsigned nb = 0;
    int na = 0, nu = 0;
    bool ok;
    const int D = a.D;
    if (BLOCK && Nb > 0) {
      // block step: block embedding, the block-decoder layers at block
      // position dstate[2], LN_b, the prefix projection (-> h, LN1 | LN2 of
      // token layer 0)
      const int bpos = a.dstate[2];
      int katt = 0;
      block_ingest_phase(a, jb, red);
      ok = grid_sync(a, ++nb * G, &s_abort);
      for (int l = 0; ok && l < Nb; ++l) {
        gemm_phase(P, P.T1, P.S1, P.nkb1, &mx1, [=](int t) { return t * 128 < 3 * D ? 0 : D; }, a.B, a.p1,
                   act, tmem, y, na, nu, a.status);
        if (!(ok = grid_sync(a, ++nb * G, &s_abort))) break;
        block_attention_phase(a, P, l, bpos, act, att_bar, q_s, katt);
        if (!(ok = grid_sync(a, ++nb * G, &s_abort))) break;
        // the out|fc2 splits go into the fixed-point accumulators by L2 reductions
        gemm_phase(P, P.T2, P.S2, P.nkb2, &ma2, [](int) { return 0; }, a.B, a.p2, act, tmem, y, na, nu,
                   a.status, a.fx, D);
        if (!(ok = grid_sync(a, ++nb * G, &s_abort))) break;
        if (l + 1 < Nb)
          reduce_ln(a, P, a.h_b, layer_ptr(a.bb_o2, l, a.layer_stride), 0, true,
                    layer_ptr(a.bln1_g, l + 1, a.layer_stride), layer_ptr(a.bln1_b, l + 1, a.layer_stride),
                    layer_ptr(a.bln2_g, l + 1, a.layer_stride), layer_ptr(a.bln2_b, l + 1, a.layer_stride),
                    a.x1, red);
        else
          reduce_ln(a, P, a.h_b, layer_ptr(a.bb_o2, l, a.layer_stride), 0, true, a.lnb_g, a.lnb_b,
                    nullptr, nullptr, a.xf, red);
        ok = grid_sync(a, ++nb * G, &s_abort);
      }
      if (ok) {
        gemm_phase(P, P.T2, P.Sp, P.nkbp, &mxf, [](int) { return 0; }, a.B, a.p2, act, tmem, y, na, nu,
                   a.status);
        ok = grid_sync(a, ++nb * G, &s_abort);
      }
      if (ok) {
        reduce_ln(a, P, a.h, a.b_prefix, P.Sp, false, a.ln1_g, a.ln1_b, a.ln2_g, a.ln2_b, a.x1, red);
        ok = grid_sync(a, ++nb * G, &s_abort);
      }
    } else {
      ingest_phase(a, jb, red);
      ok = grid_sync(a, ++nb * G, &s_abort);
    }
    for (int l = 0; ok && l < a.Nt; ++l) {
      // G1: q|k|v tiles read LN1(h), fc1 tiles LN2(h)
      gemm_phase(P, P.T1, P.S1, P.nkb1, &mx1, [=](int t) { return t * 128 < 3 * D ? 0 : D; }, a.B, a.p1,
                 act, tmem, y, na, nu, a.status);
      if (!(ok = grid_sync(a, ++nb * G, &s_abort))) break;
      r1_phase(a, P, l, pos);
      if (!(ok = grid_sync(a, ++nb * G, &s_abort))) break;
      gemm_phase(P, P.T2, P.S2, P.nkb2, &ma2, [](int) { return 0; }, a.B, a.p2, act, tmem, y, na, nu,
                 a.status, a.fx, D);
      if (!(ok = grid_sync(a, ++nb * G, &s_abort))) break;
      r2_phase(a, P, l, red);
      ok = grid_sync(a, ++nb * G, &s_abort);
    }
    // the LM tiles' epilogues fold each row's best (logit, id) into
    // a.arg_key; the last CTA out turns the keys into ids (finish_step)
    if (ok) lm_phase(a, P, &mxf, act, tmem, y, na, nu, s_arg);
    // workers that stop early (abort) release the MMA warp's waits
    if (!ok && threadIdx.x == 0) s_abort = 1;
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_free(tmem, TMEM_COLS);
  // every CTA counts itself out only after its last barrier wait and its
  // argmax updates (ordered before thread 0 by the CTA barrier above)
  if (threadIdx.x == 0) s_last = grid_exit(a.bar) ? 1 : 0;
  __syncthreads();
  if (s_last) finish_step(a);
}

// ---- host side -----------------------------------------------------------------
typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                             CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                             CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

// bf16 weight boxes of 64 K x 128 rows, 128-byte swizzle, zero fill past the
// last row; rank 3 adds the layer dimension (stride in bytes)
bool weight_map(CUtensorMap* m, const void* base, long long K, long long rows, long long layers,
                long long layer_stride) {
  EncodeFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)layers};
  cuuint64_t str[2] = {(cuuint64_t)K * 2, (cuuint64_t)layer_stride};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const cuuint32_t rank = layers > 0 ? 3 : 2;
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, str, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 activation rows [rows, cols] (row-major, ld = cols): boxes of 64
// columns x box_rows rows, 128-byte swizzle, zero fill for rows >= rows
bool act_map(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows) {
  EncodeFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t str[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, str, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Device {
  int sms = 0;
  size_t smem_max = 0;  // dynamic shared memory per CTA
  bool ready = false;
};

// per device: kernel attributes apply to the current device only
Device& device() {
  static Device per_dev[MAX_DEVICES];
  static Device none;
  const int dev = current_device();
  Device& d = dev >= 0 ? per_dev[dev] : none;
  if (!d.ready) {
    int optin = 0;
    cudaFuncAttributes fa;
    if (dev < 0 || cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, token_step_kernel<true>) != cudaSuccess)
      return d;
    // both instantiations declare the same static shared memory
    d.smem_max = (size_t)optin - fa.sharedSizeBytes;
    if (cudaFuncSetAttribute(token_step_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)d.smem_max) != cudaSuccess ||
        cudaFuncSetAttribute(token_step_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)d.smem_max) != cudaSuccess)
      return d;
    d.ready = true;
  }
  return d;
}

// largest divisor of n that is <= cap
int divisor_at_most(int n, int cap) {
  for (int s = cap < n ? cap : n; s > 1; --s)
    if (n % s == 0) return s;
  return 1;
}

bool make_plan(int B, int D, int dh, int V, int sms, size_t smem_max, Plan* P, size_t* smem,
               bool block = false) {
  Plan p{};
  p.Bp = (B + 15) / 16 * 16;
  p.T1 = 7 * D / 128;
  p.T2 = D / 128;
  p.TL = (V + 127) / 128;
  const int kb1 = D / 64, kb2 = 5 * D / 64;
  int c1 = sms / p.T1;
  if (c1 > MAX_S1) c1 = MAX_S1;
  int c2 = sms / p.T2;
  if (c2 > MAX_S2) c2 = MAX_S2;
  p.S1 = divisor_at_most(kb1, c1 < 1 ? 1 : c1);
  p.S2 = divisor_at_most(kb2, c2 < 1 ? 1 : c2);
  p.nkb1 = kb1 / p.S1;
  p.nkb2 = kb2 / p.S2;
  p.nkbL = kb1;
  // prefix projection of block steps: N = D, K = D
  int cp = sms / p.T2;
  if (cp > MAX_S2) cp = MAX_S2;
  p.Sp = divisor_at_most(kb1, cp < 1 ? 1 : cp);
  p.nkbp = kb1 / p.Sp;
  // the activation buffer holds the LM head's whole input (the largest unit)
  // and, on block steps, the decode-attention slots of the four worker warps
  int act_kb = p.nkbL;
  if (p.nkb1 > act_kb) act_kb = p.nkb1;
  if (p.nkb2 > act_kb) act_kb = p.nkb2;
  size_t act = (size_t)act_kb * p.Bp * 128;
  if (block && act < (size_t)ATT_BYTES) act = ATT_BYTES;
  if (smem_max < act + 1024 + 4 * (size_t)TILE_BYTES) return false;
  int st = (int)((smem_max - act - 1024) / TILE_BYTES);
  p.stages = st > MAX_STAGES ? MAX_STAGES : st;
  p.scale = 1.4426950408889634f / sqrtf((float)dh);
  *P = p;
  *smem = (size_t)p.stages * TILE_BYTES + act + 1024;
  return true;
}

}  // namespace

int token_step_supported(int dt, int B, int D, int H, int rot, int V, int Nt, int P_prefix, int l_cap) {
  if (dt != DT_BF16 || B < 1 || B > MAX_B || Nt < 1 || P_prefix != 1 || V < 1 || l_cap > MAX_WIN) return 0;
  if (D % 128 || D > 2048 || H < 1 || D % H) return 0;
  const int dh = D / H;
  if (dh != 32 && dh != 64 && dh != 128) return 0;
  if (rot) {
    const int half = rot / 2;
    if ((rot & 1) || rot > dh || half > 16 || (half & (half - 1))) return 0;
  }
  if (!encode_fn()) return 0;
  Device& d = device();
  if (!d.ready) return 0;
  Plan p;
  size_t smem;
  return make_plan(B, D, dh, V, d.sms, d.smem_max, &p, &smem) ? 1 : 0;
}

int token_step_block_supported(int dt, int B, int D, int H, int rot, int V, int Nt, int Nb, int P_prefix,
                               int l_cap, int n_cap, int L_B) {
  if (!token_step_supported(dt, B, D, H, rot, V, Nt, P_prefix, l_cap)) return 0;
  if (Nb < 1 || D / H != 64 || n_cap < 1 || n_cap > ATT_CH * ATT_MAX_CHUNKS) return 0;
  // a float4 of the block embedding never straddles two tokens' pieces
  if (L_B < 1 || D % L_B || (D / L_B) % 4) return 0;
  return 1;
}

size_t token_step_scratch_floats(int B, int D, int which, int H, int n_cap) {
  // upper bounds over every plan: T1 * MAX_S1 and T2 * MAX_S2 partial tiles
  if (B > MAX_B) B = MAX_B;
  if (which == 3) {
    const int C = (n_cap + ATT_CH - 1) / ATT_CH;
    return (size_t)B * H * C * ATT_PART;
  }
  return which == 1 ? (size_t)(7 * D / 128) * MAX_S1 * B * 128 : (size_t)(D / 128) * MAX_S2 * B * 128;
}

cudaError_t launch_token_step(const TokenStepArgs& a, const void* w_qkv1, const void* w_o2,
                              const void* w_lm, const void* w_qkv1_b, const void* w_o2_b,
                              const void* w_prefix, cudaStream_t s) {
  if (!token_step_supported(DT_BF16, a.B, a.D, a.H, a.rot, a.V, a.Nt, 1, a.l_cap)) return cudaErrorNotSupported;
  if (a.block && (!w_qkv1_b || !w_o2_b || !w_prefix ||
                  !token_step_block_supported(DT_BF16, a.B, a.D, a.H, a.rot, a.V, a.Nt, a.Nb, 1, a.l_cap,
                                              a.n_cap, a.L_B)))
    return cudaErrorNotSupported;
  if (!a.fx || (reinterpret_cast<uintptr_t>(a.fx) & 15) || !a.arg_key) return cudaErrorInvalidValue;
  Device& d = device();
  Plan P;
  size_t smem;
  if (!make_plan(a.B, a.D, a.dh, a.V, d.sms, d.smem_max, &P, &smem, a.block != 0)) return cudaErrorNotSupported;
  CUtensorMap mq, mo, ml;
  // one layer: any stride at least the layer's own size satisfies the encoder
  const long long lsq = a.Nt > 1 ? a.layer_stride : 14LL * a.D * a.D;
  const long long lso = a.Nt > 1 ? a.layer_stride : 10LL * a.D * a.D;
  if (!weight_map(&mq, w_qkv1, a.D, 7LL * a.D, a.Nt, lsq) || !weight_map(&mo, w_o2, 5LL * a.D, a.D, a.Nt, lso) ||
      !weight_map(&ml, w_lm, a.D, a.V, 0, 0))
    return cudaErrorInvalidValue;
  CUtensorMap mx1, ma2, mxf;
  if (!act_map(&mx1, a.x1, a.B, 2LL * a.D, P.Bp) || !act_map(&ma2, a.a2, a.B, 5LL * a.D, P.Bp) ||
      !act_map(&mxf, a.xf, a.B, a.D, P.Bp))
    return cudaErrorInvalidValue;
  // block-step weights (token steps pass the token maps; they are not read)
  CUtensorMap mqb = mq, mob = mo, mp = ml;
  if (a.block) {
    const long long bsq = a.Nb > 1 ? a.layer_stride : 14LL * a.D * a.D;
    const long long bso = a.Nb > 1 ? a.layer_stride : 10LL * a.D * a.D;
    if (!weight_map(&mqb, w_qkv1_b, a.D, 7LL * a.D, a.Nb, bsq) ||
        !weight_map(&mob, w_o2_b, 5LL * a.D, a.D, a.Nb, bso) || !weight_map(&mp, w_prefix, a.D, a.D, 0, 0))
      return cudaErrorInvalidValue;
  }
  // every CTA must be resident at once (grid barriers): one per SM
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, a.block ? token_step_kernel<true> : token_step_kernel<false>, THREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(d.sms, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  // cooperative: the driver guarantees that every CTA is resident at once
  // (the grid barriers rely on it) or refuses the launch
  cudaLaunchAttribute attr[3];
  int na = 0;
  attr[na].id = cudaLaunchAttributeCooperative;
  attr[na++].val.cooperative = 1;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na++].val.programmaticStreamSerializationAllowed = 1;
  }
  if (a.l2_window_bytes > 0) {
    // the re-read regions (LM head, local caches) persist in L2
    attr[na].id = cudaLaunchAttributeAccessPolicyWindow;
    attr[na].val.accessPolicyWindow.base_ptr = a.l2_window_base;
    attr[na].val.accessPolicyWindow.num_bytes = a.l2_window_bytes;
    attr[na].val.accessPolicyWindow.hitRatio = a.l2_hit_ratio;
    attr[na].val.accessPolicyWindow.hitProp = cudaAccessPropertyPersisting;
    attr[na++].val.accessPolicyWindow.missProp = cudaAccessPropertyStreaming;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (a.block) e = cudaLaunchKernelEx(&cfg, token_step_kernel<true>, mq, mo, ml, mx1, ma2, mxf, mqb, mob, mp, a, P);
  else e = cudaLaunchKernelEx(&cfg, token_step_kernel<false>, mq, mo, ml, mx1, ma2, mxf, mqb, mob, mp, a, P);
  note_launch();
  return e;
}

}  // namespace bt
