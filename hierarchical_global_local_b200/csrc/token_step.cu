// token_step.cu -- the token-decoder half of a decode step as one persistent
// kernel (bf16, batch <= 64): every token-decoder layer, the final LayerNorm,
// the LM head and the greedy argmax.
//
// Block Transformer (Ho et al., "Block Transformer: Global-to-Local Language
// Modeling for Fast Inference"), section 2.4 / explainer §3.4 "The Token
// Decoder": a small transformer over [prefix; tokens of the current block]
// that reads every one of its weights for a single new row per sequence.
// The step is a chain of weight-streaming matrix products separated by
// all-to-all exchanges; its cost is the latency of those exchanges.
//
// Work decomposition ("weights as A": M = 128 output features per tile,
// N = the batch padded to a multiple of 16, K in 64-wide swizzled blocks):
//   G1 units  the 7D/128 tiles of [W_qkv; W_1] (q | k | v | fc1), each
//             split in S1 K ranges: one (tile, split) per CTA, CTAs
//             [0, N1)
//   G2 units  the D/128 tiles of [W_o | W_2], each split in S2 K ranges:
//             one (tile, split) per CTA, the CTAs at the top of the grid
// so that the two sets are disjoint while they fit: every CTA then owns one
// unit per layer and its weight producer streams the next layer's unit
// while the other set computes.
//
// Per layer, with no grid-wide barrier:
//   G1  wait until every row of h and its LayerNorm statistics are written
//       (a counter the G2 units of the previous layer, or the ingest, bump);
//       normalise the unit's K range of every row (LN1 for q|k|v tiles, LN2
//       for fc1 tiles) straight into the MMA operand in shared memory; MMA;
//       store the fp32 partial tile; wait for the other splits of the same
//       tile group; reduce this CTA's share of the rows:
//         fc1 tiles: bias + GELU -> a2[:, D + ...]
//         q|k|v:     the three tiles of a head group (q, k and v of the same
//                    heads) form one group; its 3*S1 CTAs split the rows;
//                    bias, rotary on q and k, k and v appended to the local
//                    cache, attention over the local window -> a2[:, head]
//       and count the group done.
//   G2  wait for the G1 groups whose a2 columns it reads; TMA the a2 K range;
//       MMA; store the partial; wait for the tile's other splits; reduce its
//       share of the rows: h += sum + b_o + b_2, then per-(row, tile) mean and
//       sum of squared deviations of the new h for the next LayerNorm; count.
// Then: final LayerNorm rows -> xf; the LM head over the vocabulary tiles
// (every CTA; tiles prefetched into L2 during the layers); greedy argmax per
// row (lowest id on ties) and the step state advanced.
//
// All CTAs are resident at once (one per SM, cooperative launch), so every
// wait on a counter ends once its producers run; each wait is bounded by the
// launch's wait limit and a wait that runs out sets ST_WAIT_TIMEOUT and an
// abort word that every other wait sees, so the kernel always returns.
#include <cuda.h>
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "gridsync.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace bt {

namespace {

constexpr int WORKERS = 128;               // warps 0-3 (TMEM lanes 0-127)
constexpr int THREADS = WORKERS + 64;      // warp 4: TMA producer, warp 5: MMA issuer
constexpr int BOX = 128 * 64 * 2;          // one weight box: 128 rows x 64 K (bf16)
constexpr int MAX_STAGES = 16;
constexpr int MAX_KB = 32;                 // K blocks of a staged activation operand (D / 64 <= 32)
constexpr int MAX_B = 64;
constexpr int MAX_WIN = 16;                // local-window rows (P + L_B - 1)
constexpr int TMEM_COLS = 128;             // two accumulators of up to 64 columns
constexpr int PRODUCER_SLEEP_NS = 128;
constexpr int MMA_SLEEP_NS = 32;
// K splits of a G1 tile (D / 128 blocks of 64 each) and of a G2 tile
// (D / 128 blocks each): compile-time, so that the reductions over the
// splits issue all their loads at once
constexpr int S1 = 2;
constexpr int S2 = 10;

// counter slots (one 128-byte line each)
enum : int {
  C_ARRIVED = 0,   // CTAs that have read the step position
  C_H = 1,         // rows of h (+ statistics) written: ingest CTAs, then G2 units
  C_FINAL = 2,     // final-LayerNorm CTAs done
  C_LM = 3,        // LM-head CTAs done
  C_EXIT = 4,      // CTAs out (the last resets every counter)
  C_ABORT = 5,     // set by a wait that ran out
  C_G1P = 8,       // [T1] partials of G1 tile t stored (S1 per layer)
  // then C_A2 = C_G1P + T1: [5 D / 128] a2 column blocks written (block j <
  // D/128: head group j, 3 S1 per layer; else fc1 tile j - D/128, S1 per
  // layer), then C_G2P = C_A2 + 5 D / 128: [T2] G2 partials (S2 per layer)
};

struct Plan {
  int Bp;                 // batch padded to a multiple of 16 (MMA N)
  int T1, T2, TL;         // tiles: 7D/128, D/128, ceil(V/128)
  int S1, S2;             // K splits of G1 and G2 tiles
  int kb1, kb2, kbL;      // 64-wide K blocks per unit: D/(64 S1), 5D/(64 S2), D/64
  int N1, N2;             // G1 / G2 units (T1*S1, T2*S2)
  int g2_base;            // first CTA of the G2 units (units run from the top)
  int HG;                 // head groups: D/128 (q, k and v tiles of the same heads)
  int n_ing;              // CTAs that ingest rows (min(B, grid))
  int n_lm;               // CTAs with at least one vocabulary tile (min(TL, grid))
  int c_a2, c_g2p, n_slots;  // counter slots (see the enum)
  int stages;             // weight ring depth
  int act_bytes;          // activation buffer
  float scale;            // log2(e) / sqrt(d_head)
};

__device__ __forceinline__ void wsync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ unsigned* ctr(unsigned* base, int slot) { return base + (size_t)slot * 32; }

template <typename T>
__device__ __forceinline__ const T* layer_ptr(const T* base, int l, long long stride) {
  return reinterpret_cast<const T*>(reinterpret_cast<const uint8_t*>(base) + (long long)l * stride);
}

// Worker side: thread 0 adds one to a counter (release: the CTA's writes
// before the preceding worker barrier are visible to whoever acquires it).
__device__ __forceinline__ void signal(unsigned* c) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(c) : "memory");
}

// Thread 0 of the workers waits until *c >= target (bounded; see the file
// comment). Returns false once the step has been aborted.
__device__ bool wait_count(const TokenStepArgs& a, unsigned* c, unsigned target, volatile int* s_abort) {
  if (*s_abort) return false;
  const long long t0 = clock64();
  int n = 0;
  while (ld_acquire_gpu(c) < target) {
    if ((++n & 31) == 0) {
      if (ld_acquire_gpu(ctr(a.bar, C_ABORT)) != 0u) { *s_abort = 1; return false; }
      if (clock64() - t0 > a.wait_cycles) {
        atomicExch(ctr(a.bar, C_ABORT), 1u);
        set_status(a.status, ST_WAIT_TIMEOUT);
        *s_abort = 1;
        return false;
      }
    }
  }
  return true;
}

// All workers: thread 0 waits, then the others learn the outcome. The
// leading fence orders data written through the generic proxy before any
// later TMA read of it.
__device__ __forceinline__ bool workers_wait(const TokenStepArgs& a, unsigned* c, unsigned target,
                                             volatile int* s_abort) {
  if (threadIdx.x == 0) wait_count(a, c, target, s_abort);
  wsync();
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return !*s_abort;
}

// Workers' writes of a phase are done: the worker barrier orders every
// worker's writes before thread 0's release add (cumulative), which makes
// them visible to whoever acquires the count.
__device__ __forceinline__ void workers_signal(unsigned* c) {
  asm volatile("fence.proxy.async.global;" ::: "memory");  // consumers may read through TMA
  wsync();
  if (threadIdx.x == 0) signal(c);
}

// mbarrier wait of the producer / MMA warps: backs off between polls; gives
// up when the CTA has aborted or the launch's wait limit has passed
__device__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const TokenStepArgs& a, volatile int* s_abort,
                              int sleep_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  int n = 0;
  while (!mbar_try_wait(bar, parity)) {
    __nanosleep(sleep_ns);
    if ((++n & 63) == 0) {
      if (*s_abort) return false;
      if (clock64() - t0 > a.wait_cycles) {
        set_status(a.status, ST_WAIT_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__device__ __forceinline__ uint2 pack_bf16x4(float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  return u;
}

// Mean and reciprocal standard deviation of row b from its T2 per-tile
// (mean, sum of squared deviations) pairs over 128 features each (Chan's
// pairwise combination; equal tile sizes).
__device__ __forceinline__ void row_stats(const float2* hs, int T2, float eps, float& mu, float& rstd) {
  constexpr int MAXT = 16;  // D <= 2048
  float2 ps[MAXT];
#pragma unroll
  for (int t = 0; t < MAXT; ++t)
    if (t < T2) ps[t] = __ldcg(hs + t);
  float m = 0.f, m2 = 0.f;
#pragma unroll
  for (int t = 0; t < MAXT; ++t) {
    if (t >= T2) break;
    const float2 p = ps[t];
    const float n_a = 128.f * (float)t, n = n_a + 128.f;
    const float delta = p.x - m;
    m += delta * (128.f / n);
    m2 += p.y + delta * delta * (n_a * 128.f / n);
  }
  mu = m;
  rstd = rsqrtf(m2 / (128.f * (float)T2) + eps);
}

// ---- unit bookkeeping (identical on every CTA and warp) ---------------------
// G1 unit w1 = tile * S1 + split runs on CTA w1 % G; G2 unit w2 = tile * S2 +
// split on CTA (g2_base + w2) % G; LM tile t on CTA t % G. A CTA runs, per
// layer, its G1 units then its G2 units in ascending order.
__device__ __forceinline__ int first_g1(const Plan& P, int c) { return c; }
__device__ __forceinline__ int first_g2(const Plan& P, int c, int G) {
  return ((c - P.g2_base) % G + G) % G;
}

// ---- TMA producer (warp 4, one thread) ----------------------------------------
__device__ void producer(const CUtensorMap* mq, const CUtensorMap* mo, const CUtensorMap* ml, const Plan& P,
                         int Nt, uint8_t* ring, uint64_t* full, uint64_t* empty, const TokenStepArgs& a,
                         volatile int* s_abort) {
  const int G = gridDim.x, c = blockIdx.x;
  int it = 0;
  bool stop = false;
  uint64_t first;
  // weights, LM head included, are read once per step: keep them from
  // evicting the activations, partial sums and the local window that the
  // phases exchange through L2
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(first));
  auto load = [&](const CUtensorMap* m, int x, int y, int z, bool three) {
    if (stop) return;
    const int s = it % P.stages;
    if (it >= P.stages &&
        !wait_or_abort(&empty[s], ((it / P.stages) + 1) & 1, a, s_abort, PRODUCER_SLEEP_NS)) {
      stop = true;
      return;
    }
    mbar_arrive_expect_tx(&full[s], BOX);
    if (three) tc::tma_load_3d_hint(ring + (size_t)s * BOX, m, x, y, z, &full[s], first);
    else tc::tma_load_2d_hint(ring + (size_t)s * BOX, m, x, y, &full[s], first);
    ++it;
  };
  for (int l = 0; l < Nt && !stop; ++l) {
    for (int w = first_g1(P, c); w < P.N1 && !stop; w += G) {
      const int t = w / P.S1, sp = w % P.S1;
      for (int kb = 0; kb < P.kb1; ++kb) load(mq, (sp * P.kb1 + kb) * 64, t * 128, l, true);
    }
    for (int w = first_g2(P, c, G); w < P.N2 && !stop; w += G) {
      const int t = w / P.S2, sp = w % P.S2;
      for (int kb = 0; kb < P.kb2; ++kb) load(mo, (sp * P.kb2 + kb) * 64, t * 128, l, true);
    }
  }
  for (int t = c; t < P.TL && !stop; t += G)
    for (int kb = 0; kb < P.kbL; ++kb) load(ml, kb * 64, t * 128, 0, false);
  // copies still in flight (none on a normal run: the issuer consumed them)
  const int from = it > P.stages ? it - P.stages : 0;
  for (int j = from; j < it; ++j) mbar_wait_bounded(&full[j % P.stages], (j / P.stages) & 1, a.status, a.wait_cycles);
}

// Shared-memory barriers of the worker / MMA hand-off.
struct Sync {
  uint64_t* full;       // [stages] weight box landed
  uint64_t* empty;      // [stages] weight box consumed
  uint64_t* act_kb;     // [MAX_KB] K block kb of the unit's activations staged (1 arrival + TMA bytes)
  uint64_t* acc_full;   // [2] accumulator ready (tcgen05.commit)
  uint64_t* acc_empty;  // [2] accumulator drained (128 worker arrivals)
};

// One thread: the MMAs of one unit, `ntiles` row tiles of 128 accumulating
// over nkb K blocks (ring boxes in tile-minor order per K block) into TMEM
// columns tmem_d + i * Bp, then a commit to `done`.
__device__ bool issue_unit(const Plan& P, int nkb, int ntiles, uint8_t* ring, const uint8_t* act, uint32_t tmem_d,
                           const Sync& y, uint64_t* done, int& it, int* act_uses, bool need_act,
                           const TokenStepArgs& a, volatile int* s_abort) {
  const uint32_t idesc = tc::idesc_bf16_m128(P.Bp);
  for (int kb = 0; kb < nkb; ++kb) {
    // K block kb of the activations: MMAs start on the first block staged
    if (need_act) {
      if (!wait_or_abort(&y.act_kb[kb], act_uses[kb] & 1, a, s_abort, MMA_SLEEP_NS)) return false;
      ++act_uses[kb];
      tc::fence_after();
    }
    const uint64_t db = tc::desc_sw128(smem_u32(act + (size_t)kb * P.Bp * 128));
    for (int i = 0; i < ntiles; ++i, ++it) {
      const int s = it % P.stages;
      mbar_wait_bounded(&y.full[s], (it / P.stages) & 1, a.status, a.wait_cycles);
      tc::fence_after();
      const uint64_t da = tc::desc_sw128(smem_u32(ring + (size_t)s * BOX));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)  // 16-wide K slices: +32 bytes = +2 in descriptor units
        tc::mma_bf16(tmem_d + (uint32_t)(i * P.Bp), da + 2 * kk, db + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
      tc::commit(&y.empty[s]);
    }
  }
  tc::commit(done);
  return true;
}


// MMA warp (one thread): the unit sequence of the producer. Waits for the
// staged activations and a drained accumulator.
__device__ void mma_issuer(const Plan& P, int Nt, uint8_t* ring, const uint8_t* act, uint32_t tmem, const Sync& y,
                           const TokenStepArgs& a, volatile int* s_abort) {
  const int G = gridDim.x, c = blockIdx.x;
  int it = 0, nu = 0;
  int act_uses[MAX_KB];
#pragma unroll
  for (int k = 0; k < MAX_KB; ++k) act_uses[k] = 0;
  auto unit = [&](int nkb, int ntiles, bool need_act) -> bool {
    const int buf = nu & 1;
    if (nu >= 2 && !wait_or_abort(&y.acc_empty[buf], ((nu >> 1) + 1) & 1, a, s_abort, MMA_SLEEP_NS)) return false;
    tc::fence_after();
    if (!issue_unit(P, nkb, ntiles, ring, act, tmem + (uint32_t)(buf * 64), y, &y.acc_full[buf], it,
                    act_uses, need_act, a, s_abort))
      return false;
    ++nu;
    return true;
  };
  bool ok = true;
  for (int l = 0; ok && l < Nt; ++l) {
    for (int w = first_g1(P, c); ok && w < P.N1; w += G) ok = unit(P.kb1, 1, true);
    for (int w = first_g2(P, c, G); ok && w < P.N2; w += G) ok = unit(P.kb2, 1, true);
  }
  bool first = true;
  for (int t = c; ok && t < P.TL; t += G) {
    ok = unit(P.kbL, 1, first);  // every vocabulary tile reads the same staged input
    first = false;
  }
  // MMAs still writing TMEM must finish before the accumulators are freed
  if (nu > 0) mbar_wait_bounded(&y.acc_full[(nu - 1) & 1], ((nu - 1) >> 1) & 1, a.status, a.wait_cycles);
}

// ---- worker phases ----------------------------------------------------------
// Thread t of the workers owns TMEM lane t (the tile's feature t) in the
// accumulators; column b is batch row b.

// Store the fp32 accumulator tile (128 features x B rows) to part[b][128].
__device__ void store_partial(uint32_t tbuf, float* part, int B, int Bp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t trow = tbuf + ((uint32_t)(warp * 32) << 16);
  float* dst = part + warp * 32 + lane;
  for (int c0 = 0; c0 < Bp; c0 += 16) {
    float v[16];
    tc::tmem_ld16(trow + c0, v);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (c0 + j < B) __stcg(dst + (size_t)(c0 + j) * 128, v[j]);
  }
}

// Ingest: for rows b of this CTA, h[b] = token embedding of src[b] (token
// steps; the prefix row already in h otherwise) and its per-tile statistics.
__device__ void ingest_phase(const TokenStepArgs& a, const Plan& P, int jb) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = a.D;
  for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
    int tok = 0;
    if (a.ingest) {
      tok = a.src[b];
      if (tok < 0 || tok >= a.V) {
        if (threadIdx.x == 0) set_status(a.status, ST_BAD_TOKEN);
        tok = 0;
      }
      if (threadIdx.x == 0) a.block_tok[b * a.L_B + jb] = tok;
    }
    float* hrow = a.h + (size_t)b * D;
    for (int t = warp; t < P.T2; t += 4) {
      const int f = t * 128 + 4 * lane;
      float4 v;
      if (a.ingest) {
        const uint2 w = *reinterpret_cast<const uint2*>(a.tok_emb + (size_t)tok * D + f);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
        v = make_float4(lo.x, lo.y, hi.x, hi.y);
        __stcg(reinterpret_cast<float4*>(hrow + f), v);
      } else {
        v = __ldcg(reinterpret_cast<const float4*>(hrow + f));
      }
      *reinterpret_cast<uint2*>(a.hb + (size_t)b * D + f) = pack_bf16x4(v.x, v.y, v.z, v.w);
      const float mean = warp_sum((v.x + v.y) + (v.z + v.w)) * (1.f / 128.f);
      const float dx = v.x - mean, dy = v.y - mean, dz = v.z - mean, dw = v.w - mean;
      const float m2 = warp_sum((dx * dx + dy * dy) + (dz * dz + dw * dw));
      if (lane == 0) __stcg(a.hstat + (size_t)b * P.T2 + t, make_float2(mean, m2));
    }
  }
}

// Per-row LayerNorm statistics (mean, 1 / std) of rows 0..B-1 and the
// LayerNorm gain / shift of features [k0, k0 + 64 kb1) into shared memory.
__device__ void ln_params_to_smem(const TokenStepArgs& a, const Plan& P, int k0, const float* g, const float* beta,
                                  float* s_mu, float* s_rs, float* s_g, float* s_b) {
  for (int b = threadIdx.x; b < a.B; b += WORKERS) {
    float mu, rstd;
    row_stats(a.hstat + (size_t)b * P.T2, P.T2, a.eps, mu, rstd);
    s_mu[b] = mu;
    s_rs[b] = rstd;
  }
  for (int f = threadIdx.x * 4; f < P.kb1 * 64; f += WORKERS * 4) {
    *reinterpret_cast<float4*>(s_g + f) = *reinterpret_cast<const float4*>(g + k0 + f);
    *reinterpret_cast<float4*>(s_b + f) = *reinterpret_cast<const float4*>(beta + k0 + f);
  }
}

// G1 activations: rows 0..Bp-1 of features [k0, k0 + 64 kb1) of the bf16
// copy of h, staged by TMA straight into the swizzled K-major operand layout
// (box kb on staged_kb[kb]; rows >= B arrive as zeros), are normalised in
// place: x = (h - mean) / std * g + beta with the rows' exact fp32
// statistics, rounded to bf16 again. Block kb is announced on bars[kb]
// (thread 0, after the worker barrier) as soon as it is done, so its MMAs
// start while the next block is normalised. Item = (row, 16-byte chunk of 8
// features) of a block; Bp * 8 <= 4 * WORKERS.
__device__ void ln_to_operand(const TokenStepArgs& a, const Plan& P, const float* s_g, const float* s_b,
                              const float* s_mu, const float* s_rs, uint8_t* act, uint64_t* staged_kb,
                              uint32_t parity, uint64_t* bars, int* staged) {
  constexpr int U = 4;
  const int n_items = P.Bp * 8;
  for (int kb = 0; kb < P.kb1; ++kb) {
    mbar_wait_bounded(&staged_kb[kb], parity, a.status, a.wait_cycles);
    uint8_t* blk = act + (size_t)kb * P.Bp * 128;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int item = threadIdx.x + u * WORKERS;
      const int b = item >> 3, ch = item & 7;
      if (item < n_items && b < a.B) {
        uint4* cp = reinterpret_cast<uint4*>(blk + tc::sw128_offset(b, ch));
        const uint4 w = *cp;
        float x[8];
        unpack16(w, x, (const bf16*)nullptr);
        const int f = kb * 64 + ch * 8;
        const float mu = s_mu[b], rstd = s_rs[b];
        const float4 g0 = *reinterpret_cast<const float4*>(s_g + f);
        const float4 g1 = *reinterpret_cast<const float4*>(s_g + f + 4);
        const float4 b0 = *reinterpret_cast<const float4*>(s_b + f);
        const float4 b1 = *reinterpret_cast<const float4*>(s_b + f + 4);
        const uint2 lo = pack_bf16x4((x[0] - mu) * rstd * g0.x + b0.x, (x[1] - mu) * rstd * g0.y + b0.y,
                                     (x[2] - mu) * rstd * g0.z + b0.z, (x[3] - mu) * rstd * g0.w + b0.w);
        const uint2 hi = pack_bf16x4((x[4] - mu) * rstd * g1.x + b1.x, (x[5] - mu) * rstd * g1.y + b1.y,
                                     (x[6] - mu) * rstd * g1.z + b1.z, (x[7] - mu) * rstd * g1.w + b1.w);
        *cp = make_uint4(lo.x, lo.y, hi.x, hi.y);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    wsync();
    if (threadIdx.x == 0) {
      mbar_arrive(&bars[kb]);
      ++staged[kb];
    }
  }
}

// Bulk copies of the local-window rows 0..pos-1 (K and V) of this CTA's
// attention items (rows r0..r1-1 x the nh heads of head group hg) into `win`
// (item i: K at i * 2 * W, V at i * 2 * W + W, W = pos * dh * 2 bytes),
// completion on `bar`. One thread. Rows were written by earlier steps.
__device__ void window_copies(const TokenStepArgs& a, int l, int hg, int nh, int r0, int r1, int pos, uint8_t* win,
                              uint64_t* bar) {
  const uint32_t W = (uint32_t)pos * a.dh * 2;
  const int n_items = (r1 - r0) * nh;
  mbar_arrive_expect_tx(bar, 2u * W * (uint32_t)n_items);
  if (W == 0) return;
  const bf16* kc = a.kt + (size_t)l * a.kt_layer;
  const bf16* vc = a.vt + (size_t)l * a.kt_layer;
  for (int i = 0; i < n_items; ++i) {
    const int r = r0 + i / nh, h = hg * nh + i % nh;
    const size_t off = ((size_t)r * a.H + h) * a.l_cap * a.dh;
    bulk_g2s(win + (size_t)i * 2 * W, kc + off, W, bar);
    bulk_g2s(win + (size_t)i * 2 * W + W, vc + off, W, bar);
  }
}

// q|k|v head group hg, rows r0..r1-1: four threads per (row, head), thread q
// holding head dims [q * dh/4, (q + 1) * dh/4). q, k, v = the S1 partial
// sums of the group's three tiles + bias; rotary on q and k (the rotary dims
// are all in thread 0's quarter); k, v appended to the local cache at `pos`;
// attention of q over the window rows (staged in `win`) and the new row.
// Rotary dims: none, or the first d_head/4 (rot == DPT).
template <int DH>
__device__ void attention_items(const TokenStepArgs& a, const Plan& P, int l, int hg, int r0, int r1, int pos,
                                const uint8_t* win) {
  constexpr int DPT = DH / 4;
  const int nh = 128 / DH;
  const int quarter = threadIdx.x & 3;
  const int n_items = (r1 - r0) * nh;
  const float* bias = layer_ptr(a.b_qkv1, l, a.layer_stride);
  bf16* kc = a.kt + (size_t)l * a.kt_layer;
  bf16* vc = a.vt + (size_t)l * a.kt_layer;
  const uint32_t W = (uint32_t)pos * DH * 2;
  for (int i0 = 0; i0 < n_items; i0 += WORKERS / 4) {
    const int i = i0 + (threadIdx.x >> 2);
    const bool active = i < n_items;
    const int r = active ? r0 + i / nh : r0, hh = active ? i % nh : 0;
    const int h = hg * nh + hh;
    const int e0 = quarter * DPT;
    float q[DPT], k[DPT], v[DPT];
#pragma unroll
    for (int e = 0; e < DPT; e += 4) {
      const int fq = h * DH + e0 + e;  // feature of q; k at D + fq, v at 2D + fq
      float4 sq = *reinterpret_cast<const float4*>(bias + fq);
      float4 sk = *reinterpret_cast<const float4*>(bias + a.D + fq);
      float4 sv = *reinterpret_cast<const float4*>(bias + 2 * a.D + fq);
      if (active) {
        const int f = hh * DH + e0 + e;  // feature within the tile
#pragma unroll
        for (int sp = 0; sp < S1; ++sp) {
          const size_t o = ((size_t)sp * a.B + r) * 128 + f;
          sq = f4add(sq, __ldcg(reinterpret_cast<const float4*>(a.p1 + ((size_t)hg * S1) * a.B * 128 + o)));
          sk = f4add(sk, __ldcg(reinterpret_cast<const float4*>(
                             a.p1 + ((size_t)(P.HG + hg) * S1) * a.B * 128 + o)));
          sv = f4add(sv, __ldcg(reinterpret_cast<const float4*>(
                             a.p1 + ((size_t)(2 * P.HG + hg) * S1) * a.B * 128 + o)));
        }
      }
      q[e] = sq.x; q[e + 1] = sq.y; q[e + 2] = sq.z; q[e + 3] = sq.w;
      k[e] = sk.x; k[e + 1] = sk.y; k[e + 2] = sk.z; k[e + 3] = sk.w;
      v[e] = sv.x; v[e + 1] = sv.y; v[e + 2] = sv.z; v[e + 3] = sv.w;
    }
    if (quarter == 0 && a.rot == DPT) {
      // rotate-half pairs (e, e + DPT/2), e < DPT/2: all in this thread
      constexpr int HALF = DPT / 2;
#pragma unroll
      for (int e = 0; e < HALF; ++e) {
        const float2 cs = a.rope_tab[(size_t)pos * HALF + e];
        const float q0 = q[e], q1 = q[e + HALF], k0 = k[e], k1 = k[e + HALF];
        q[e] = q0 * cs.x - q1 * cs.y;
        q[e + HALF] = q1 * cs.x + q0 * cs.y;
        k[e] = k0 * cs.x - k1 * cs.y;
        k[e + HALF] = k1 * cs.x + k0 * cs.y;
      }
    }
    // k, v into the cache (bf16); attention reads what the cache holds
    const size_t crow = (((size_t)r * a.H + h) * a.l_cap + pos) * DH + e0;
#pragma unroll
    for (int e = 0; e < DPT; e += 4) {
      const uint2 kp = pack_bf16x4(k[e], k[e + 1], k[e + 2], k[e + 3]);
      const uint2 vp = pack_bf16x4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      if (active) {
        *reinterpret_cast<uint2*>(kc + crow + e) = kp;
        *reinterpret_cast<uint2*>(vc + crow + e) = vp;
      }
      const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kp.x));
      const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kp.y));
      const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vp.x));
      const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vp.y));
      k[e] = k01.x; k[e + 1] = k01.y; k[e + 2] = k23.x; k[e + 3] = k23.y;
      v[e] = v01.x; v[e + 1] = v01.y; v[e + 2] = v23.x; v[e + 3] = v23.y;
    }
    // online softmax over window rows 0..pos-1 (shared memory) then the new row
    const uint8_t* wk = win + (size_t)(active ? i : 0) * 2 * W;
    const uint8_t* wv = wk + W;
    float m = -FLT_MAX, lsum = 0.f, o[DPT];
#pragma unroll
    for (int e = 0; e < DPT; ++e) o[e] = 0.f;
    for (int j = 0; j <= pos; ++j) {
      float kj[DPT], vj[DPT];
      if (j < pos) {
#pragma unroll
        for (int e = 0; e < DPT; e += 8) {
          float t8[8];
          unpack16(*reinterpret_cast<const uint4*>(wk + ((size_t)j * DH + e0 + e) * 2), t8, (const bf16*)nullptr);
#pragma unroll
          for (int x = 0; x < 8; ++x) kj[e + x] = t8[x];
          unpack16(*reinterpret_cast<const uint4*>(wv + ((size_t)j * DH + e0 + e) * 2), t8, (const bf16*)nullptr);
#pragma unroll
          for (int x = 0; x < 8; ++x) vj[e + x] = t8[x];
        }
      } else {
#pragma unroll
        for (int e = 0; e < DPT; ++e) { kj[e] = k[e]; vj[e] = v[e]; }
      }
      float sc = 0.f;
#pragma unroll
      for (int e = 0; e < DPT; ++e) sc = fmaf(q[e], kj[e], sc);
      sc += __shfl_xor_sync(0xffffffffu, sc, 1);
      sc += __shfl_xor_sync(0xffffffffu, sc, 2);
      sc *= P.scale;
      const float mn = fmaxf(m, sc);
      const float cf = exp2f(m - mn), p = exp2f(sc - mn);
      lsum = lsum * cf + p;
#pragma unroll
      for (int e = 0; e < DPT; ++e) o[e] = fmaf(p, vj[e], o[e] * cf);
      m = mn;
    }
    if (active) {
      bf16* out = a.a2 + (size_t)r * 5 * a.D + h * DH + e0;
      const float inv = 1.f / lsum;
#pragma unroll
      for (int e = 0; e < DPT; e += 4)
        *reinterpret_cast<uint2*>(out + e) = pack_bf16x4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv);
    }
  }
}

// fc1 tile f (features 3D + 128 f ..), rows r0..r1-1: the S1 partial sums +
// bias, GELU -> a2[:, D + 128 f ..]
__device__ void gelu_rows(const TokenStepArgs& a, const Plan& P, int l, int f, int r0, int r1) {
  const int t = 3 * P.HG + f;
  const float* bias = layer_ptr(a.b_qkv1, l, a.layer_stride) + 3 * a.D + f * 128;
  const float* part = a.p1 + (size_t)t * S1 * a.B * 128;
  const int n = (r1 - r0) * 32;  // float4 groups
  constexpr int U = 4;           // groups per thread in flight
  for (int i0 = threadIdx.x; i0 < n; i0 += U * WORKERS) {
    float4 acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * WORKERS;
      if (i < n) {
        const int r = r0 + i / 32, c = (i % 32) * 4;
        acc[u] = *reinterpret_cast<const float4*>(bias + c);
#pragma unroll
        for (int sp = 0; sp < S1; ++sp)
          acc[u] = f4add(acc[u], __ldcg(reinterpret_cast<const float4*>(part + ((size_t)sp * a.B + r) * 128 + c)));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * WORKERS;
      if (i < n) {
        const int r = r0 + i / 32, c = (i % 32) * 4;
        *reinterpret_cast<uint2*>(a.a2 + (size_t)r * 5 * a.D + a.D + f * 128 + c) =
            pack_bf16x4(gelu_erf(acc[u].x), gelu_erf(acc[u].y), gelu_erf(acc[u].z), gelu_erf(acc[u].w));
      }
    }
  }
}

// G2 tile t2, rows r0..r1-1: h += the S2 partial sums + (b_o + b_2); the
// new rows' per-tile statistics. Warp w takes rows r0 + w, r0 + w + 4, ...;
// lane holds features 4 lane .. 4 lane + 3 of the tile.
__device__ void residual_rows(const TokenStepArgs& a, const Plan& P, int l, int t2, int r0, int r1) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = t2 * 128 + 4 * lane;
  const float4 bo = *reinterpret_cast<const float4*>(layer_ptr(a.b_o2, l, a.layer_stride) + f);
  const float* part = a.p2 + (size_t)t2 * S2 * a.B * 128;
  for (int r = r0 + warp; r < r1; r += 4) {
    float* hrow = a.h + (size_t)r * a.D;
    float4 acc = f4add(__ldcg(reinterpret_cast<const float4*>(hrow + f)), bo);
    float4 ps[S2];
#pragma unroll
    for (int sp = 0; sp < S2; ++sp)
      ps[sp] = __ldcg(reinterpret_cast<const float4*>(part + ((size_t)sp * a.B + r) * 128 + 4 * lane));
#pragma unroll
    for (int sp = 0; sp < S2; ++sp) acc = f4add(acc, ps[sp]);
    __stcg(reinterpret_cast<float4*>(hrow + f), acc);
    *reinterpret_cast<uint2*>(a.hb + (size_t)r * a.D + f) = pack_bf16x4(acc.x, acc.y, acc.z, acc.w);
    const float mean = warp_sum((acc.x + acc.y) + (acc.z + acc.w)) * (1.f / 128.f);
    const float dx = acc.x - mean, dy = acc.y - mean, dz = acc.z - mean, dw = acc.w - mean;
    const float m2 = warp_sum((dx * dx + dy * dy) + (dz * dz + dw * dw));
    if (lane == 0) __stcg(a.hstat + (size_t)r * P.T2 + t2, make_float2(mean, m2));
  }
}

// Final LayerNorm of row b -> xf[b] (bf16)
__device__ void final_ln_row(const TokenStepArgs& a, const Plan& P, int b) {
  float mu, rstd;
  row_stats(a.hstat + (size_t)b * P.T2, P.T2, a.eps, mu, rstd);
  const float* hrow = a.h + (size_t)b * a.D;
  for (int c = threadIdx.x * 4; c < a.D; c += WORKERS * 4) {
    const float4 x = __ldcg(reinterpret_cast<const float4*>(hrow + c));
    const float4 g = *reinterpret_cast<const float4*>(a.lnf_g + c);
    const float4 be = *reinterpret_cast<const float4*>(a.lnf_b + c);
    *reinterpret_cast<uint2*>(a.xf + (size_t)b * a.D + c) =
        pack_bf16x4((x.x - mu) * rstd * g.x + be.x, (x.y - mu) * rstd * g.y + be.y,
                    (x.z - mu) * rstd * g.z + be.z, (x.w - mu) * rstd * g.w + be.w);
  }
}

__device__ __forceinline__ void better(float& v, int& i, float ov, int oi) {
  if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
}

// Per-row argmax over the warp's 32 features for 32 rows held one per
// register (v[r], index ix): a transposing butterfly -- at each of the 5
// levels a lane keeps half of its rows and trades the other half with its
// partner -- leaves row `lane` reduced over the 32 lanes.
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

// LM epilogue of vocabulary tile t: logits (optional) and the tile's argmax per row
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
      if (n >= a.V || m >= a.B || (c0 + 16 >= Bp && j >= 16)) v[j] = -INFINITY;
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
    __stcg(a.arg_part + (size_t)t * a.B + r, best);
  }
  wsync();  // s_arg is reused by the next tile
}

// Greedy id per row from the tile partials (lowest id on ties)
__device__ void argmax_rows(const TokenStepArgs& a, const Plan& P) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int U = 16;  // tile partials per lane in flight (TL <= 512 * 32 / 32)
  for (int b = blockIdx.x * 4 + warp; b < a.B; b += 4 * gridDim.x) {
    float bv = -INFINITY;
    int bi = INT_MAX;
    for (int t0 = lane; t0 < P.TL; t0 += U * 32) {
      float2 o[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u * 32;
        o[u] = t < P.TL ? __ldcg(a.arg_part + (size_t)t * a.B + b) : make_float2(-INFINITY, __int_as_float(INT_MAX));
      }
#pragma unroll
      for (int u = 0; u < U; ++u) better(bv, bi, o[u].x, __float_as_int(o[u].y));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      better(bv, bi, ov, oi);
    }
    if (lane == 0) a.next[b] = bi;
  }
}

// TMA of nkb activation boxes (Bp rows x 64 columns, columns col0 + 64 kb)
// into `act`, box kb completing on bars[kb]. One thread; the rows were
// written through the generic proxy by other CTAs before the counter this
// thread acquired.
__device__ void load_act(const CUtensorMap* map, uint8_t* act, int col0, int nkb, int Bp, uint64_t* bars,
                         int* staged) {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  for (int kb = 0; kb < nkb; ++kb) {
    mbar_arrive_expect_tx(&bars[kb], (uint32_t)(Bp * 128));
    tc::tma_load_2d(act + (size_t)kb * Bp * 128, map, col0 + kb * 64, 0, &bars[kb]);
    ++staged[kb];
  }
}

template <int DH>
__global__ void __launch_bounds__(THREADS, 1)
token_step2_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mo,
                   const __grid_constant__ CUtensorMap ml, const __grid_constant__ CUtensorMap ma2,
                   const __grid_constant__ CUtensorMap mxf, const __grid_constant__ CUtensorMap mhb,
                   const TokenStepArgs a, const Plan P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;
  uint8_t* act = smem + (size_t)P.stages * BOX;
  __shared__ __align__(8) uint64_t full[MAX_STAGES], empty[MAX_STAGES], act_kb[MAX_KB], hb_kb[MAX_KB],
      acc_full[2], acc_empty[2], win_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ float2 s_arg[4][MAX_B];
  __shared__ float s_mu[MAX_B], s_rs[MAX_B];
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < P.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < MAX_KB; ++i) {
      mbar_init(&act_kb[i], 1);
      mbar_init(&hb_kb[i], 1);
    }
    mbar_init(&win_bar, 1);
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
  const Sync y{full, empty, act_kb, acc_full, acc_empty};
  pdl_trigger();

  if (warp == 4) {
    // weights do not depend on earlier kernels: no wait before streaming them
    if ((threadIdx.x & 31) == 0) producer(&mq, &mo, &ml, P, a.Nt, ring, full, empty, a, &s_abort);
  } else if (warp == 5) {
    if ((threadIdx.x & 31) == 0) mma_issuer(P, a.Nt, ring, act, tmem, y, a, &s_abort);
  } else {
    pdl_wait();
    const int G = gridDim.x, c = blockIdx.x;
    const int B = a.B;
    const int pos = pos_base(a.pos);  // read before anyone can advance the step state
    const int jb = a.dstate[1];
    unsigned* cb = a.bar;
    wsync();
    if (threadIdx.x == 0) signal(ctr(cb, C_ARRIVED));
    int nu = 0, nw = 0, n_hb = 0;
    bool hb_pending = false;
    int staged[MAX_KB];  // worker-side uses of each activation barrier (thread 0)
#pragma unroll
    for (int k = 0; k < MAX_KB; ++k) staged[k] = 0;
    bool win_pending = false;
    bool ok = true;
    const int nh = 128 / DH;
    // ingest: rows of h and their statistics
    if (c < B) {
      ingest_phase(a, P, jb);
      workers_signal(ctr(cb, C_H));
    }
    for (int l = 0; ok && l < a.Nt; ++l) {
      const unsigned h_ready = (unsigned)(P.n_ing + l * P.N2);
      for (int w = c; ok && w < P.N1; w += G) {
        const int t = w / P.S1, sp = w % P.S1;
        if (!(ok = workers_wait(a, ctr(cb, C_H), h_ready, &s_abort))) break;
        const bool qkv = t < 3 * P.HG;
        const int k0 = sp * P.kb1 * 64;
        // the unit's K range of every row (bf16 copy of h) into the operand
        // buffer by TMA while the statistics and parameters are gathered
        if (threadIdx.x == 0) {
          asm volatile("fence.proxy.async.global;" ::: "memory");
          for (int kb = 0; kb < P.kb1; ++kb) {
            mbar_arrive_expect_tx(&hb_kb[kb], (uint32_t)(P.Bp * 128));
            tc::tma_load_2d(act + (size_t)kb * P.Bp * 128, &mhb, k0 + kb * 64, 0, &hb_kb[kb]);
          }
          hb_pending = true;
        }
        const float* g = layer_ptr(qkv ? a.ln1_g : a.ln2_g, l, a.layer_stride);
        const float* be = layer_ptr(qkv ? a.ln1_b : a.ln2_b, l, a.layer_stride);
        // LayerNorm parameters of the unit's K range after the operand
        float* s_g = reinterpret_cast<float*>(act + (size_t)P.kb1 * P.Bp * 128);
        float* s_b = s_g + P.kb1 * 64;
        ln_params_to_smem(a, P, k0, g, be, s_mu, s_rs, s_g, s_b);
        wsync();
        ln_to_operand(a, P, s_g, s_b, s_mu, s_rs, act, hb_kb, (uint32_t)(n_hb & 1), act_kb, staged);
        ++n_hb;
        if (threadIdx.x == 0) hb_pending = false;
        const int buf = nu & 1;
        mbar_wait_bounded(&acc_full[buf], (nu >> 1) & 1, a.status, a.wait_cycles);
        tc::fence_after();
        // the operand buffer is free now (the MMAs completed): stage the
        // attention window there while the partials go out
        const int hg = t % P.HG, rank = (t / P.HG) * P.S1 + sp;
        const int ra0 = rank * B / (3 * P.S1), ra1 = (rank + 1) * B / (3 * P.S1);
        if (qkv && threadIdx.x == 0) {
          window_copies(a, l, hg, nh, ra0, ra1, pos, act, &win_bar);
          win_pending = true;
        }
        store_partial(tmem + (uint32_t)(buf * 64), a.p1 + (size_t)(t * P.S1 + sp) * B * 128, B, P.Bp);
        tc::fence_before();
        mbar_arrive(&acc_empty[buf]);
        ++nu;
        workers_signal(ctr(cb, C_G1P + t));
        if (qkv) {
          if (threadIdx.x == 0)
            for (int m = 0; m < 3 && !s_abort; ++m)
              wait_count(a, ctr(cb, C_G1P + m * P.HG + hg), (unsigned)((l + 1) * P.S1), &s_abort);
          wsync();
          if (!(ok = !s_abort)) break;
          mbar_wait_bounded(&win_bar, nw & 1, a.status, a.wait_cycles);
          ++nw;
          if (threadIdx.x == 0) win_pending = false;
          attention_items<DH>(a, P, l, hg, ra0, ra1, pos, act);
          workers_signal(ctr(cb, P.c_a2 + hg));
        } else {
          const int f = t - 3 * P.HG;
          if (!(ok = workers_wait(a, ctr(cb, C_G1P + t), (unsigned)((l + 1) * P.S1), &s_abort))) break;
          gelu_rows(a, P, l, f, sp * B / P.S1, (sp + 1) * B / P.S1);
          workers_signal(ctr(cb, P.c_a2 + P.HG + f));
        }
      }
      for (int w = first_g2(P, c, G); ok && w < P.N2; w += G) {
        const int t2 = w / P.S2, sp = w % P.S2;
        const int col0 = sp * P.kb2 * 64;
        const int j0 = col0 / 128, j1 = (col0 + P.kb2 * 64 - 1) / 128;
        if (threadIdx.x == 0)
          for (int j = j0; j <= j1 && !s_abort; ++j)
            wait_count(a, ctr(cb, P.c_a2 + j), (unsigned)((l + 1) * (j < P.HG ? 3 * P.S1 : P.S1)), &s_abort);
        wsync();
        if (!(ok = !s_abort)) break;
        if (threadIdx.x == 0) load_act(&ma2, act, col0, P.kb2, P.Bp, act_kb, staged);
        const int buf = nu & 1;
        mbar_wait_bounded(&acc_full[buf], (nu >> 1) & 1, a.status, a.wait_cycles);
        tc::fence_after();
        store_partial(tmem + (uint32_t)(buf * 64), a.p2 + (size_t)(t2 * P.S2 + sp) * B * 128, B, P.Bp);
        tc::fence_before();
        mbar_arrive(&acc_empty[buf]);
        ++nu;
        workers_signal(ctr(cb, P.c_g2p + t2));
        if (!(ok = workers_wait(a, ctr(cb, P.c_g2p + t2), (unsigned)((l + 1) * P.S2), &s_abort))) break;
        residual_rows(a, P, l, t2, sp * B / P.S2, (sp + 1) * B / P.S2);
        workers_signal(ctr(cb, C_H));
      }
    }
    // final LayerNorm rows -> xf
    if (ok && c < B) {
      if ((ok = workers_wait(a, ctr(cb, C_H), (unsigned)(P.n_ing + a.Nt * P.N2), &s_abort))) {
        for (int b = c; b < B; b += G) final_ln_row(a, P, b);
        workers_signal(ctr(cb, C_FINAL));
      }
    }
    // LM head over this CTA's vocabulary tiles
    if (ok && c < P.TL) {
      if ((ok = workers_wait(a, ctr(cb, C_FINAL), (unsigned)P.n_ing, &s_abort))) {
        if (threadIdx.x == 0) load_act(&mxf, act, 0, P.kbL, P.Bp, act_kb, staged);
        for (int t = c; t < P.TL; t += G) {
          const int buf = nu & 1;
          mbar_wait_bounded(&acc_full[buf], (nu >> 1) & 1, a.status, a.wait_cycles);
          tc::fence_after();
          lm_epilogue(tmem + (uint32_t)(buf * 64), t, a, P.Bp, s_arg);
          mbar_arrive(&acc_empty[buf]);  // lm_epilogue ended with the tcgen05 fence + barrier
          ++nu;
        }
        workers_signal(ctr(cb, C_LM));
      }
    }
    // greedy argmax, then the step state advanced once every CTA has read it
    if (ok && c * 4 < B) {
      if ((ok = workers_wait(a, ctr(cb, C_LM), (unsigned)P.n_lm, &s_abort))) {
        argmax_rows(a, P);
        if (c == 0 && threadIdx.x == 0 && wait_count(a, ctr(cb, C_ARRIVED), (unsigned)G, &s_abort)) {
          const int t = a.dstate[0] + 1;
          a.dstate[0] = t;
          a.dstate[1] = t % a.L_B;
          a.dstate[2] = t / a.L_B;
        }
      }
    }
    if (!ok && threadIdx.x == 0) s_abort = 1;  // releases the producer / MMA warps' waits
    // copies into shared memory still in flight must land before the CTA exits
    if (threadIdx.x == 0) {
      if (win_pending) mbar_wait_bounded(&win_bar, nw & 1, a.status, a.wait_cycles);
      if (hb_pending)
        for (int k = 0; k < P.kb1; ++k) mbar_wait_bounded(&hb_kb[k], n_hb & 1, a.status, a.wait_cycles);
      for (int k = 0; k < MAX_KB; ++k)
        if (staged[k] > 0) mbar_wait_bounded(&act_kb[k], (staged[k] - 1) & 1, a.status, a.wait_cycles);
    }
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_free(tmem, TMEM_COLS);
  if (threadIdx.x == 0) {
    // the last CTA out resets every counter except the abort word
    __threadfence();
    if (atomicAdd(ctr(a.bar, C_EXIT), 1u) == gridDim.x - 1) {
      for (int sl = 0; sl < P.n_slots; ++sl)
        if (sl != C_ABORT) *ctr(a.bar, sl) = 0u;
      __threadfence();
    }
  }
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

// bf16 activation rows [rows, cols] (row-major): boxes of 64 columns x
// box_rows rows, 128-byte swizzle, zero fill for rows >= rows
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
        cudaFuncGetAttributes(&fa, token_step2_kernel<64>) != cudaSuccess)
      return d;
    d.smem_max = (size_t)optin - fa.sharedSizeBytes;  // every instance declares the same static memory
    if (cudaFuncSetAttribute(token_step2_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)d.smem_max) != cudaSuccess ||
        cudaFuncSetAttribute(token_step2_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)d.smem_max) != cudaSuccess ||
        cudaFuncSetAttribute(token_step2_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)d.smem_max) != cudaSuccess)
      return d;
    d.ready = true;
  }
  return d;
}


bool make_plan(int B, int D, int dh, int V, int l_cap, int sms, size_t smem_max, Plan* P, size_t* smem) {
  Plan p{};
  p.Bp = (B + 15) / 16 * 16;
  p.HG = D / 128;
  p.T1 = 7 * p.HG;
  p.T2 = p.HG;
  p.TL = (V + 127) / 128;
  p.S1 = S1;
  p.S2 = S2;
  p.kb1 = D / 64 / p.S1;
  p.kb2 = 5 * D / 64 / p.S2;
  p.kbL = D / 64;
  p.N1 = p.T1 * p.S1;
  p.N2 = p.T2 * p.S2;
  p.g2_base = (p.N1 + p.N2 <= sms) ? sms - p.N2 : p.N1 % sms;
  p.n_ing = B < sms ? B : sms;
  p.n_lm = p.TL < sms ? p.TL : sms;
  p.c_a2 = C_G1P + p.T1;
  p.c_g2p = p.c_a2 + 5 * p.HG;
  p.n_slots = p.c_g2p + p.T2;
  // the activation buffer: the largest operand, or the attention windows
  size_t act = (size_t)p.kb1 * p.Bp * 128 + (size_t)p.kb1 * 64 * 2 * sizeof(float);  // + LayerNorm parameters
  act = act > (size_t)p.kb2 * p.Bp * 128 ? act : (size_t)p.kb2 * p.Bp * 128;
  act = act > (size_t)p.kbL * p.Bp * 128 ? act : (size_t)p.kbL * p.Bp * 128;
  const int rows_max = (B + 3 * p.S1 - 1) / (3 * p.S1);
  const size_t win = (size_t)rows_max * (128 / dh) * 2 * (l_cap - 1) * dh * 2;
  act = act > win ? act : win;
  act = (act + 1023) & ~(size_t)1023;
  if (smem_max < act + 1024 + 4 * (size_t)BOX) return false;
  int st = (int)((smem_max - act - 1024) / BOX);
  p.stages = st > MAX_STAGES ? MAX_STAGES : st;
  p.act_bytes = (int)act;
  p.scale = 1.4426950408889634f / sqrtf((float)dh);
  *P = p;
  *smem = (size_t)p.stages * BOX + act + 1024;
  return true;
}

}  // namespace

size_t token_step2_counter_bytes(int D) {
  const int hg = D / 128;
  return (size_t)(C_G1P + 7 * hg + 5 * hg + hg) * 32 * sizeof(unsigned);
}

size_t token_step2_scratch_floats(int B, int D, int which) {
  if (B > MAX_B) B = MAX_B;
  const int hg = D / 128;
  if (which == 1) return (size_t)7 * hg * S1 * B * 128;   // G1 partials
  if (which == 2) return (size_t)hg * S2 * B * 128;       // G2 partials
  if (which == 4) return (size_t)B * D / 2;               // bf16 copy of h (floats' worth)
  return (size_t)B * hg * 2;                              // per-(row, tile) statistics
}

int token_step2_supported(int dt, int B, int D, int H, int rot, int V, int Nt, int l_cap) {
  if (dt != DT_BF16 || B < 1 || B > MAX_B || Nt < 1 || V < 1 || l_cap < 1 || l_cap > MAX_WIN) return 0;
  if (D % 128 || D < 128 || D > 2048 || H < 1 || D % H) return 0;
  const int dh = D / H;
  if (dh != 32 && dh != 64 && dh != 128) return 0;
  if (rot != 0 && rot != dh / 4) return 0;  // the rotary dims sit in one thread's quarter of the head
  if ((5 * D / 64) % S2 || (D / 64) % S1) return 0;
  if (!encode_fn()) return 0;
  Device& d = device();
  if (!d.ready) return 0;
  Plan p;
  size_t smem;
  return make_plan(B, D, dh, V, l_cap, d.sms, d.smem_max, &p, &smem) ? 1 : 0;
}

cudaError_t launch_token_step2(const TokenStepArgs& a, const void* w_qkv1, const void* w_o2, const void* w_lm,
                               cudaStream_t s) {
  if (!token_step2_supported(DT_BF16, a.B, a.D, a.H, a.rot, a.V, a.Nt, a.l_cap)) return cudaErrorNotSupported;
  Device& d = device();
  Plan P;
  size_t smem;
  if (!make_plan(a.B, a.D, a.dh, a.V, a.l_cap, d.sms, d.smem_max, &P, &smem)) return cudaErrorNotSupported;
  CUtensorMap mq, mo, ml, ma2, mxf, mhb;
  // one layer: any stride at least the layer's own size satisfies the encoder
  const long long lsq = a.Nt > 1 ? a.layer_stride : 14LL * a.D * a.D;
  const long long lso = a.Nt > 1 ? a.layer_stride : 10LL * a.D * a.D;
  if (!weight_map(&mq, w_qkv1, a.D, 7LL * a.D, a.Nt, lsq) || !weight_map(&mo, w_o2, 5LL * a.D, a.D, a.Nt, lso) ||
      !weight_map(&ml, w_lm, a.D, a.V, 0, 0))
    return cudaErrorInvalidValue;
  if (!act_map(&ma2, a.a2, a.B, 5LL * a.D, P.Bp) || !act_map(&mxf, a.xf, a.B, a.D, P.Bp) ||
      !act_map(&mhb, a.hb, a.B, a.D, P.Bp))
    return cudaErrorInvalidValue;
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, TokenStepArgs, Plan) =
      a.dh == 32 ? token_step2_kernel<32> : (a.dh == 64 ? token_step2_kernel<64> : token_step2_kernel<128>);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(d.sms, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  // cooperative: the driver guarantees that every CTA is resident at once
  // (the counter waits rely on it) or refuses the launch
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
  e = cudaLaunchKernelEx(&cfg, kern, mq, mo, ml, ma2, mxf, mhb, a, P);
  note_launch();
  return e;
}

}  // namespace bt
