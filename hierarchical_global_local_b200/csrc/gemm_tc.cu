// gemm_tc.cu -- bf16 dense projections on the 5th-generation tensor cores
// (tcgen05 + TMEM), sm_100a.
//
// D[r, c] = sum_k A[r, k] * B[c, k]; A and B K-major bf16 in global memory,
// fp32 accumulation in tensor memory. One CTA per 128 x BN output tile (and
// per K split):
//   * one thread issues TMA tile loads (128-byte swizzle, no multicast) into a
//     4-stage shared-memory ring guarded by full/empty mbarriers;
//   * one thread issues tcgen05.mma (M = 128, N = BN, K = 16) per 16-wide K
//     slice and commits each stage back to its empty barrier;
//   * all four warps read the accumulator with tcgen05.ld (warp w owns TMEM
//     lanes 32w..32w+31) and apply the fused epilogue.
// Two orientations:
//   decode ("weights as A"): A = W [N, K] (128 output features per tile),
//     B = X [M, K] (the M <= 256 tokens of the batch, padded to BN by TMA
//     zero fill). K is split across the ks CTAs of a thread-block cluster so
//     that enough SMs stream weights; each CTA parks its fp32 partial tile in
//     its own shared memory and the cluster reduce-scatters over distributed
//     shared memory: rank q sums columns [q*BN/ks, (q+1)*BN/ks) of all ks
//     partials in rank order (deterministic) and runs the epilogue on them.
//   prefill ("activations as A"): A = X (128 tokens per tile), B = W (BN
//     features per tile), one K split.
// Every mbarrier wait is bounded; a wait that runs out sets a status bit.
#include <cooperative_groups.h>
#include <cuda.h>
#include <stdio.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace bt {

namespace {

constexpr int BM = 128;  // MMA M (TMEM lanes)
constexpr int BK = 64;   // K elements per stage = one 128-byte swizzle row
constexpr size_t PART_BUDGET = 256;  // split-K reduces in distributed shared memory

constexpr int MAX_STAGES = 8;
constexpr int MAX_KS = 16;  // K splits of one tile: CTAs of one (non-portable) cluster
// Warp roles: EPI epilogue warps, then the TMA producer warp and the MMA
// issuer warp. The activations-as-A orientation (prefill) runs eight
// epilogue warps: two per quarter of the TMEM lanes, each taking half of the
// tile's columns (its epilogue -- GELU and stores of every output -- is the
// bound there, not the tensor pipe); weights-as-A (decode) runs four.
template <bool SWAP>
struct Roles {
  static constexpr int EPI = SWAP ? 4 : 8;
  static constexpr int THREADS = EPI * 32 + 64;
  static constexpr int PRODUCER = EPI, MMA = EPI + 1;
};

template <int BN>
__host__ __device__ constexpr size_t stage_bytes() {
  return (size_t)(BM * BK * 2 + BN * BK * 2);
}

// TMEM columns: two fp32 accumulators of BN columns (double buffer)
template <int BN>
__host__ __device__ constexpr int tmem_cols() {
  return 2 * BN < 32 ? 32 : 2 * BN;
}

// Fused LayerNorm (see Epi::ln_*): called by the four epilogue warps after
// they stored rows [m_lo, m_hi) of out0 for this feature tile. The tile that
// completes a row (counter reaches the number of feature tiles) normalises
// it; every other tile only counts. One warp per row.
__device__ __forceinline__ void ep_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ void post_ln(const Epi& e, int m_lo, int m_hi, int M, int N, int nfeat_tiles,
                        int* s_rows, int* s_n) {
  __threadfence();
  ep_sync();
  if (threadIdx.x == 0) *s_n = 0;
  ep_sync();
  for (int m = m_lo + (int)threadIdx.x; m < m_hi && m < M; m += 128)
    if (atomicAdd(&e.ln_cnt[m], 1) == nfeat_tiles - 1) s_rows[atomicAdd(s_n, 1)] = m;
  ep_sync();
  const int nrows = *s_n;
  __threadfence();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* hsrc = reinterpret_cast<const float*>(e.out0);
  constexpr int MAXV = 16;  // float4 per lane: rows up to 2048 wide
  for (int i = warp; i < nrows; i += 4) {
    const int m = s_rows[i];
    const float* x = hsrc + (size_t)m * e.ld0;
    // the whole row in registers: one round trip to L2
    float4 v[MAXV];
#pragma unroll
    for (int u = 0; u < MAXV; ++u) {
      const int c = (lane + 32 * u) * 4;
      v[u] = (c < N) ? __ldcg(reinterpret_cast<const float4*>(x + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < MAXV; ++u) sum += (v[u].x + v[u].y) + (v[u].z + v[u].w);
    const float mu = warp_sum(sum) / (float)N;
    float sq = 0.f;
#pragma unroll
    for (int u = 0; u < MAXV; ++u) {
      const int c = (lane + 32 * u) * 4;
      if (c < N) {
        const float a = v[u].x - mu, b = v[u].y - mu, cc = v[u].z - mu, d = v[u].w - mu;
        sq += (a * a + b * b) + (cc * cc + d * d);
      }
    }
    const float rstd = rsqrtf(warp_sum(sq) / (float)N + e.ln_eps);
    const bool dual = e.ln_g2 != nullptr;
    const bool take = dual || (m % e.ln_step) == e.ln_off;
    if (take) {
      bf16* o = reinterpret_cast<bf16*>(e.ln_out) +
                (dual ? (size_t)m * 2 * N : (size_t)(m / e.ln_step) * N);
#pragma unroll
      for (int u = 0; u < MAXV; ++u) {
        const int c = (lane + 32 * u) * 4;
        if (c < N) {
          const float n0 = (v[u].x - mu) * rstd, n1 = (v[u].y - mu) * rstd;
          const float n2 = (v[u].z - mu) * rstd, n3 = (v[u].w - mu) * rstd;
          const float4 g = *reinterpret_cast<const float4*>(e.ln_g1 + c);
          const float4 bb = *reinterpret_cast<const float4*>(e.ln_b1 + c);
          __nv_bfloat162 lo = __floats2bfloat162_rn(n0 * g.x + bb.x, n1 * g.y + bb.y);
          __nv_bfloat162 hi = __floats2bfloat162_rn(n2 * g.z + bb.z, n3 * g.w + bb.w);
          uint2 w;
          w.x = *reinterpret_cast<uint32_t*>(&lo);
          w.y = *reinterpret_cast<uint32_t*>(&hi);
          *reinterpret_cast<uint2*>(o + c) = w;
          if (dual) {
            const float4 g2 = *reinterpret_cast<const float4*>(e.ln_g2 + c);
            const float4 b2 = *reinterpret_cast<const float4*>(e.ln_b2 + c);
            lo = __floats2bfloat162_rn(n0 * g2.x + b2.x, n1 * g2.y + b2.y);
            hi = __floats2bfloat162_rn(n2 * g2.z + b2.z, n3 * g2.w + b2.w);
            w.x = *reinterpret_cast<uint32_t*>(&lo);
            w.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(o + N + c) = w;
          }
        }
      }
    }
    if (lane == 0) e.ln_cnt[m] = 0;
  }
  ep_sync();  // s_rows / s_n reused by the next tile
}

// ---- the kernel ---------------------------------------------------------------
// SWAP = true: A = weights (rows = output features), B = activations (rows =
// tokens). SWAP = false: A = activations, B = weights.
// ks == 1: persistent; CTA c handles tiles c, c + gridDim.x, ... with a
//   continuous TMA ring across tiles and two TMEM accumulators, so the
//   epilogue of one tile overlaps the loads and MMAs of the next.
// ks > 1: one tile per CTA, K split over the cluster's ks CTAs, partial
//   tiles reduce-scattered over distributed shared memory.
template <int BN, bool SWAP>
__global__ void __launch_bounds__(Roles<SWAP>::THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               int M, int N, int nkb, int ks, int stages, int ntA, int ntB, int xk_split,
               int xk_off, Epi e, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  bf16* sA = reinterpret_cast<bf16*>(smem);
  bf16* sB = reinterpret_cast<bf16*>(smem + (size_t)stages * BM * BK * 2);
  __shared__ __align__(8) uint64_t full[MAX_STAGES], empty[MAX_STAGES], acc_full[2], acc_empty[2];
  __shared__ uint32_t tmem_slot;
  __shared__ float2 s_arg[4][BN <= 64 ? BN : 1];  // fused argmax: per warp, per column
  __shared__ int s_rows[256];                      // fused LayerNorm: rows completed here
  __shared__ int s_nrows;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = ntA * ntB;
  const int t_first = blockIdx.x;
  const int t_step = (ks == 1) ? gridDim.x : ntiles;  // split mode: exactly one tile
  const int z = blockIdx.z;
  const int kb_begin = (int)(((long long)z * nkb) / ks);
  const int kb_end = (int)(((long long)(z + 1) * nkb) / ks);

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], Roles<SWAP>::EPI * 32);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&tmem_slot, tmem_cols<BN>());
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_slot;
  // split K: announce that this CTA is running; peers wait on it before
  // their first store into this CTA's shared memory
  if (ks > 1) tc::cluster_arrive_relaxed();

  pdl_trigger();
  if (warp == Roles<SWAP>::PRODUCER) {
    // ---- TMA producer ----
    if (lane == 0) {
      const uint32_t bytes = (uint32_t)stage_bytes<BN>();
      const int nloc = kb_end - kb_begin;
      const int my_tiles = (t_first < ntiles) ? (ntiles - t_first + t_step - 1) / t_step : 0;
      const int total = my_tiles * nloc;
      // load iteration -> (A row, B row, K column of the weights, activation K offset)
      auto coords = [&](int it, int& a0, int& b0, int& k, int& koff) {
        const int t = t_first + (it / nloc) * t_step;
        a0 = (t % ntA) * BM;
        b0 = (t / ntA) * BN;
        k = (kb_begin + it % nloc) * BK;
        koff = ((SWAP ? a0 : b0) >= xk_split) ? xk_off : 0;
      };
      auto load_w = [&](int it, int s) {  // the weight operand
        int a0, b0, k, koff;
        coords(it, a0, b0, k, koff);
        if (SWAP) tc::tma_load_2d(sA + (size_t)s * BM * BK, &mapA, k, a0, &full[s]);
        else tc::tma_load_2d(sB + (size_t)s * BN * BK, &mapB, k, b0, &full[s]);
      };
      auto load_x = [&](int it, int s) {  // the activation operand
        int a0, b0, k, koff;
        coords(it, a0, b0, k, koff);
        if (SWAP) tc::tma_load_2d(sB + (size_t)s * BN * BK, &mapB, k + koff, b0, &full[s]);
        else tc::tma_load_2d(sA + (size_t)s * BM * BK, &mapA, k + koff, a0, &full[s]);
      };
      // weights do not depend on earlier kernels: fill the first ring with
      // them while the previous kernel finishes, then wait for it
      const int pre = total < stages ? total : stages;
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(&full[it], bytes);
        load_w(it, it);
      }
      pdl_wait();
      for (int it = 0; it < pre; ++it) load_x(it, it);
      for (int it = pre; it < total; ++it) {
        const int s = it % stages;
        mbar_wait_bounded(&empty[s], ((it / stages) + 1) & 1, status);
        mbar_arrive_expect_tx(&full[s], bytes);
        load_w(it, s);
        load_x(it, s);
      }
    }
  } else if (warp == Roles<SWAP>::MMA) {
    // ---- MMA issuer ----
    pdl_wait();
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_m128(BN);
      int it = 0, tl = 0;
      for (int t = t_first; t < ntiles; t += t_step, ++tl) {
        const int buf = tl & 1;
        if (tl >= 2) mbar_wait_bounded(&acc_empty[buf], ((tl >> 1) + 1) & 1, status);
        tc::fence_after();
        const uint32_t dt = tmem + (uint32_t)(buf * BN);
        for (int kb = kb_begin; kb < kb_end; ++kb, ++it) {
          const int s = it % stages;
          mbar_wait_bounded(&full[s], (it / stages) & 1, status);
          tc::fence_after();
          const uint64_t da = tc::desc_sw128(smem_u32(sA + (size_t)s * BM * BK));
          const uint64_t db = tc::desc_sw128(smem_u32(sB + (size_t)s * BN * BK));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)  // 32 bytes per K slice: +2 in 16-byte units
            tc::mma_bf16(dt, da + 2 * kk, db + 2 * kk, idesc, (kb > kb_begin || kk > 0) ? 1u : 0u);
          tc::commit(&empty[s]);
        }
        tc::commit(&acc_full[buf]);
      }
    }
  } else {
    // ---- epilogue warps: TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31 ----
    pdl_wait();  // outputs may still be read by earlier kernels
    const int quarter = warp & 3;     // TMEM lane quarter
    const int r = quarter * 32 + lane;  // row of A = TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    // fused rotary: the rotate-half partner of feature f is f ^ (rot/2), held
    // by lane ^ (rot/2) of the same warp (heads are 32-feature aligned)
    const bool rope = SWAP && e.kind == EPI_QKV1_ROPE;
    const int rhalf = e.rot >> 1;
    int tl = 0;
    for (int t = t_first; t < ntiles; t += t_step, ++tl) {
      const int buf = tl & 1;
      const int a0 = (t % ntA) * BM, b0 = (t / ntA) * BN;
      mbar_wait_bounded(&acc_full[buf], (tl >> 1) & 1, status);
      tc::fence_after();
      const uint32_t tb = trow + (uint32_t)(buf * BN);
      if (ks > 1) {
        // push this CTA's partial columns to their owners, four columns per
        // 16-byte store: column quad c..c+3 goes to rank c / (BN/ks), float4
        // slot [my rank][(c % (BN/ks)) / 4][row] of its receive buffer
        // (BN/ks is a multiple of 4; remote stores do not wait for a round
        // trip)
        namespace cg = cooperative_groups;
        cg::cluster_group cluster = cg::this_cluster();
        const uint32_t recv = smem_u32(smem + (size_t)stages * stage_bytes<BN>());
        const int cpr = BN / ks, qpr = cpr / 4;
        const int me = (int)cluster.block_rank();
        tc::cluster_wait_acquire();  // every CTA of the cluster has started
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16];
          tc::tmem_ld16(tb + c0, v);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = c0 + 4 * u;
            const uint32_t slot = recv + (uint32_t)((((me * qpr + (c % cpr) / 4) * BM) + r) * 16);
            tc::st_cluster_v4(tc::map_rank(slot, (uint32_t)(c / cpr)), v[4 * u], v[4 * u + 1],
                              v[4 * u + 2], v[4 * u + 3]);
          }
        }
      } else if (SWAP && BN <= 64 && e.kind == EPI_LOGITS_ARGMAX) {
        // LM head: logits (optional) and the tile's argmax per token column:
        // warp shuffles, then the four warps through shared memory
        const int n = a0 + r;
        float* logits = reinterpret_cast<float*>(e.out0);
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16];
          tc::tmem_ld16(tb + c0, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = b0 + c0 + j;
            if (logits && m < M && n < N) logits[(size_t)m * e.ld0 + n] = v[j];
            float bv = (n < N) ? v[j] : -INFINITY;
            int bi = n;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
              const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
              if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
            }
            if (lane == 0) s_arg[warp][c0 + j] = make_float2(bv, __int_as_float(bi));
          }
        }
        tc::fence_before();
        mbar_arrive(&acc_empty[buf]);
        asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
        if (r < BN && b0 + r < M) {
          float2 best = s_arg[0][r];
#pragma unroll
          for (int w = 1; w < 4; ++w) {
            const float2 o = s_arg[w][r];
            if (o.x > best.x || (o.x == best.x && __float_as_int(o.y) < __float_as_int(best.y)))
              best = o;
          }
          reinterpret_cast<float2*>(e.aux)[(size_t)(t % ntA) * M + b0 + r] = best;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");  // s_arg reused by the next tile
      } else if (BN <= 64) {
        // drain the whole accumulator first, release it, then store
        float v[BN];
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 16) tc::tmem_ld16(tb + c0, v + c0);
        tc::fence_before();
        mbar_arrive(&acc_empty[buf]);
        if constexpr (SWAP) {
          const int n = a0 + r;
#pragma unroll
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float pv[16];
            if (rope) {
#pragma unroll
              for (int j = 0; j < 16; ++j) pv[j] = __shfl_xor_sync(0xffffffffu, v[c0 + j], rhalf);
            }
            if (n < N && b0 + c0 < M) epi_cols<bf16, 16>(e, b0 + c0, 16, n, M, v + c0, pv);
          }
        } else {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            const int m = a0 + r, n = b0 + c;
            if (m < M && n < N) epi_apply<bf16>(e, m, n, v[c]);
          }
        }
        if (SWAP && e.ln_cnt) post_ln(e, b0, b0 + BN, M, N, ntA, s_rows, &s_nrows);
      } else if (!SWAP) {
        // activations as A: TMEM lane = token row. Transpose 32 x 32 blocks
        // through this warp's shared-memory tile so that one store
        // instruction covers 32 consecutive output columns of one row
        float* tile = reinterpret_cast<float*>(smem + (size_t)stages * stage_bytes<BN>()) + warp * 32 * 33;
        // the two warps of a lane quarter take the two halves of the columns
        constexpr int CW = BN / (Roles<SWAP>::EPI / 4);
        const int cbeg = (warp >> 2) * CW;
        for (int c0 = cbeg; c0 < cbeg + CW; c0 += 32) {
          float v[32];
          tc::tmem_ld16(tb + c0, v);
          tc::tmem_ld16(tb + c0 + 16, v + 16);
#pragma unroll
          for (int j = 0; j < 32; ++j) tile[lane * 33 + j] = v[j];
          __syncwarp();
          // the lane's column n is fixed over the block's 32 rows: the
          // chunked epilogue issues a 16-row chunk's loads (bias, residual)
          // before its stores
          const int n = b0 + c0 + lane;
          const int m0 = a0 + quarter * 32;
#pragma unroll
          for (int rr0 = 0; rr0 < 32; rr0 += 16) {
            float vv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) vv[j] = tile[(rr0 + j) * 33 + lane];
            if (n < N && m0 + rr0 < M) epi_cols<bf16, 16>(e, m0 + rr0, 16, n, M, vv, nullptr);
          }
          __syncwarp();
        }
        tc::fence_before();
        mbar_arrive(&acc_empty[buf]);
      } else {
        // weights as A with BN > 64 (the activations-as-A path is above)
        const int n = a0 + r;
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16], pv[16];
          tc::tmem_ld16(tb + c0, v);
          if (rope) {
#pragma unroll
            for (int j = 0; j < 16; ++j) pv[j] = __shfl_xor_sync(0xffffffffu, v[j], rhalf);
          }
          if (n < N && b0 + c0 < M) epi_cols<bf16, 16>(e, b0 + c0, 16, n, M, v, pv);
        }
        tc::fence_before();
        mbar_arrive(&acc_empty[buf]);
        if (SWAP && e.ln_cnt) post_ln(e, b0, b0 + BN, M, N, ntA, s_rows, &s_nrows);
      }
    }
  }

  if (ks > 1) {
    // every partial has been pushed once all ranks pass this barrier (every
    // thread of every CTA takes part); then rank q sums, in rank order
    // (deterministic), the ks slices of its columns [q*BN/ks, (q+1)*BN/ks)
    // from its own shared memory. Nobody touches another CTA's shared
    // memory after the barrier, so no second barrier is needed.
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    if (warp >= Roles<SWAP>::EPI) tc::cluster_wait_acquire();  // producer / MMA warps: first phase
    tc::cluster_arrive_release();               // second phase: all pushes done
    tc::cluster_wait_acquire();
    if (warp < Roles<SWAP>::EPI) {
      const int r = warp * 32 + lane;
      const bool rope = SWAP && e.kind == EPI_QKV1_ROPE;
      const int rhalf = e.rot >> 1;
      const int a0 = (t_first % ntA) * BM, b0 = (t_first / ntA) * BN;
      const uint32_t recv = smem_u32(smem + (size_t)stages * stage_bytes<BN>());
      const int cpr = BN / ks, qpr = cpr / 4;
      const int cbeg = (int)cluster.block_rank() * cpr;
      // split K is weights-as-A only: feature n = a0 + r, rows b0 + c.
      // Chunks of up to 16 rows: the partial sums first (shared-memory
      // loads only), then the epilogue's loads, then its stores.
      const int n = a0 + r;
      for (int cc0 = 0; cc0 < cpr; cc0 += 16) {
        const int cnt = (cpr - cc0 < 16) ? cpr - cc0 : 16;
        float acc[16], pv[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          // the ks partials of column quad cc0/4 + u, summed in rank order,
          // four ranks' loads in flight at a time
          const int q = cc0 / 4 + u;
          float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int p0 = 0; p0 < MAX_KS; p0 += 4) {
            if (p0 >= ks) break;
            float4 part[4];
#pragma unroll
            for (int p = 0; p < 4; ++p)
              if (p0 + p < ks && 4 * u < cnt)
                part[p] = tc::ld_shared_v4(recv + (uint32_t)((((p0 + p) * qpr + q) * BM + r) * 16));
#pragma unroll
            for (int p = 0; p < 4; ++p)
              if (p0 + p < ks && 4 * u < cnt) {
                t.x += part[p].x;
                t.y += part[p].y;
                t.z += part[p].z;
                t.w += part[p].w;
              }
          }
          acc[4 * u] = t.x;
          acc[4 * u + 1] = t.y;
          acc[4 * u + 2] = t.z;
          acc[4 * u + 3] = t.w;
        }
        if (rope) {
#pragma unroll
          for (int j = 0; j < 16; ++j) pv[j] = __shfl_xor_sync(0xffffffffu, acc[j], rhalf);
        }
        const int m0 = b0 + cbeg + cc0;
        if (n < N && m0 < M) epi_cols<bf16, 16>(e, m0, cnt, n, M, acc, pv);
      }
      if (SWAP && e.ln_cnt) post_ln(e, b0 + cbeg, b0 + cbeg + cpr, M, N, ntA, s_rows, &s_nrows);
    }
  }

  tc::fence_before();
  __syncthreads();
  if (warp == 0)
    tc::tmem_free(tmem, tmem_cols<BN>());
}

// ---- host side -------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major bf16 matrix [rows, cols] with row stride ld (elements); box of
// 64 columns x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dynamic shared memory ceiling of one instantiation: the device's opt-in
// per-block limit less the kernel's static shared memory.
template <int BN, bool SWAP>
size_t& dyn_smem_max() {
  static size_t v = 0;
  return v;
}

template <int BN, bool SWAP>
cudaError_t prepare_one() {
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaFuncAttributes fa;
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, gemm_tc_kernel<BN, SWAP>);
  if (e != cudaSuccess) return e;
  const size_t mx = (size_t)optin - fa.sharedSizeBytes;
  e = cudaFuncSetAttribute(gemm_tc_kernel<BN, SWAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)mx);
  // split-K clusters of up to 16 CTAs (above the portable 8)
  if (e == cudaSuccess && SWAP)
    e = cudaFuncSetAttribute(gemm_tc_kernel<BN, SWAP>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) dyn_smem_max<BN, SWAP>() = mx;
  return e;
}

int sm_count() { return device_sm_count(); }

// Ring depth and dynamic shared memory of one launch with ks K splits.
template <int BN, bool SWAP>
size_t launch_smem(int nkb, int ks, int* stages_out) {
  constexpr size_t SB = stage_bytes<BN>();
  const size_t SMEM_MAX = dyn_smem_max<BN, SWAP>();
  const int nloc = (nkb + ks - 1) / ks;
  int stages = (int)((SMEM_MAX - 1024) / SB);
  if (stages > MAX_STAGES) stages = MAX_STAGES;
  size_t recv_bytes = 0;
  if (ks > 1) {
    // one tile per CTA: no deeper ring than its K blocks, plus a receive
    // buffer for the [BN][BM] fp32 partials pushed by the cluster
    recv_bytes = (size_t)BN * BM * 4;
    int fit = (int)((SMEM_MAX - 1024 - recv_bytes) / SB);
    stages = nloc < stages ? nloc : stages;
    if (stages > fit) stages = fit;
  }
  // activations as A: per-warp 32 x 33 fp32 transpose tiles for the epilogue
  const size_t tr_bytes = SWAP ? 0 : (size_t)Roles<SWAP>::EPI * 32 * 33 * 4;
  if (!SWAP) {
    int fit = (int)((SMEM_MAX - 1024 - tr_bytes) / SB);
    if (stages > fit) stages = fit;
  }
  if (stages < 2) stages = 2;
  *stages_out = stages;
  return (size_t)stages * SB + recv_bytes + tr_bytes + 1024;
}

// CTAs of ks-CTA clusters that fit on the device at once with this much
// shared memory (the occupancy calculator's cluster count times ks), cached
// per device, instantiation, split and size.
template <int BN, bool SWAP>
int resident_ctas(int ks, size_t smem) {
  struct Entry { int dev, ks; size_t smem; int ctas; };
  static Entry cache[64];
  static int n_cache = 0;
  const int dev = current_device();
  for (int i = 0; i < n_cache; ++i)
    if (cache[i].dev == dev && cache[i].ks == ks && cache[i].smem == smem) return cache[i].ctas;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, ks);
  cfg.blockDim = dim3(Roles<SWAP>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = ks;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, gemm_tc_kernel<BN, SWAP>, &cfg) != cudaSuccess) {
    cudaGetLastError();  // not sticky: clear it
    clusters = 0;
  }
  const int ctas = clusters * ks;
  if (n_cache < 64) cache[n_cache++] = Entry{dev, ks, smem, ctas};
  return ctas;
}

// K splits of a weights-as-A launch with nt feature tiles and nkb K blocks:
// the largest power of two <= 16 whose nt * ks CTAs all fit on the device
// at once (one wave: the cluster shape limits residency below one CTA per
// SM) with at least one K block per split; 1 (persistent over the tiles)
// when even two splits do not fit.
template <int BN>
int plan_splits(int nt, int nkb) {
  for (int ks = MAX_KS; ks >= 2; ks >>= 1) {
    if (nkb < ks || BN / ks < 4) continue;  // a K block per split; column quads per rank
    int stages = 0;
    const size_t smem = launch_smem<BN, true>(nkb, ks, &stages);
    if (nt * ks <= resident_ctas<BN, true>(ks, smem)) return ks;
  }
  return 1;
}

template <int BN, bool SWAP>
cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mb, int M, int N, int nkb,
                       int ks, int ntA, int ntB, int xk_split, int xk_off, const Epi& e,
                       int* status, cudaStream_t s) {
  constexpr size_t SB = stage_bytes<BN>();
  if (dyn_smem_max<BN, SWAP>() < 3 * SB) return cudaErrorInvalidConfiguration;
  int stages = 0;
  const size_t smem = launch_smem<BN, SWAP>(nkb, ks, &stages);
  const int ntiles = ntA * ntB;
  dim3 grid;
  if (ks > 1) {
    grid = dim3(ntiles, 1, ks);
  } else {
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemm_tc_kernel<BN, SWAP>, Roles<SWAP>::THREADS, smem);
    if (per_sm < 1) per_sm = 1;
    const int slots = sm_count() * per_sm;
    grid = dim3(ntiles < slots ? ntiles : slots, 1, 1);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(Roles<SWAP>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = ks;  // the K splits of one tile form a cluster
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, SWAP>, ma, mb, M, N, nkb, ks,
                                       stages, ntA, ntB, xk_split, xk_off, e, status);
  note_launch();
  return err;
}

int swap_bn(int M) {
  int bn = 32;
  while (bn < M) bn <<= 1;
  return bn;
}

}  // namespace

cudaError_t gemm_tc_prepare() {
  // kernel attributes apply to the current device only
  static bool done[MAX_DEVICES] = {};
  const int dev = current_device();
  if (dev >= 0 && done[dev]) return cudaSuccess;
  cudaError_t e;
  if ((e = prepare_one<32, true>()) != cudaSuccess) return e;
  if ((e = prepare_one<64, true>()) != cudaSuccess) return e;
  if ((e = prepare_one<128, true>()) != cudaSuccess) return e;
  if ((e = prepare_one<256, true>()) != cudaSuccess) return e;
  if ((e = prepare_one<256, false>()) != cudaSuccess) return e;
  if (dev >= 0) done[dev] = true;
  return cudaSuccess;
}

size_t gemm_scratch_bytes(int max_M, int max_N) { return PART_BUDGET; }
int gemm_counter_count(int max_N) { return (max_N + BM - 1) / BM + 64; }

int gemm_rope_fusable(int dt, int M, int N, int K, int xk_split, int xk_off, int d_head, int rot) {
  if (!gemm_tc_supported(dt, M, N, K, xk_split, xk_off) || M > 256) return 0;
  const int half = rot / 2;
  // partner lane = lane ^ half inside a warp: half a power of two <= 16,
  // heads at least one warp (32 features) wide
  if (d_head < 32 || half < 1 || half > 16 || (half & (half - 1))) return 0;
  return 1;
}

int gemm_argmax_fusable(int dt, int M, int N, int K) {
  return (gemm_tc_supported(dt, M, N, K, 1 << 30, 0) && M <= 64) ? 1 : 0;
}

int gemm_tc_supported(int dt, int M, int N, int K, int xk_split, int xk_off) {
  if (dt != DT_BF16 || M < 1 || N < 1 || K < BK || (K % BK)) return 0;
  if (encoder() == nullptr) return 0;
  const int ftile = (M <= 256) ? BM : 256;
  if (xk_split < N && (xk_split % ftile)) return 0;
  if (xk_off % 8) return 0;
  return 1;
}

cudaError_t launch_gemm_tc(int dt, const void* X, int ldx, const void* W, int ldw, int M, int N,
                           int K, int xk_split, int xk_off, const Epi& e,
                           const GemmScratch& scr, int* status, cudaStream_t s) {
  cudaError_t err = gemm_tc_prepare();
  if (err != cudaSuccess) return err;
  const int nkb = K / BK;
  const int xcols = (xk_split < N) ? xk_off + K : K;  // columns of X any tile reads
  CUtensorMap ma, mb;
  if (M <= 256) {
    const int BN = swap_bn(M);
    const int nt = (N + BM - 1) / BM;
    if (!make_map(&ma, W, N, K, ldw, BM) || !make_map(&mb, X, M, xcols, ldx, BN))
      return cudaErrorInvalidValue;
    // K splits: as many as fit in one wave (plan_splits); without a split
    // the kernel runs persistent over the tiles. The argmax epilogue needs
    // whole tiles.
    int ks = 1;
    if (e.kind != EPI_LOGITS_ARGMAX) {
      switch (BN) {
        case 32: ks = plan_splits<32>(nt, nkb); break;
        case 64: ks = plan_splits<64>(nt, nkb); break;
        case 128: ks = plan_splits<128>(nt, nkb); break;
        default: ks = plan_splits<256>(nt, nkb); break;
      }
    }
    switch (BN) {
      case 32: return launch_one<32, true>(ma, mb, M, N, nkb, ks, nt, 1, xk_split, xk_off, e, status, s);
      case 64: return launch_one<64, true>(ma, mb, M, N, nkb, ks, nt, 1, xk_split, xk_off, e, status, s);
      case 128: return launch_one<128, true>(ma, mb, M, N, nkb, ks, nt, 1, xk_split, xk_off, e, status, s);
      default: return launch_one<256, true>(ma, mb, M, N, nkb, ks, nt, 1, xk_split, xk_off, e, status, s);
    }
  }
  constexpr int BNP = 256;
  if (!make_map(&ma, X, M, xcols, ldx, BM) || !make_map(&mb, W, N, K, ldw, BNP))
    return cudaErrorInvalidValue;
  return launch_one<BNP, false>(ma, mb, M, N, nkb, 1, (M + BM - 1) / BM, (N + BNP - 1) / BNP,
                                xk_split, xk_off, e, status, s);
}

}  // namespace bt
