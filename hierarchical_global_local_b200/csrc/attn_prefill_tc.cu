// attn_prefill_tc.cu -- causal attention of the block decoder at prefill on
// the 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
//
// "Block Transformer: Global-to-Local Language Modeling for Fast Inference",
// §3.4 "The Block Decoder": standard causal self-attention over the n block
// embeddings of the prompt (n = T / L_B).
//
// One CTA per (sequence, head, 128-query tile), flash-attention style:
//   S = Q K^T           tcgen05.mma, M = 128 queries, N = 128 keys, into TMEM
//   P = softmax pieces  4 warps, one query row per thread (tcgen05.ld), online
//                       max / sum, causal + tail masking (only on the
//                       diagonal and tail tiles), P written to shared memory
//                       in the 128-byte-swizzled K-major layout
//   O += P V            tcgen05.mma, M = 128, N = d, K = 128 keys: O stays in
//                       TMEM across the key tiles and is rescaled there when
//                       a row's running max grows by more than 8 (log2)
// The MMA warp issues S of tile j+1 before P_j V_j, so the softmax's max pass
// over the next tile overlaps P V.
// Operands come in by TMA with 3-D tensor maps bounded per (sequence, head),
// so keys / queries past n read as zeros (no stale cache bytes reach the
// products). V is read through its transpose V^T [B*H][d][n_pad] (written
// next to the cache during prefill), so both MMAs take K-major operands.
// Warps: 0-3 softmax/epilogue, 4 TMA producer, 5 MMA issuer. All waits are
// bounded.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace bt {

// 2^x by the special-function unit's approximation (PTX ex2.approx.ftz.f32;
// subnormal results flush to zero, so a softmax weight below 2^-126 of the
// row's largest counts as 0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

namespace {

constexpr int QT = 128;   // queries per CTA (MMA M)
constexpr int KT = 128;   // keys per tile (MMA N of S, K of P V)
constexpr int THREADS = 192;

// shared memory plan (bytes), all tiles 1024-aligned
template <int DH>
struct Plan {
  static constexpr int KB = DH / 64;                  // 64-wide K blocks of Q and K
  static constexpr int Q_BYTES = QT * DH * 2;         // KB blocks of [128 x 64]
  static constexpr int K_BYTES = KT * DH * 2;         // per stage
  static constexpr int VT_BYTES = DH * KT * 2;        // per stage: 2 blocks of [DH x 64 keys]
  static constexpr int P_BYTES = QT * KT * 2;         // 2 blocks of [128 x 64 keys]
  static constexpr int STAGES = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_VT = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_P = OFF_VT + STAGES * VT_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;     // mbarriers and the TMEM slot
  static constexpr int BAR_BYTES = 128;
  // CTAs per SM: two for d_head 64 (their shared memory, with the 1 KB the
  // system keeps per block, fits the SM's 228 KB only without static shared
  // variables -- hence the barriers in the dynamic allocation), else one
  static constexpr int CTAS = DH == 64 ? 2 : 1;
  static constexpr int LIMIT = 233472 / CTAS - 1024;
  static constexpr int NEED = OFF_BAR + BAR_BYTES;
  static constexpr int BYTES = NEED + 1024 < LIMIT ? NEED + 1024 : LIMIT;
  static constexpr int SLACK = BYTES - NEED;           // room for aligning the base to 1024
  static constexpr int TMEM_COLS = 256;               // S: 128 columns, O: DH columns
  static_assert(SLACK >= 0, "shared-memory plan");
};

template <int DH>
__global__ void __launch_bounds__(THREADS, Plan<DH>::CTAS)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                       const __grid_constant__ CUtensorMap mVt, int H, int n, bf16* __restrict__ out,
                       int ld_out, float scale_log2, int* status, int g) {
  using PL = Plan<DH>;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  // the plan leaves SLACK bytes for aligning the base; a base further off
  // (none in practice: the kernel has no static shared variables) is
  // reported instead of overrunning the allocation
  if ((size_t)(sm - smem_raw) > (size_t)PL::SLACK) {
    if (threadIdx.x == 0) set_status(status, ST_BAD_ARGS);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 1 + PL::STAGES;
  uint64_t* s_full = bars + 1 + 2 * PL::STAGES;
  uint64_t* p_full = s_full + 1;
  uint64_t* o_full = s_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 3);

  // longest first: CTAs are numbered q-tile-major from the last (causal)
  // q-tile down, so the tiles with the most key tiles start first and the
  // one-key-tile ones fill the tail
  const int nqt = (n + QT - 1) / QT;
  const int BH = gridDim.x / nqt;
  const int qt = nqt - 1 - (int)(blockIdx.x / BH);
  const int bh = blockIdx.x % BH;  // b * H + h
  const int b = bh / H, h = bh - b * H;
  const int kvh = b * (H / g) + h / g;  // key/value head (grouped-query attention)
  const int q0 = qt * QT;
  const int ntiles = (q0 + QT - 1) / KT + 1;  // key tiles intersecting the causal band
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < PL::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, PL::TMEM_COLS);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + KT;
  pdl_wait();

  if (warp == 4) {
    if (lane == 0) {
      // Q tile (KB blocks of 64 dims), then K / V^T tiles through the ring
      mbar_arrive_expect_tx(q_full, PL::Q_BYTES);
      for (int kb = 0; kb < PL::KB; ++kb)
        tc::tma_load_3d(sm + PL::OFF_Q + kb * QT * 128, &mQ, h * DH + kb * 64, q0, b, q_full);
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % PL::STAGES;
        if (j >= PL::STAGES) mbar_wait_bounded(&kv_empty[s], ((j / PL::STAGES) + 1) & 1, status);
        mbar_arrive_expect_tx(&kv_full[s], PL::K_BYTES + PL::VT_BYTES);
        for (int kb = 0; kb < PL::KB; ++kb)
          tc::tma_load_3d(sm + PL::OFF_K + s * PL::K_BYTES + kb * KT * 128, &mK, kb * 64, j * KT, kvh, &kv_full[s]);
        for (int kb = 0; kb < KT / 64; ++kb)
          tc::tma_load_3d(sm + PL::OFF_VT + s * PL::VT_BYTES + kb * DH * 128, &mVt, j * KT + kb * 64, 0, kvh,
               &kv_full[s]);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16_m128(KT), idO = tc::idesc_bf16_m128(DH);
      mbar_wait_bounded(q_full, 0, status);
      // S = Q K^T of key tile j (stage j % STAGES) over DH (KB blocks x 4
      // slices of 16) into the S columns
      auto issue_s = [&](int j) {
        const int s = j % PL::STAGES;
        mbar_wait_bounded(&kv_full[s], (j / PL::STAGES) & 1, status);
        tc::fence_after();
        for (int kb = 0; kb < PL::KB; ++kb) {
          const uint64_t dq = tc::desc_sw128(smem_u32(sm + PL::OFF_Q + kb * QT * 128));
          const uint64_t dk = tc::desc_sw128(smem_u32(sm + PL::OFF_K + s * PL::K_BYTES + kb * KT * 128));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(tS, dq + 2 * kk, dk + 2 * kk, idS, (kb | kk) ? 1u : 0u);
        }
        tc::commit(s_full);
      };
      issue_s(0);
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % PL::STAGES;
        // P_j is written (the softmax is done reading S_j, and O has been
        // rescaled where the running max moved): S_{j+1} goes first, so the
        // softmax's max pass over tile j+1 overlaps P_j V_j
        mbar_wait_bounded(p_full, j & 1, status);
        tc::fence_after();
        if (j + 1 < ntiles) issue_s(j + 1);
        // O += P_j V_j over the 128 keys (2 blocks x 4 slices of 16); O
        // accumulates in TMEM across the key tiles
        for (int kb = 0; kb < KT / 64; ++kb) {
          const uint64_t dp = tc::desc_sw128(smem_u32(sm + PL::OFF_P + kb * QT * 128));
          const uint64_t dv = tc::desc_sw128(smem_u32(sm + PL::OFF_VT + s * PL::VT_BYTES + kb * DH * 128));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(tO, dp + 2 * kk, dv + 2 * kk, idO, (j | kb | kk) ? 1u : 0u);
        }
        tc::commit(o_full);
        tc::commit(&kv_empty[s]);
      }
    }
  } else {
    // ---- softmax / epilogue: thread r owns query row q0 + r ----
    const int r = warp * 32 + lane;
    const int qi = q0 + r;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m = -INFINITY, l = 0.f;
    uint8_t* prow = sm + PL::OFF_P;
    for (int j = 0; j < ntiles; ++j) {
      mbar_wait_bounded(s_full, j & 1, status);
      tc::fence_after();
      const int k0 = j * KT;
      // every key of the tile is visible to every query row of the CTA (left
      // of the diagonal, inside n): no per-element masking (warp-uniform)
      const bool full = (k0 + KT - 1 <= q0) && (k0 + KT <= n);
      // pass 1: row max over this tile (masked keys excluded), 32 columns at a time
      // (eight independent max chains: two softmax warps share a scheduler,
      // so one 128-long dependency chain per row would leave it idle)
      float mx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
      if (full) {
        // the scale is positive: scale the raw maximum once
#pragma unroll
        for (int c = 0; c < KT; c += 32) {
          float sv[32];
          tc::tmem_ld32(tS + lane_base + c, sv);
#pragma unroll
          for (int u = 0; u < 32; ++u) mx[u & 7] = fmaxf(mx[u & 7], sv[u]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < KT; c += 32) {
          float sv[32];
          tc::tmem_ld32(tS + lane_base + c, sv);
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int kj = k0 + c + u;
            if (kj <= qi && kj < n) mx[u & 7] = fmaxf(mx[u & 7], sv[u]);
          }
        }
      }
      float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                         fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      if (tmax != -INFINITY) tmax *= scale_log2;
      // the running max m moves only when the tile's exceeds it by more than
      // 8 (log2 units): the weights exp2(s - m) then stay below 2^8, which
      // bf16 holds at the same relative precision, and l uses the same m, so
      // O / l is unchanged while most tiles skip rescaling O
      const bool grow = (m == -INFINITY) || (tmax > m + 8.f);
      const float mn = grow ? fmaxf(m, tmax) : m;
      const float corr = (!grow || mn == -INFINITY || m == -INFINITY) ? 1.f : exp2f(m - mn);
      if (j > 0) {
        // O holds sum_{i<j} P_i V_i at the old maxima: once P_{j-1} V_{j-1}
        // is in, rescale the rows whose running max moved (warp-uniform: the
        // TMEM accesses are warp-collective), before P_j V_j accumulates
        mbar_wait_bounded(o_full, (j - 1) & 1, status);
        tc::fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
          for (int c = 0; c < DH; c += 16) {
            float ov[16];
            tc::tmem_ld16(tO + lane_base + c, ov);
#pragma unroll
            for (int u = 0; u < 16; ++u) ov[u] *= corr;
            tc::tmem_st16(tO + lane_base + c, ov);
          }
          tc::tmem_wait_st();
        }
      }
      // pass 2: P = exp2(s - mn) as bf16 into the swizzled K-major tile
      // (eight partial row sums, one per position in an 8-key chunk)
      float ls[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ls[u] = 0.f;
#pragma unroll
      for (int c = 0; c < KT; c += 32) {
        float sv[32];
        tc::tmem_ld32(tS + lane_base + c, sv);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          float p[8];
          if (full) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              p[u] = ex2_approx(fmaf(sv[c8 * 8 + u], scale_log2, -mn));
              ls[u] += p[u];
            }
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int kj = k0 + c + c8 * 8 + u;
              p[u] = (kj <= qi && kj < n) ? ex2_approx(fmaf(sv[c8 * 8 + u], scale_log2, -mn)) : 0.f;
              ls[u] += p[u];
            }
          }
          __nv_bfloat162 h0 = __floats2bfloat162_rn(p[0], p[1]), h1 = __floats2bfloat162_rn(p[2], p[3]);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(p[4], p[5]), h3 = __floats2bfloat162_rn(p[6], p[7]);
          uint4 w;
          w.x = *reinterpret_cast<uint32_t*>(&h0); w.y = *reinterpret_cast<uint32_t*>(&h1);
          w.z = *reinterpret_cast<uint32_t*>(&h2); w.w = *reinterpret_cast<uint32_t*>(&h3);
          const int col8 = (c >> 3) + c8;          // 8-key chunk index within the 128 keys
          const int kb = col8 >> 3, chunk = col8 & 7;  // 64-key block, 16-byte chunk in the row
          uint8_t* dst = prow + kb * QT * 128 + r * 128 + ((chunk ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = w;
        }
      }
      fence_proxy_async();  // P visible to the tensor core
      tc::fence_before();
      mbar_arrive(p_full);
      const float lt = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      l = l * corr + lt;
      m = mn;
    }
    // the last P V is in: O / l, read from TMEM 16 columns at a time
    mbar_wait_bounded(o_full, (ntiles - 1) & 1, status);
    tc::fence_after();
    const float inv = (qi < n && l > 0.f) ? 1.f / l : 0.f;
    bf16* dst = out + ((size_t)b * n + qi) * ld_out + h * DH;
#pragma unroll
    for (int c = 0; c < DH; c += 16) {
      float ov[16];
      tc::tmem_ld16(tO + lane_base + c, ov);
      if (qi < n) {
#pragma unroll
        for (int e = 0; e < 16; e += 8) {
          __nv_bfloat162 h0 = __floats2bfloat162_rn(ov[e] * inv, ov[e + 1] * inv);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(ov[e + 2] * inv, ov[e + 3] * inv);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(ov[e + 4] * inv, ov[e + 5] * inv);
          __nv_bfloat162 h3 = __floats2bfloat162_rn(ov[e + 6] * inv, ov[e + 7] * inv);
          uint4 w;
          w.x = *reinterpret_cast<uint32_t*>(&h0); w.y = *reinterpret_cast<uint32_t*>(&h1);
          w.z = *reinterpret_cast<uint32_t*>(&h2); w.w = *reinterpret_cast<uint32_t*>(&h3);
          *reinterpret_cast<uint4*>(dst + c + e) = w;
        }
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0)
    tc::tmem_free(tmem, PL::TMEM_COLS);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn enc3() {
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

// 3-D bf16 map {x (contiguous), y, z}, strides in elements for y and z, box
// {64, by, 1}, 128-byte swizzle, zero fill outside [0, dims).
bool map3(CUtensorMap* m, const void* base, long long x, long long y, long long z, long long sy,
          long long sz, int by) {
  EncodeTiledFn f = enc3();
  if (!f) return false;
  cuuint64_t dims[3] = {(cuuint64_t)x, (cuuint64_t)y, (cuuint64_t)z};
  cuuint64_t str[2] = {(cuuint64_t)sy * 2, (cuuint64_t)sz * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)by, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, str, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DH>
cudaError_t launch_tc(const void* q, int ldq, const void* kc, const void* vt, int vt_ld, int B,
                      int H, int cap, int n, void* out, int ld_out, int* status, cudaStream_t s, int Hk) {
  // the attribute applies to the current device only
  static bool prepared[MAX_DEVICES] = {};
  const int dev = current_device();
  if (dev < 0 || !prepared[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_tc_kernel<DH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Plan<DH>::BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0) prepared[dev] = true;
  }
  CUtensorMap mQ, mK, mVt;
  // Q rows b*n + i, dims (h*d + e): {ldq cols, n rows, B}
  if (!map3(&mQ, q, ldq, n, B, ldq, (long long)n * ldq, QT)) return cudaErrorInvalidValue;
  // K cache [B*Hk][cap][d], valid rows < n
  if (!map3(&mK, kc, DH, n, (long long)B * Hk, DH, (long long)cap * DH, KT)) return cudaErrorInvalidValue;
  // V^T [B*Hk][d][vt_ld], valid keys < n
  if (!map3(&mVt, vt, n, DH, (long long)B * Hk, vt_ld, (long long)DH * vt_ld, DH)) return cudaErrorInvalidValue;
  const int nqt = (n + QT - 1) / QT;
  const float scale = 1.4426950408889634f / sqrtf((float)DH);
  BT_LAUNCH(attn_prefill_tc_kernel<DH>, dim3(B * H * nqt), dim3(THREADS), Plan<DH>::BYTES, s, mQ, mK,
            mVt, H, n, (bf16*)out, ld_out, scale, status, H / Hk);
  return cudaSuccess;
}

}  // namespace

int attn_prefill_tc_supported(int dt, int d, int ldq, int vt_ld) {
  return (dt == DT_BF16 && (d == 64 || d == 128) && (ldq % 8) == 0 && (vt_ld % 8) == 0 &&
          enc3() != nullptr)
             ? 1
             : 0;
}

cudaError_t launch_attn_prefill_tc(const void* q, int ldq, const void* k_cache, const void* vt,
                                   int vt_ld, int B, int H, int d, int cap, int n, void* out,
                                   int ld_out, int* status, cudaStream_t s, int Hk) {
  if (B * H * n == 0) return cudaSuccess;
  if (Hk <= 0) Hk = H;
  if (H % Hk) return cudaErrorInvalidValue;
  if (d == 64) return launch_tc<64>(q, ldq, k_cache, vt, vt_ld, B, H, cap, n, out, ld_out, status, s, Hk);
  if (d == 128) return launch_tc<128>(q, ldq, k_cache, vt, vt_ld, B, H, cap, n, out, ld_out, status, s, Hk);
  return cudaErrorInvalidValue;
}

}  // namespace bt
