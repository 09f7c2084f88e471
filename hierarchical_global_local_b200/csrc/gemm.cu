// gemm.cu -- dense projections of the Block Transformer: dispatcher, the
// shared epilogues and the SIMT (FFMA) path.
//
// out = X . W^T with W row-major [N, K] (torch Linear layout), fp32
// accumulation, fused epilogues:
//   EPI_QKV1   q|k|v (+bias) to the qkv buffer and GELU(fc1 + bias) to the
//              MLP half of the second GEMM's input (Pythia's parallel
//              residual: both branches read the same residual row);
//   EPI_RESID  residual += acc + (b_o + b_2)   ([W_o | W_2] as one K = 5D GEMM);
//   EPI_F32 / EPI_ACT  plain stores (prefix projection, LM head logits).
// The SIMT path serves fp32 workloads (FFMA, no TF32) and any shape the
// tensor-core path does not take.
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace bt {

// 64x64 output tile, K step 16, 256 threads, 4x4 outputs per thread.
template <typename T>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(const T* __restrict__ X, int ldx, const T* __restrict__ W, int ldw, int M,
                 int N, int K, int n_base, Epi e) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sX[16][64 + 4];
  __shared__ float sW[16][64 + 4];
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int idx = threadIdx.x; idx < 64 * 16; idx += 256) {
      const int r = idx >> 4, c = idx & 15;
      const int gm = m0 + r, gn = n0 + r, gk = k0 + c;
      sX[c][r] = (gm < M && gk < K) ? to_f(X[(size_t)gm * ldx + gk]) : 0.f;
      sW[c][r] = (gn < N && gk < K) ? to_f(W[(size_t)gn * ldw + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sX[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sW[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < M && n < N) epi_apply<T>(e, m, n_base + n, acc[i][j]);
    }
}

static int g_gemm_path = 0;
void gemm_set_path(int path) { g_gemm_path = path; }

// tensor-core path (gemm_tc.cu)
cudaError_t launch_gemm_tc(int dt, const void* X, int ldx, const void* W, int ldw, int M, int N,
                           int K, int xk_split, int xk_off, const Epi& e,
                           const GemmScratch& scr, int* status, cudaStream_t s);

cudaError_t launch_gemm(int dt, const void* X, int ldx, const void* W, int ldw, int M, int N,
                        int K, int xk_split, int xk_off, const Epi& e, const GemmScratch& scr,
                        int* status, cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (e.kind == EPI_QKV1_ROPE && (g_gemm_path == 1 || !gemm_rope_fusable(dt, M, N, K, xk_split, xk_off, e.D / e.H, e.rot)))
    return cudaErrorNotSupported;  // the caller runs EPI_QKV1 + the rotary kernel instead
  if (e.kind == EPI_LOGITS_ARGMAX && (g_gemm_path == 1 || !gemm_argmax_fusable(dt, M, N, K)))
    return cudaErrorNotSupported;  // the caller runs EPI_F32 + the argmax kernel instead
  const bool tc_ok = gemm_tc_supported(dt, M, N, K, xk_split, xk_off) != 0;
  if (g_gemm_path != 1 && tc_ok)
    return launch_gemm_tc(dt, X, ldx, W, ldw, M, N, K, xk_split, xk_off, e, scr, status, s);
  if (g_gemm_path == 2) return cudaErrorNotSupported;
  // columns [0, xk_split) read X as given; columns [xk_split, N) read X
  // shifted by xk_off: two launches, each with its own column range.
  const size_t es = dt_size(dt);
  const int n1 = xk_split < N ? xk_split : N;
  for (int part = 0; part < 2; ++part) {
    const int nb = part == 0 ? 0 : n1;
    const int nn = part == 0 ? n1 : N - n1;
    if (nn <= 0) continue;
    const uint8_t* Xp = (const uint8_t*)X + (part ? (size_t)xk_off * es : 0);
    const uint8_t* Wp = (const uint8_t*)W + (size_t)nb * ldw * es;
    dim3 grid((nn + 63) / 64, (M + 63) / 64);
    if (dt == DT_BF16) {
      BT_LAUNCH(gemm_simt_kernel<bf16>, dim3(grid), dim3(256), 0, s, (const bf16*)Xp, ldx, (const bf16*)Wp, ldw, M,
                                                  nn, K, nb, e);
    }
    else {
      BT_LAUNCH(gemm_simt_kernel<float>, dim3(grid), dim3(256), 0, s, (const float*)Xp, ldx, (const float*)Wp, ldw,
                                                   M, nn, K, nb, e);
    }
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace bt
