// ops.cu -- single-kernel C-ABI entry points (bt_ops.h).
#include <cuda_runtime.h>

#include "../../include/bt_ops.h"
#include "common.cuh"
#include "kernels.h"

using namespace bt;

static int status_of(cudaError_t e) {
  if (e == cudaSuccess) return BT_OK;
  note_cuda_error("kernel launch", e);
  return BT_ECUDA;
}

extern "C" {

size_t bt_op_decode_attention_scratch_bytes(int dtype, int B, int H, int d, int cap) {
  if (B <= 0 || H <= 0 || cap <= 0 || (d != 32 && d != 64 && d != 128)) return 0;
  return attn_decode_scratch_bytes(B, H, d, cap, dtype);
}

int bt_op_decode_attention(int dtype, const void* q, int ldq, const void* k, const void* v, int B,
                           int H, int d, int cap, int n, void* out, int ld_out, void* scratch,
                           size_t scratch_bytes, void* stream) {
  if (dtype != BT_FP32 && dtype != BT_BF16) return BT_EINVAL;
  if (!q || !k || !v || !out || B <= 0 || H <= 0 || n < 1 || n > cap) return BT_EINVAL;
  if (d != 32 && d != 64 && d != 128) return BT_ENOTSUP;
  if (!scratch || ((uintptr_t)scratch & 255) ||
      scratch_bytes < attn_decode_scratch_bytes(B, H, d, cap, dtype))
    return BT_EWORKSPACE;
  PosSpec kv{nullptr, POS_ZERO, n - 1, 1};
  return status_of(launch_attn_decode(dtype, q, ldq, k, v, B, H, d, cap, kv, out, ld_out, scratch,
                                      nullptr, (cudaStream_t)stream));
}

int bt_op_prefill_attention(int dtype, const void* q, int ldq, const void* k, const void* v, int B,
                            int H, int d, int cap, int n, void* out, int ld_out, void* stream) {
  if (dtype != BT_FP32 && dtype != BT_BF16) return BT_EINVAL;
  if (!q || !k || !v || !out || B <= 0 || H <= 0 || n < 1 || n > cap) return BT_EINVAL;
  if (d != 32 && d != 64 && d != 128) return BT_ENOTSUP;
  return status_of(launch_attn_prefill(dtype, q, ldq, k, v, B, H, d, cap, n, out, ld_out,
                                       (cudaStream_t)stream));
}

int bt_op_prefill_attention_tc(const void* q, int ldq, const void* k, const void* vt, int vt_ld,
                               int B, int H, int d, int cap, int n, void* out, int ld_out,
                               void* stream) {
  if (!q || !k || !vt || !out || B <= 0 || H <= 0 || n < 1 || n > cap || vt_ld < n) return BT_EINVAL;
  if (!attn_prefill_tc_supported(BT_BF16, d, ldq, vt_ld)) return BT_ENOTSUP;
  return status_of(launch_attn_prefill_tc(q, ldq, k, vt, vt_ld, B, H, d, cap, n, out, ld_out,
                                          nullptr, (cudaStream_t)stream));
}

size_t bt_op_linear_scratch_bytes(int M, int N) {
  if (M <= 0 || N <= 0) return 0;
  return gemm_scratch_bytes(M, N) + 256 + (size_t)gemm_counter_count(N) * 4;
}

int bt_op_linear(int dtype, const void* x, int ldx, const void* w, const float* bias, float* out,
                 int ld_out, int M, int N, int K, int path, void* scratch, size_t scratch_bytes,
                 void* stream) {
  if (dtype != BT_FP32 && dtype != BT_BF16) return BT_EINVAL;
  if (!x || !w || !out || M <= 0 || N <= 0 || K <= 0 || ldx < K || ld_out < N) return BT_EINVAL;
  if (path < 0 || path > 2) return BT_EINVAL;
  if (!scratch || ((uintptr_t)scratch & 255) || scratch_bytes < bt_op_linear_scratch_bytes(M, N))
    return BT_EWORKSPACE;
  if (path == 2 && !gemm_tc_supported(dtype, M, N, K, 1 << 30, 0)) return BT_ENOTSUP;
  GemmScratch gs;
  gs.part = (float*)scratch;
  gs.part_bytes = gemm_scratch_bytes(M, N);
  gs.counters = (int*)((uint8_t*)scratch + ((gs.part_bytes + 255) & ~(size_t)255));
  gs.n_counters = gemm_counter_count(N);
  Epi e{EPI_F32, out, ld_out, nullptr, 0, bias, 0, 0};
  gemm_set_path(path);
  cudaError_t err = launch_gemm(dtype, x, ldx, w, K, M, N, K, 1 << 30, 0, e, gs, nullptr,
                                (cudaStream_t)stream);
  gemm_set_path(0);
  return status_of(err);
}

int bt_op_layernorm(int dtype, const float* h, int M, int D, const float* g, const float* b,
                    float eps, void* out, void* stream) {
  if (dtype != BT_FP32 && dtype != BT_BF16) return BT_EINVAL;
  if (!h || !g || !b || !out || M <= 0 || D <= 0 || (D % 4)) return BT_EINVAL;
  return status_of(launch_ln_rows(dtype, h, M, 1, 0, D, g, b, eps, out, (cudaStream_t)stream));
}

int bt_op_embed_prompt(int dtype, const int32_t* tokens, int B, int T, int L, const void* table,
                       int V, int D, float* h, int32_t* status, void* stream) {
  if (dtype != BT_FP32 && dtype != BT_BF16) return BT_EINVAL;
  if (!tokens || !table || !h || B <= 0 || L <= 0 || T < L || (T % L) || D % L) return BT_EINVAL;
  return status_of(launch_embed_prompt(dtype, tokens, B, T, L, table, V, D, h, (int*)status,
                                       (cudaStream_t)stream));
}

}  // extern "C"
