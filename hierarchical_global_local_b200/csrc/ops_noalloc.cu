// ops_noalloc.cu -- block-decoder decode attention without caller-provided
// scratch (bt_op_decode_attention_noalloc in bt_ops.h).
//
// Who needs this: code that cannot allocate device memory when it wants to
// run the kernel. Examples are a caller recording into a CUDA graph or stream
// capture (cudaMalloc is not a capturable operation), a serving runtime whose
// device memory is owned by a fixed-size pool carved once at start-up, and a
// host library that is not allowed to reach the process's allocator at all.
// Such a caller can still pass its inputs and outputs; the split-K merge
// state the kernel needs lives in a fixed array compiled into this library.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/bt_ops.h"
#include "common.cuh"
#include "kernels.h"

using namespace bt;

namespace {

// Largest problem the fixed array serves: B*H <= 8192 (sequence, head) pairs
// and d_head <= 128. Size: 8192 merge counters + the split partials, ~4.3 MB.
constexpr int NOALLOC_MAX_PAIRS = 8192;
constexpr int NOALLOC_MAX_D = 128;
constexpr size_t NOALLOC_BYTES = attn_decode_scratch_bytes_for(NOALLOC_MAX_PAIRS, NOALLOC_MAX_D);
static_assert(NOALLOC_BYTES % 256 == 0 && NOALLOC_BYTES < (8u << 20),
              "the fixed array covers the largest problem within the limits and stays modest");

// Shared by every call on a device and kept between calls; every GPU that
// loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
void* g_addr[MAX_DEVICES] = {};

// Device address of the array on the current device. The host-side symbol
// is only a stand-in, so the address is looked up once per device, with that
// device current, and cached.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    note_cuda_error("cudaGetDevice", e);
    return BT_ECUDA;
  }
  if (dev < 0 || dev >= MAX_DEVICES) return BT_ENOTSUP;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      note_cuda_error("cudaGetSymbolAddress", e == cudaSuccess ? cudaErrorInvalidSymbol : e);
      return BT_ECUDA;
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return BT_OK;
}

}  // namespace

extern "C" {

int bt_op_decode_attention_noalloc(int dtype, const void* q, int ldq, const void* k,
                                   const void* v, int B, int H, int d, int cap, int n,
                                   void* out, int ld_out, void* stream) {
  if (dtype != BT_FP32 && dtype != BT_BF16) return BT_EINVAL;
  if (!q || !k || !v || !out || B <= 0 || H <= 0 || n < 1 || n > cap) return BT_EINVAL;
  if (d != 32 && d != 64 && d != 128) return BT_ENOTSUP;
  // sizes beyond the fixed array are refused, never served partially
  if ((long long)B * H > NOALLOC_MAX_PAIRS || d > NOALLOC_MAX_D) return BT_ECAPACITY;
  const size_t need = attn_decode_scratch_bytes(B, H, d, cap, dtype);
  if (need > NOALLOC_BYTES) return BT_ECAPACITY;
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != BT_OK) return rc;
  // the merge counters (the first B*H ints) must start at zero; whatever an
  // earlier call left in the rest of the array is overwritten before use
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(scratch, 0, (size_t)B * H * sizeof(int), s);
  if (e != cudaSuccess) {
    note_cuda_error("cudaMemsetAsync", e);
    return BT_ECUDA;
  }
  PosSpec kv{nullptr, POS_ZERO, n - 1, 1};
  e = launch_attn_decode(dtype, q, ldq, k, v, B, H, d, cap, kv, out, ld_out, scratch, nullptr, s);
  if (e != cudaSuccess) {
    note_cuda_error("kernel launch", e);
    return BT_ECUDA;
  }
  return BT_OK;
}

}  // extern "C"
