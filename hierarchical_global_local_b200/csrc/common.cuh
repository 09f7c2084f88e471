// common.cuh -- shared device helpers for the Block Transformer kernels
// (sm_100a): element conversions, status bits, step-state positions,
// mbarrier / bulk-copy wrappers with bounded waits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bt {

typedef __nv_bfloat16 bf16;

// ---- status word bits (device-side failures, read by bt_sync) -------------
enum : int {
  ST_BAD_TOKEN = 1,     // a token id outside [0, vocab) was clamped to 0
  ST_WAIT_TIMEOUT = 2,  // a bounded mbarrier wait ran out
  ST_BAD_ARGS = 4,      // a kernel saw arguments outside its contract
};

__device__ __forceinline__ void set_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// ---- conversions ----------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// 16-byte vector of T
template <typename T> struct Vec16 { static constexpr int N = 16 / sizeof(T); };

__device__ __forceinline__ void unpack16(const uint4& u, float* f, const bf16*) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void unpack16(const uint4& u, float* f, const float*) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}

// exact GELU, x * Phi(x)
__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752440f));
}

// ---- step state -------------------------------------------------------------
// dstate[0] = t (position of the token fed in the current decode call, or
// the prompt length after prefill), dstate[1] = t % L_B, dstate[2] = t / L_B.
enum PosMode : int { POS_ZERO = 0, POS_BLOCK = 1, POS_LOCAL = 2 };

struct PosSpec {
  const int* dstate;  // may be null for POS_ZERO
  int mode;           // PosMode
  int add;            // constant added to the state-derived base
  int rows_per_seq;   // consecutive rows of one sequence
  // POS_BLOCK only (may be null): per-sequence lag behind the longest
  // sequence of a ragged batch; sequence b's block position is
  // dstate[2] - row_lag[b]
  const int* row_lag = nullptr;
};

// position base shared by every sequence (POS_BLOCK: the longest one's)
__device__ __forceinline__ int pos_base(const PosSpec& p) {
  int b = 0;
  if (p.mode == POS_BLOCK) b = p.dstate[2];
  else if (p.mode == POS_LOCAL) b = p.dstate[1];
  return b + p.add;
}

// position base of sequence `seq`
__device__ __forceinline__ int pos_base(const PosSpec& p, int seq) {
  const int b = pos_base(p);
  return (p.mode == POS_BLOCK && p.row_lag) ? b - p.row_lag[seq] : b;
}

// ---- mbarrier + bulk copy (PTX) -------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after ~max_cycles SM clocks, sets ST_WAIT_TIMEOUT
// and returns false. No wait in this library is unbounded.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* status,
                                                  long long max_cycles = 4000000000LL) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > max_cycles) {
      set_status(status, ST_WAIT_TIMEOUT);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> shared (this CTA), completion on an mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16. No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- programmatic dependent launch ------------------------------------------
// Every kernel of the library calls pdl_trigger() first (its dependents may be
// scheduled as soon as all of its CTAs are running) and pdl_wait() before it
// reads or writes anything an earlier kernel in the stream touches (returns
// once the preceding grid has completed and its writes are visible). Without
// the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace bt
