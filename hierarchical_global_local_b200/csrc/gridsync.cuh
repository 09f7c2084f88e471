// gridsync.cuh -- bounded grid-wide barrier for persistent kernels whose CTAs
// are all resident at once (cooperative launch).
//
// Three words in global memory, zero before the first launch:
//   bar[0]  arrival counter: barrier k of a launch completes when it reaches
//           k * gridDim.x (release by a red.release add, acquire by polling)
//   bar[1]  exit counter: the last CTA out of the kernel resets bar[0] and
//           bar[1] for the next launch (grid_exit)
//   bar[2]  abort word: set by a CTA whose wait ran out; every other CTA sees
//           it in its poll loop and stops waiting
// Every wait is bounded by `limit` SM clock cycles; a wait that runs out sets
// ST_WAIT_TIMEOUT in the status word and the abort word, and the barrier
// returns false. Nothing here can hang the GPU.
#pragma once

#include "common.cuh"

namespace bt {

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Barrier among the `nthreads` threads of named barrier `id` in every CTA
// (thread 0 of the CTA must be one of them). `target` = (barriers passed so
// far + 1) * gridDim.x. `arrive` = false withholds this CTA's arrival (only
// the self-test uses it). Returns false once the launch has been aborted,
// here or in another CTA.
__device__ __forceinline__ bool grid_barrier(unsigned* bar, unsigned target, long long limit, int* status,
                                             volatile int* s_abort, int id, int nthreads,
                                             bool arrive = true) {
  // data written before the barrier may be read through the async proxy
  // (TMA) after it
  asm volatile("fence.proxy.async.global;" ::: "memory");
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
  if (threadIdx.x == 0 && !*s_abort) {
    // release: this CTA's writes (ordered before by the CTA barrier above)
    // are visible to any CTA that acquires the count
    if (arrive) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&bar[0]) : "memory");
    const long long t0 = clock64();
    int n = 0;
    while (ld_acquire_gpu(&bar[0]) < target) {
      if ((++n & 63) == 0) {
        if (ld_acquire_gpu(&bar[2]) != 0u) { *s_abort = 1; break; }
        if (clock64() - t0 > limit) {
          atomicExch(&bar[2], 1u);
          set_status(status, ST_WAIT_TIMEOUT);
          *s_abort = 1;
          break;
        }
      }
    }
  }
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
  return !*s_abort;
}

// Called once by thread 0 of every CTA after its last barrier wait (and
// after a CTA barrier that orders the CTA's other writes before it): the last
// CTA out resets the arrival and exit counters for the next launch (the abort
// word stays set until the host clears it) and gets true; every CTA's writes
// before its exit are then visible to it.
__device__ __forceinline__ bool grid_exit(unsigned* bar) {
  __threadfence();
  if (atomicAdd(&bar[1], 1u) == gridDim.x - 1) {
    bar[0] = 0u;
    bar[1] = 0u;
    __threadfence();
    return true;
  }
  return false;
}

}  // namespace bt
