// gemm_tc.cu -- tensor-core (tcgen05) GEMM path. Placeholder until the
// kernel lands: reports no supported shapes, so the SIMT path runs.
#include "common.cuh"
#include "kernels.h"

namespace bt {

size_t gemm_scratch_bytes(int max_M, int max_N) { return 256; }
int gemm_counter_count(int max_N) { return 64; }
int gemm_tc_supported(int dt, int M, int N, int K, int xk_split, int xk_off) { return 0; }

cudaError_t launch_gemm_tc(int dt, const void* X, int ldx, const void* W, int ldw, int M, int N,
                           int K, int xk_split, int xk_off, const Epi& e,
                           const GemmScratch& scr, int* status, cudaStream_t s) {
  return cudaErrorNotSupported;
}

}  // namespace bt
