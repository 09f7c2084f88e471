// selftest.cu -- self-test of the bounded grid barrier (gridsync.cuh) that the
// persistent decode kernel synchronises its phases with: failure detection
// checked on the device without a fault. One CTA can withhold its arrival at
// the first barrier; every wait then runs out after the given bound, the
// kernel records ST_WAIT_TIMEOUT and returns, and the context stays usable.
#include <cuda_runtime.h>

#include "../../include/bt_ops.h"
#include "common.cuh"
#include "gridsync.cuh"
#include "kernels.h"

using namespace bt;

namespace {

constexpr int SELFTEST_THREADS = 128;

__global__ void __launch_bounds__(SELFTEST_THREADS)
barrier_selftest_kernel(unsigned* bar, int rounds, int withhold, long long limit, int* status, int* passed) {
  __shared__ volatile int s_abort;
  if (threadIdx.x == 0) s_abort = 0;
  __syncthreads();
  int done = 0;
  for (int r = 0; r < rounds; ++r) {
    const bool arrive = !(r == 0 && (int)blockIdx.x == withhold);
    if (!grid_barrier(bar, (unsigned)(r + 1) * gridDim.x, limit, status, &s_abort, 1, SELFTEST_THREADS, arrive))
      break;
    ++done;
  }
  if (threadIdx.x == 0) {
    atomicAdd(passed, done);
    grid_exit(bar);
  }
}

}  // namespace

extern "C" {

int bt_op_grid_barrier_selftest(int rounds, int withhold_cta, long long wait_cycles, unsigned* words_dev,
                                int* status_dev, int* passed_dev, void* stream) {
  if (rounds < 1 || wait_cycles < 1 || !words_dev || !status_dev || !passed_dev) return BT_EINVAL;
  int dev = 0, coop = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
  if (e != cudaSuccess) {
    note_cuda_error("device query", e);
    return BT_ECUDA;
  }
  if (!coop) return BT_ENOTSUP;
  const int G = device_sm_count();  // one CTA per SM: all resident under a cooperative launch
  if (withhold_cta >= G) return BT_EINVAL;
  void* args[] = {&words_dev, &rounds, &withhold_cta, &wait_cycles, &status_dev, &passed_dev};
  e = cudaLaunchCooperativeKernel((const void*)barrier_selftest_kernel, dim3(G), dim3(SELFTEST_THREADS), args, 0,
                                  (cudaStream_t)stream);
  note_launch();
  if (e != cudaSuccess) {
    note_cuda_error("cudaLaunchCooperativeKernel", e);
    return BT_ECUDA;
  }
  return BT_OK;
}

}  // extern "C"
