// device.cu -- per-device queries shared by the launchers.
#include <cuda_runtime.h>

#include "kernels.h"

namespace bt {

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return -1;
  return dev;
}

int device_sm_count() {
  static int cached[MAX_DEVICES] = {};
  const int dev = current_device();
  if (dev >= 0 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  cached[dev] = n;
  return n;
}

}  // namespace bt
