// epilogue.cuh -- fused GEMM epilogues shared by the SIMT and tensor-core
// paths (see EpiKind in kernels.h). Applied per output element (m, n).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace bt {

template <typename T>
__device__ __forceinline__ void epi_apply(const Epi& e, int m, int n, float acc) {
  switch (e.kind) {
    case EPI_QKV1: {
      const float v = acc + e.bias[n];
      if (n < e.split_n)
        reinterpret_cast<T*>(e.out0)[(size_t)m * e.ld0 + n] = from_f<T>(v);
      else
        reinterpret_cast<T*>(e.out1)[(size_t)m * e.ld1 + e.D + (n - e.split_n)] =
            from_f<T>(gelu_erf(v));
      break;
    }
    case EPI_RESID: {
      float* o = reinterpret_cast<float*>(e.out0) + (size_t)m * e.ld0 + n;
      *o = *o + (acc + e.bias[n]);
      break;
    }
    case EPI_F32:
      reinterpret_cast<float*>(e.out0)[(size_t)m * e.ld0 + n] = acc + (e.bias ? e.bias[n] : 0.f);
      break;
    default:
      reinterpret_cast<T*>(e.out0)[(size_t)m * e.ld0 + n] =
          from_f<T>(acc + (e.bias ? e.bias[n] : 0.f));
      break;
  }
}

}  // namespace bt
