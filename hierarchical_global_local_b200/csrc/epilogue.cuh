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

// EPI_QKV1_ROPE for one element; `partner` is the value of feature n ^ (rot/2)
// (its rotate-half pair) of the same token, fetched by the caller.
template <typename T>
__device__ __forceinline__ void epi_apply_rope(const Epi& e, int m, int n, float acc,
                                               float partner) {
  const float v = acc + e.bias[n];
  const int D = e.D;
  if (n >= 3 * D) {
    reinterpret_cast<T*>(e.out1)[(size_t)m * e.ld1 + D + (n - 3 * D)] = from_f<T>(gelu_erf(v));
    return;
  }
  const int part = n / D, c = n - part * D;
  const int d = D / e.H;
  const int hh = c / d, dim = c - hh * d;
  const int b = m / e.pos.rows_per_seq;
  const int pos = pos_base(e.pos, b) + (m - b * e.pos.rows_per_seq);
  float out = v;
  if (part < 2 && dim < e.rot) {
    const int half = e.rot >> 1;
    const float pv = partner + e.bias[n ^ half];
    const float2 cs = e.rope_tab[(size_t)pos * half + (dim & (half - 1))];
    out = (dim < half) ? v * cs.x - pv * cs.y : v * cs.x + pv * cs.y;
  }
  if (part == 0) {
    reinterpret_cast<T*>(e.out0)[(size_t)m * e.ld0 + c] = from_f<T>(out);
  } else {
    T* cache = reinterpret_cast<T*>(part == 1 ? e.kc : e.vc);
    cache[(((size_t)b * e.H + hh) * e.cap + pos) * d + dim] = from_f<T>(out);
  }
}

}  // namespace bt
