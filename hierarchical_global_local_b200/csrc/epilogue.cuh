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
  const int d = D / e.H;
  const int Dk = (e.Hk > 0 ? e.Hk : e.H) * d;
  if (n >= D + 2 * Dk) {
    reinterpret_cast<T*>(e.out1)[(size_t)m * e.ld1 + D + (n - D - 2 * Dk)] = from_f<T>(gelu_erf(v));
    return;
  }
  const int part = n < D ? 0 : (n < D + Dk ? 1 : 2);
  const int c = part == 0 ? n : (part == 1 ? n - D : n - D - Dk);
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
    cache[(((size_t)b * (Dk / d) + hh) * e.cap + pos) * d + dim] = from_f<T>(out);
  }
}

// Weights-as-A orientation (the thread's output feature n is fixed, n < N):
// the epilogue of rows m0 .. m0 + cnt - 1 (cnt <= CH) with values v[j];
// partner[j] is the value of feature n ^ (rot/2) of the same row (rotary
// epilogue only). Every load the epilogue needs (bias, positions, rotary
// table, residual) is issued before the first store: a load placed after a
// store that the compiler cannot prove independent of it costs one memory
// round trip per row, which made the per-element form latency-bound.
template <typename T, int CH>
__device__ __forceinline__ void epi_cols(const Epi& e, int m0, int cnt, int n, int M, const float* v,
                                         const float* partner) {
  const int lim = (M - m0 < cnt) ? M - m0 : cnt;  // rows of the chunk inside [0, M)
  switch (e.kind) {
    case EPI_QKV1_ROPE: {
      const float bn = e.bias[n];
      const int D = e.D;
      const int d = D / e.H;
      const int Hk = e.Hk > 0 ? e.Hk : e.H, Dk = Hk * d;
      if (n >= D + 2 * Dk) {
        T* o = reinterpret_cast<T*>(e.out1) + D + (n - D - 2 * Dk);
#pragma unroll
        for (int j = 0; j < CH; ++j)
          if (j < lim) o[(size_t)(m0 + j) * e.ld1] = from_f<T>(gelu_erf(v[j] + bn));
        return;
      }
      // q (H heads) | k (Hk heads) | v (Hk heads)
      const int part = n < D ? 0 : (n < D + Dk ? 1 : 2);
      const int c = part == 0 ? n : (part == 1 ? n - D : n - D - Dk);
      const int hh = c / d, dim = c - hh * d;
      const int half = e.rot >> 1;
      const bool rot = part < 2 && dim < e.rot;
      const float bp = rot ? e.bias[n ^ half] : 0.f;
      const int rps = e.pos.rows_per_seq;
      int pos[CH], seq[CH];
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const int m = (j < lim) ? m0 + j : m0;  // rows past the end: any in-range row
        seq[j] = m / rps;
        pos[j] = pos_base(e.pos, seq[j]) + (m - seq[j] * rps);
      }
      float2 cs[CH];
      if (rot) {
#pragma unroll
        for (int j = 0; j < CH; ++j) cs[j] = e.rope_tab[(size_t)pos[j] * half + (dim & (half - 1))];
      }
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        if (j >= lim) break;
        float out = v[j] + bn;
        if (rot) {
          const float pv = partner[j] + bp;
          out = (dim < half) ? out * cs[j].x - pv * cs[j].y : out * cs[j].x + pv * cs[j].y;
        }
        if (part == 0) {
          reinterpret_cast<T*>(e.out0)[(size_t)(m0 + j) * e.ld0 + c] = from_f<T>(out);
        } else {
          T* cache = reinterpret_cast<T*>(part == 1 ? e.kc : e.vc);
          cache[(((size_t)seq[j] * Hk + hh) * e.cap + pos[j]) * d + dim] = from_f<T>(out);
        }
      }
      return;
    }
    case EPI_QKV1: {
      const float bn = e.bias[n];
      if (n < e.split_n) {
        T* o = reinterpret_cast<T*>(e.out0) + n;
#pragma unroll
        for (int j = 0; j < CH; ++j)
          if (j < lim) o[(size_t)(m0 + j) * e.ld0] = from_f<T>(v[j] + bn);
      } else {
        T* o = reinterpret_cast<T*>(e.out1) + e.D + (n - e.split_n);
#pragma unroll
        for (int j = 0; j < CH; ++j)
          if (j < lim) o[(size_t)(m0 + j) * e.ld1] = from_f<T>(gelu_erf(v[j] + bn));
      }
      return;
    }
    case EPI_RESID: {
      const float bn = e.bias[n];
      float* o = reinterpret_cast<float*>(e.out0) + n;
      float r[CH];
#pragma unroll
      for (int j = 0; j < CH; ++j) r[j] = (j < lim) ? o[(size_t)(m0 + j) * e.ld0] : 0.f;
#pragma unroll
      for (int j = 0; j < CH; ++j)
        if (j < lim) o[(size_t)(m0 + j) * e.ld0] = r[j] + (v[j] + bn);
      return;
    }
    case EPI_F32: {
      const float bn = e.bias ? e.bias[n] : 0.f;
      float* o = reinterpret_cast<float*>(e.out0) + n;
#pragma unroll
      for (int j = 0; j < CH; ++j)
        if (j < lim) o[(size_t)(m0 + j) * e.ld0] = v[j] + bn;
      return;
    }
    default: {
      const float bn = e.bias ? e.bias[n] : 0.f;
      T* o = reinterpret_cast<T*>(e.out0) + n;
#pragma unroll
      for (int j = 0; j < CH; ++j)
        if (j < lim) o[(size_t)(m0 + j) * e.ld0] = from_f<T>(v[j] + bn);
      return;
    }
  }
}

}  // namespace bt
