// GEMM epilogue shared by the GEMM kernels: applies the fused operation of
// an Epi to one pair of adjacent output columns (c, c + 1) of row r.
#pragma once
#include "common.cuh"
#include "layers.h"

namespace sf {

template <typename T>
__device__ __forceinline__ void epi_store2(const Epi& e, int r, int c, float v0, float v1) {
  const int64_t orow = e.rpg ? (int64_t)(r / e.rpg) * e.gstride + (r % e.rpg) : (int64_t)r;
  if (e.bias) {
    v0 += e.bias[c];
    v1 += e.bias[c + 1];
  }
  switch (e.kind) {
    case EPI_BIAS:
    case EPI_BIAS_RELU:
    case EPI_BIAS_SWISH: {
      if (e.kind == EPI_BIAS_RELU) { v0 = fmaxf(v0, 0.f); v1 = fmaxf(v1, 0.f); }
      if (e.kind == EPI_BIAS_SWISH) { v0 = v0 / (1.f + expf(-v0)); v1 = v1 / (1.f + expf(-v1)); }
      T* o = reinterpret_cast<T*>(e.out) + orow * e.ldo + c;
      o[0] = from_f<T>(v0);
      o[1] = from_f<T>(v1);
      break;
    }
    case EPI_BIAS_GLU: {
      T* o = reinterpret_cast<T*>(e.out) + orow * e.ldo + (c >> 1);
      o[0] = from_f<T>(v0 / (1.f + expf(-v1)));
      break;
    }
    case EPI_RESID: {
      float* o = reinterpret_cast<float*>(e.out) + orow * e.ldo + c;
      o[0] += e.alpha * v0;
      o[1] += e.alpha * v1;
      break;
    }
    case EPI_F32:
    case EPI_F32_AND_T: {
      float* o = reinterpret_cast<float*>(e.out) + orow * e.ldo + c;
      o[0] = v0;
      o[1] = v1;
      if (e.kind == EPI_F32_AND_T) {
        T* o2 = reinterpret_cast<T*>(e.out2) + orow * e.ldo2 + c;
        o2[0] = from_f<T>(v0);
        o2[1] = from_f<T>(v1);
      }
      break;
    }
    default:
      break;
  }
}

}  // namespace sf
