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

// Logistic sigmoid for an output of type T.  A bf16 output keeps 8
// significant bits, so the hardware exp2 approximation and an approximate
// reciprocal (relative error ~1e-7 each) are far inside its rounding; an
// f32 output takes expf and an IEEE division.  Large negative x gives
// exp(-x) = inf and a sigmoid of exactly 0.
template <typename T>
__device__ __forceinline__ float sigm(float x) {
  if (sizeof(T) == 2) return __fdividef(1.f, 1.f + __expf(-x));
  return 1.f / (1.f + expf(-x));
}

// Pointer to element (r, c) of an f32 output with the row remap applied.
__device__ __forceinline__ float* epi_f32_ptr(const Epi& e, int r, int c) {
  const int64_t orow = e.rpg ? (int64_t)(r / e.rpg) * e.gstride + (r % e.rpg) : (int64_t)r;
  return reinterpret_cast<float*>(e.out) + orow * e.ldo + c;
}

// Four consecutive columns c .. c + 3 of row r (c % 4 == 0, c + 3 < N),
// bias already added; kind fixed at compile time.
template <int EK, typename T>
__device__ __forceinline__ void epi_store4(const Epi& e, int r, int c, float4 v) {
  const int64_t orow = e.rpg ? (int64_t)(r / e.rpg) * e.gstride + (r % e.rpg) : (int64_t)r;
  if (EK == EPI_BIAS_RELU) {
    v.x = fmaxf(v.x, 0.f); v.y = fmaxf(v.y, 0.f); v.z = fmaxf(v.z, 0.f); v.w = fmaxf(v.w, 0.f);
  }
  if (EK == EPI_BIAS_SWISH) {
    v.x *= sigm<T>(v.x); v.y *= sigm<T>(v.y); v.z *= sigm<T>(v.z); v.w *= sigm<T>(v.w);
  }
  if (EK == EPI_BIAS || EK == EPI_BIAS_RELU || EK == EPI_BIAS_SWISH) {
    T* o = reinterpret_cast<T*>(e.out) + orow * e.ldo + c;
    if (sizeof(T) == 2) {
      __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&a);
      pk.y = *reinterpret_cast<uint32_t*>(&b);
      *reinterpret_cast<uint2*>(o) = pk;
    } else {
      *reinterpret_cast<float4*>(o) = v;
    }
  } else if (EK == EPI_BIAS_GLU) {
    T* o = reinterpret_cast<T*>(e.out) + orow * e.ldo + (c >> 1);
    const float g0 = v.x * sigm<T>(v.y), g1 = v.z * sigm<T>(v.w);
    if (sizeof(T) == 2) {
      __nv_bfloat162 a = __floats2bfloat162_rn(g0, g1);
      *reinterpret_cast<__nv_bfloat162*>(o) = a;
    } else {
      *reinterpret_cast<float2*>(o) = make_float2(g0, g1);
    }
  } else if (EK == EPI_RESID) {
    float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(e.out) + orow * e.ldo + c);
    float4 x = *o;
    x.x += e.alpha * v.x; x.y += e.alpha * v.y; x.z += e.alpha * v.z; x.w += e.alpha * v.w;
    *o = x;
  } else {   // EPI_F32, EPI_F32_AND_T
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(e.out) + orow * e.ldo + c) = v;
    if (EK == EPI_F32_AND_T) {
      T* o2 = reinterpret_cast<T*>(e.out2) + orow * e.ldo2 + c;
      o2[0] = from_f<T>(v.x); o2[1] = from_f<T>(v.y); o2[2] = from_f<T>(v.z); o2[3] = from_f<T>(v.w);
    }
  }
}

}  // namespace sf
