// Row-wise and elementwise kernels: LayerNorm, the conformer conv module's
// depthwise conv (BatchNorm folded) + swish, the head's output layer,
// precision conversion and packed-row extraction.
#include "common.cuh"
#include "layers.h"

namespace sf {

// VEC consecutive floats at p (VEC = 2 or 4, aligned).
template <int VEC>
__device__ __forceinline__ void ld_vec(const float* p, float* v) {
  if (VEC == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    v[0] = t.x; v[1 % VEC] = t.y; v[2 % VEC] = t.z; v[3 % VEC] = t.w;
  } else {
    const float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x; v[1 % VEC] = t.y;
  }
}
template <int VEC>
__device__ __forceinline__ void st_vec(float* p, const float* v) {
  if (VEC == 4) *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1 % VEC], v[2 % VEC], v[3 % VEC]);
  else *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1 % VEC]);
}
template <int VEC>
__device__ __forceinline__ void st_vec(bf16* p, const float* v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1 % VEC]);
  if (VEC == 4) {
    const __nv_bfloat162 c = __floats2bfloat162_rn(v[2 % VEC], v[3 % VEC]);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&a);
    pk.y = *reinterpret_cast<const uint32_t*>(&c);
    *reinterpret_cast<uint2*>(p) = pk;
  } else {
    *reinterpret_cast<__nv_bfloat162*>(p) = a;
  }
}

// One warp per row; lane j holds VEC-wide vectors j, j + 32, ... (coalesced).
// With g2/b2 set, a second LayerNorm follows on the first one's output (the
// conformer's layer-final LN and the next layer's first LN): x gets LN1(x),
// h gets LN2(LN1(x)).
template <typename T, int D, int VEC>
__global__ void __launch_bounds__(256) layernorm_kernel(float* __restrict__ x, const float* __restrict__ g,
                                                        const float* __restrict__ b, int M, bool write_x,
                                                        T* __restrict__ h, const float* __restrict__ g2,
                                                        const float* __restrict__ b2) {
  SF_PDL_ENTRY();
  constexpr int NV = D / (32 * VEC);
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  float* xr = x + (int64_t)row * D;
  T* hr = h ? h + (int64_t)row * D : nullptr;
  float v[NV][VEC];
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    ld_vec<VEC>(xr + (lane + 32 * j) * VEC, v[j]);
#pragma unroll
    for (int k = 0; k < VEC; ++k) s += v[j][k];
  }
  const float mean = warp_sum(s) * (1.0f / D);
  float q = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j)
#pragma unroll
    for (int k = 0; k < VEC; ++k) { const float d = v[j][k] - mean; q = fmaf(d, d, q); }
  const float inv = 1.0f / sqrtf(warp_sum(q) * (1.0f / D) + 1e-5f);
  float s2 = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (lane + 32 * j) * VEC;
    float gg[VEC], bb[VEC];
    ld_vec<VEC>(g + c, gg);
    ld_vec<VEC>(b + c, bb);
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      v[j][k] = (v[j][k] - mean) * inv * gg[k] + bb[k];
      s2 += v[j][k];
    }
    if (write_x || g2) st_vec<VEC>(xr + c, v[j]);
    if (!g2 && hr) st_vec<VEC>(hr + c, v[j]);
  }
  if (!g2) return;
  // x <- LN1(x) (stored above), then LN2 over it into h
  const float mean2 = warp_sum(s2) * (1.0f / D);
  float q2 = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j)
#pragma unroll
    for (int k = 0; k < VEC; ++k) { const float dd = v[j][k] - mean2; q2 = fmaf(dd, dd, q2); }
  const float inv2 = 1.0f / sqrtf(warp_sum(q2) * (1.0f / D) + 1e-5f);
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (lane + 32 * j) * VEC;
    float gg[VEC], bb[VEC], y[VEC];
    ld_vec<VEC>(g2 + c, gg);
    ld_vec<VEC>(b2 + c, bb);
#pragma unroll
    for (int k = 0; k < VEC; ++k) y[k] = (v[j][k] - mean2) * inv2 * gg[k] + bb[k];
    st_vec<VEC>(hr + c, y);
  }
}

template <typename T>
cudaError_t launch_layernorm(float* x, const float* g, const float* b, int M, int D, bool write_x, T* h,
                             cudaStream_t st, const float* g2, const float* b2) {
  if (M <= 0) return cudaSuccess;
  if (g2 && (!h || !b2)) return cudaErrorInvalidValue;
  const int grid = (M + 7) / 8;
  if (D == 512)
    CK_LAUNCH(launch_k(layernorm_kernel<T, 512, 4>, dim3(grid), dim3(256), 0, st, x, g, b, M, write_x, h, g2, b2));
  else if (D == 192)
    CK_LAUNCH(launch_k(layernorm_kernel<T, 192, 2>, dim3(grid), dim3(256), 0, st, x, g, b, M, write_x, h, g2, b2));
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

template <typename T> struct Vec2;
template <> struct Vec2<float> {
  typedef float2 type;
  static __device__ __forceinline__ float2 load(const float* p) { return *reinterpret_cast<const float2*>(p); }
  static __device__ __forceinline__ void store(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
  static __device__ __forceinline__ float lo(float2 v) { return v.x; }
  static __device__ __forceinline__ float hi(float2 v) { return v.y; }
};
template <> struct Vec2<bf16> {
  typedef __nv_bfloat162 type;
  static __device__ __forceinline__ __nv_bfloat162 load(const bf16* p) { return *reinterpret_cast<const __nv_bfloat162*>(p); }
  static __device__ __forceinline__ void store(bf16* p, float a, float b) { *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b); }
  static __device__ __forceinline__ float lo(__nv_bfloat162 v) { return __low2float(v); }
  static __device__ __forceinline__ float hi(__nv_bfloat162 v) { return __high2float(v); }
};

// Each thread: two channels x DW_ROWS consecutive rows; the DW_ROWS + K - 1
// input rows they need are loaded once into registers (32-row blocks keep
// the halo re-read at K - 1 rows per 32 and the weight loads amortised;
// 8-row blocks give short inputs more CTAs).  The two channels are one
// packed f32x2 FMA per tap (each lane an ordinary fused multiply-add).
// Taps outside the output row's sequence read as zero.  Swish: exact expf and
// division for f32 outputs; for bf16 outputs sigmoid(a) = (1 + tanh(a/2)) / 2
// with the hardware tanh approximation (absolute error about 2^-11, below
// bf16 rounding; one special-function operation where exp and reciprocal
// take two).
constexpr int DW_KMAX = 9;
template <typename T>
__device__ __forceinline__ float dw_swish(float a) {
  if (sizeof(T) == 2) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * a));
    return a * fmaf(0.5f, t, 0.5f);
  }
  return a / (1.f + expf(-a));
}
template <typename T, int DW_ROWS>
__global__ void __launch_bounds__(128) dwconv1d_kernel(const T* __restrict__ in, T* __restrict__ out,
                                                       const float* __restrict__ w, const float* __restrict__ bias,
                                                       int M, int D, int K, const SeqTable* __restrict__ seq) {
  SF_PDL_ENTRY();
  const int c = 2 * (blockIdx.y * 128 + threadIdx.x);
  if (c >= D) return;
  const int r0 = blockIdx.x * DW_ROWS;
  const int pad = (K - 1) / 2;
  float2 wc[DW_KMAX];
#pragma unroll
  for (int j = 0; j < DW_KMAX; ++j)   // channels c, c + 1: 2K consecutive floats at c * K
    wc[j] = j < K ? make_float2(w[(int64_t)c * K + j], w[(int64_t)c * K + K + j]) : make_float2(0.f, 0.f);
  const float2 bc = make_float2(bias[c], bias[c + 1]);
  float2 xc[DW_ROWS + DW_KMAX - 1];
#pragma unroll
  for (int i = 0; i < DW_ROWS + DW_KMAX - 1; ++i) {
    const int ri = r0 - pad + i;
    xc[i] = make_float2(0.f, 0.f);
    if (ri >= 0 && ri < M && i < DW_ROWS + K - 1) {
      const auto v = Vec2<T>::load(in + (int64_t)ri * D + c);
      xc[i] = make_float2(Vec2<T>::lo(v), Vec2<T>::hi(v));
    }
  }
  int s = seq_of_row(seq, r0 < M ? r0 : M - 1);
  int sb = seq->off[s], se = seq->off[s + 1];
#pragma unroll
  for (int k = 0; k < DW_ROWS; ++k) {
    const int r = r0 + k;
    if (r >= M) break;
    if (r >= se) {   // next sequence (rows are packed sequence after sequence)
      while (r >= seq->off[s + 1]) ++s;
      sb = seq->off[s];
      se = seq->off[s + 1];
    }
    float2 a = bc;
    if (r - pad >= sb && r + pad < se) {   // interior row: every tap inside the sequence
#pragma unroll
      for (int j = 0; j < DW_KMAX; ++j)
        if (j < K) a = __ffma2_rn(wc[j], xc[k + j], a);
    } else {
#pragma unroll
      for (int j = 0; j < DW_KMAX; ++j) {
        const int ri = r + j - pad;
        if (j < K && ri >= sb && ri < se) a = __ffma2_rn(wc[j], xc[k + j], a);
      }
    }
    Vec2<T>::store(out + (int64_t)r * D + c, dw_swish<T>(a.x), dw_swish<T>(a.y));
  }
}

template <typename T>
cudaError_t launch_dwconv1d(const T* in, T* out, const float* w, const float* b, int M, int D, int K,
                            const SeqTable* seq, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  if (K > DW_KMAX || (D % 2)) return cudaErrorInvalidValue;
  // 32-row blocks when there are enough of them to fill the GPU (streaming
  // batches); 8-row blocks for short inputs (one clip), where parallelism wins
  if (M >= 32 * 2 * 148) {
    dim3 grid((M + 31) / 32, (D / 2 + 127) / 128);
    CK_LAUNCH(launch_k(dwconv1d_kernel<T, 32>, dim3(grid), dim3(128), 0, st, in, out, w, b, M, D, K, seq));
  } else {
    dim3 grid((M + 7) / 8, (D / 2 + 127) / 128);
    CK_LAUNCH(launch_k(dwconv1d_kernel<T, 8>, dim3(grid), dim3(128), 0, st, in, out, w, b, M, D, K, seq));
  }
  return cudaGetLastError();
}

// One warp per row: 4 dot products of length E, sigmoid.
template <typename T>
__global__ void __launch_bounds__(256) head_out_kernel(const T* __restrict__ h, const float* __restrict__ w,
                                                       const float* __restrict__ b, float* __restrict__ probs,
                                                       int M, int E) {
  SF_PDL_ENTRY();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  for (int c = lane; c < E; c += 32) {
    const float x = to_f<T>(h[(int64_t)row * E + c]);
#pragma unroll
    for (int s = 0; s < 4; ++s) a[s] = fmaf(x, w[s * E + c], a[s]);
  }
#pragma unroll
  for (int s = 0; s < 4; ++s) a[s] = warp_sum(a[s]);
  if (lane == 0) {
    float4 o;
    o.x = 1.f / (1.f + expf(-(a[0] + b[0])));
    o.y = 1.f / (1.f + expf(-(a[1] + b[1])));
    o.z = 1.f / (1.f + expf(-(a[2] + b[2])));
    o.w = 1.f / (1.f + expf(-(a[3] + b[3])));
    reinterpret_cast<float4*>(probs)[row] = o;
  }
}

template <typename T>
cudaError_t launch_head_out(const T* h, const float* w, const float* b, float* probs, int M, int E,
                            cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  CK_LAUNCH(launch_k(head_out_kernel<T>, dim3((M + 7) / 8), dim3(256), 0, st, h, w, b, probs, M, E));
  return cudaGetLastError();
}

template <typename T>
__global__ void to_f32_kernel(const T* __restrict__ in, float* __restrict__ out, int64_t n) {
  SF_PDL_ENTRY();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = to_f<T>(in[i]);
}

template <typename T>
cudaError_t launch_to_f32(const T* in, float* out, int64_t n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int64_t want = (n + 255) / 256;
  const int64_t blocks = want < 148 * 16 ? want : 148 * 16;
  CK_LAUNCH(launch_k(to_f32_kernel<T>, dim3((int)blocks), dim3(256), 0, st, in, out, n));
  return cudaGetLastError();
}

__global__ void extract_rows_kernel(const float* __restrict__ packed, const SeqTable* __restrict__ seq,
                                    const int* __restrict__ first, const int* __restrict__ count,
                                    const int* __restrict__ dst, float* __restrict__ out, int t_max) {
  SF_PDL_ENTRY();
  const int s = blockIdx.y;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= t_max) return;
  const int len = seq->off[s + 1] - seq->off[s];
  const int f = first ? first[s] : 0;
  const int n = count ? count[s] : len;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (t < n && f + t < len) v = reinterpret_cast<const float4*>(packed)[seq->off[s] + f + t];
  reinterpret_cast<float4*>(out)[(int64_t)(dst ? dst[s] : s) * t_max + t] = v;
}

cudaError_t launch_extract_rows(const float* packed, const SeqTable* seq, const int* d_first, const int* d_count,
                                const int* d_dst, int n_seq, float* out, int t_max, cudaStream_t st) {
  if (n_seq <= 0 || t_max <= 0) return cudaSuccess;
  CK_LAUNCH(launch_k(extract_rows_kernel, dim3(dim3((t_max + 127) / 128, n_seq)), dim3(128), 0, st, packed, seq, d_first, d_count, d_dst, out,
                                                                         t_max));
  return cudaGetLastError();
}

template cudaError_t launch_layernorm<float>(float*, const float*, const float*, int, int, bool, float*, cudaStream_t,
                                             const float*, const float*);
template cudaError_t launch_layernorm<bf16>(float*, const float*, const float*, int, int, bool, bf16*, cudaStream_t,
                                            const float*, const float*);
template cudaError_t launch_dwconv1d<float>(const float*, float*, const float*, const float*, int, int, int, const SeqTable*, cudaStream_t);
template cudaError_t launch_dwconv1d<bf16>(const bf16*, bf16*, const float*, const float*, int, int, int, const SeqTable*, cudaStream_t);
template cudaError_t launch_head_out<float>(const float*, const float*, const float*, float*, int, int, cudaStream_t);
template cudaError_t launch_head_out<bf16>(const bf16*, const float*, const float*, float*, int, int, cudaStream_t);
template cudaError_t launch_to_f32<float>(const float*, float*, int64_t, cudaStream_t);
template cudaError_t launch_to_f32<bf16>(const bf16*, float*, int64_t, cudaStream_t);

}  // namespace sf
