// ConvSubsampling 8x ("Streaming Sortformer Diarizer", Pipeline / pre_encode
// and torch.export Fixes 3-5): conv3x3 s2 (1 -> 256) + ReLU, then twice
// [depthwise 3x3 s2 + pointwise 256 -> 256 + ReLU]; the pointwise convs and
// the final 4096 -> 512 Linear run as GEMMs (gemm.cu).  Layout is
// channels-last per window: [window][time][freq][256], so the pointwise convs
// are plain row-major GEMMs and the flattened (freq, channel) rows feed the
// Linear directly (its weight columns are permuted at load to match).
// Time rows outside each stage's valid length read as zero (MaskedConvSequential).
#include "common.cuh"
#include "layers.h"

namespace sf {

// out[i][t1][f1][c] = relu(b[c] + sum_{dt,df} w[c][dt][df] * in(2 t1 + dt - 1, 2 f1 + df - 1))
// with in(t, f) = feats[buf_i][f][start_i + t] for 0 <= t < W_i, 0 <= f < 128, else 0.
template <typename T>
__global__ void __launch_bounds__(256) conv1_kernel(const float* __restrict__ feats, int64_t t_buf, PreArgs args,
                                                     const float* __restrict__ w, const float* __restrict__ bias,
                                                     T* __restrict__ out, int T1max) {
  SF_PDL_ENTRY();
  constexpr int R = 4;                 // output rows per CTA
  __shared__ float patch[2 * R + 1][130];
  const int i = blockIdx.y;
  const int t1_0 = blockIdx.x * R;
  const int buf = args.buf[i];
  const int64_t start = args.start[i];
  const int64_t W = args.frames[i];
  const float* src = feats + (int64_t)buf * 128 * t_buf;
  for (int e = threadIdx.x; e < (2 * R + 1) * 130; e += 256) {
    const int r = e / 130, fc = e % 130;
    const int64_t t = 2 * t1_0 - 1 + r;
    const int f = fc - 1;
    float v = 0.f;
    if (t >= 0 && t < W && f >= 0 && f < 128) v = src[(int64_t)f * t_buf + start + t];
    patch[r][fc] = v;
  }
  __syncthreads();
  const int c = threadIdx.x;
  float wr[9];
#pragma unroll
  for (int j = 0; j < 9; ++j) wr[j] = w[c * 9 + j];
  const float b = bias[c];
  for (int r = 0; r < R; ++r) {
    const int t1 = t1_0 + r;
    if (t1 >= T1max) break;
    T* o = out + (((int64_t)i * T1max + t1) * 64) * 256 + c;
    for (int f1 = 0; f1 < 64; ++f1) {
      float acc = b;
#pragma unroll
      for (int dt = 0; dt < 3; ++dt)
#pragma unroll
        for (int df = 0; df < 3; ++df) acc = fmaf(wr[dt * 3 + df], patch[2 * r + dt][2 * f1 + df], acc);
      o[f1 * 256] = from_f<T>(fmaxf(acc, 0.f));
    }
  }
}

// Depthwise 3x3 stride 2 over [window][Tin][Fin][256]: rows >= l_in of the
// window are zero.  No activation (the pointwise GEMM adds bias + ReLU).
template <typename T>
__global__ void __launch_bounds__(256) dwconv3x3s2_kernel(const T* __restrict__ in, int Tin_max, int Fin,
                                                          T* __restrict__ out, int Tout_max, int Fout, PreArgs args,
                                                          int stage, const float* __restrict__ w,
                                                          const float* __restrict__ bias) {
  SF_PDL_ENTRY();
  const int t = blockIdx.x, i = blockIdx.y, c = threadIdx.x;
  int64_t l = args.frames[i];
  for (int s = 0; s < stage; ++s) l = 1 + (l - 1) / 2;     // valid rows of the input stage
  float wr[9];
#pragma unroll
  for (int j = 0; j < 9; ++j) wr[j] = w[c * 9 + j];
  const float b = bias[c];
  const T* base = in + (int64_t)i * Tin_max * Fin * 256 + c;
  T* o = out + (((int64_t)i * Tout_max + t) * Fout) * 256 + c;
  for (int f = 0; f < Fout; ++f) {
    float acc = b;
#pragma unroll
    for (int dt = 0; dt < 3; ++dt) {
      const int ti = 2 * t + dt - 1;
      if (ti < 0 || ti >= l) continue;
#pragma unroll
      for (int df = 0; df < 3; ++df) {
        const int fi = 2 * f + df - 1;
        if (fi < 0 || fi >= Fin) continue;
        acc = fmaf(wr[dt * 3 + df], to_f<T>(base[((int64_t)ti * Fin + fi) * 256]), acc);
      }
    }
    o[f * 256] = from_f<T>(acc);
  }
}

// conv1 and the first depthwise stage in one pass (subsampling path 1): the
// 3x3 s2 conv's outputs (rounded to the activation type, as path 0 stores
// them) are computed on the fly from a mel patch in shared memory and fed
// straight into the depthwise accumulators, so the [T1][64][256] stage-1
// tensor never goes to memory.  One CTA = R2 output rows of one window, one
// thread per channel.  A stage-1 value at (row ti, column fi) feeds output
// column f = fi / 2 (fi even, tap 1) or f = (fi - 1) / 2 and (fi + 1) / 2
// (fi odd, taps 2 and 0), and output row r through tap ti - 2 (t0 + r) + 1;
// rows are visited in increasing ti and columns in increasing fi, so every
// output sums its taps in the order of dwconv3x3s2_kernel and the result is
// the same to the bit.
template <typename T, int R2>
__global__ void __launch_bounds__(256) conv1_dw_kernel(const float* __restrict__ feats, int64_t t_buf, PreArgs args,
                                                        const float* __restrict__ w1, const float* __restrict__ b1,
                                                        const float* __restrict__ w2, const float* __restrict__ b2,
                                                        T* __restrict__ out, int T2max) {
  SF_PDL_ENTRY();
  constexpr int NJ = 2 * R2 + 1;   // stage-1 rows touched by R2 output rows
  constexpr int NM = 4 * R2 + 3;   // mel rows those need
  __shared__ float patch[NM][130];
  const int i = blockIdx.y;
  const int t0 = blockIdx.x * R2;
  const int buf = args.buf[i];
  const int64_t start = args.start[i];
  const int64_t W = args.frames[i];
  const int64_t l1 = 1 + (W - 1) / 2;   // valid stage-1 rows
  const float* src = feats + (int64_t)buf * 128 * t_buf;
  for (int e = threadIdx.x; e < NM * 130; e += 256) {
    const int pr = e / 130, fc = e % 130;
    const int64_t t = 4 * (int64_t)t0 - 3 + pr;
    const int f = fc - 1;
    float v = 0.f;
    if (t >= 0 && t < W && f >= 0 && f < 128) v = src[(int64_t)f * t_buf + start + t];
    patch[pr][fc] = v;
  }
  __syncthreads();
  const int c = threadIdx.x;
  float w1r[9], w2r[9];
#pragma unroll
  for (int j = 0; j < 9; ++j) {
    w1r[j] = w1[c * 9 + j];
    w2r[j] = w2[c * 9 + j];
  }
  const float b1c = b1[c], b2c = b2[c];
  float acc[R2][32];
#pragma unroll
  for (int r = 0; r < R2; ++r)
#pragma unroll
    for (int f = 0; f < 32; ++f) acc[r][f] = b2c;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int64_t ti = 2 * (int64_t)t0 - 1 + j;
    if (ti < 0 || ti >= l1) continue;   // same for the whole CTA
#pragma unroll
    for (int fp = 0; fp < 32; ++fp) {
      // stage-1 values at columns 2 fp and 2 fp + 1 of row ti; mel row
      // 2 ti - 1 + dt is patch row 2 j + dt, mel column 2 fi - 1 + df is
      // patch column 2 fi + df
      float ve = b1c, vo = b1c;
#pragma unroll
      for (int dt = 0; dt < 3; ++dt)
#pragma unroll
        for (int df = 0; df < 3; ++df) ve = fmaf(w1r[dt * 3 + df], patch[2 * j + dt][4 * fp + df], ve);
#pragma unroll
      for (int dt = 0; dt < 3; ++dt)
#pragma unroll
        for (int df = 0; df < 3; ++df) vo = fmaf(w1r[dt * 3 + df], patch[2 * j + dt][4 * fp + 2 + df], vo);
      ve = to_f<T>(from_f<T>(fmaxf(ve, 0.f)));
      vo = to_f<T>(from_f<T>(fmaxf(vo, 0.f)));
#pragma unroll
      for (int r = 0; r < R2; ++r) {
        const int dt = j - 2 * r;
        if (dt < 0 || dt > 2) continue;
        acc[r][fp] = fmaf(w2r[dt * 3 + 1], ve, acc[r][fp]);
        acc[r][fp] = fmaf(w2r[dt * 3 + 2], vo, acc[r][fp]);
        if (fp + 1 < 32) acc[r][fp + 1] = fmaf(w2r[dt * 3 + 0], vo, acc[r][fp + 1]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R2; ++r) {
    const int t = t0 + r;
    if (t >= T2max) break;
    T* o = out + (((int64_t)i * T2max + t) * 32) * 256 + c;
#pragma unroll
    for (int f = 0; f < 32; ++f) o[f * 256] = from_f<T>(acc[r][f]);
  }
}

template <typename T>
cudaError_t launch_conv1_dw(const float* feats, int64_t t_buf, const PreArgs& a, int n_win, const float* w1,
                            const float* b1, const float* w2, const float* b2, T* out, int T2max, cudaStream_t st) {
  constexpr int R2 = 2;
  CK_LAUNCH(launch_k(conv1_dw_kernel<T, R2>, dim3(dim3((T2max + R2 - 1) / R2, n_win)), dim3(256), 0, st, feats, t_buf,
                     a, w1, b1, w2, b2, out, T2max));
  return cudaGetLastError();
}

template cudaError_t launch_conv1_dw<float>(const float*, int64_t, const PreArgs&, int, const float*, const float*,
                                            const float*, const float*, float*, int, cudaStream_t);
template cudaError_t launch_conv1_dw<bf16>(const float*, int64_t, const PreArgs&, int, const float*, const float*,
                                           const float*, const float*, bf16*, int, cudaStream_t);

template <typename T>
cudaError_t launch_conv1(const float* feats, int64_t t_buf, const PreArgs& a, int n_win, const float* w,
                         const float* b, T* out, int T1max, cudaStream_t st) {
  CK_LAUNCH(launch_k(conv1_kernel<T>, dim3(dim3((T1max + 3) / 4, n_win)), dim3(256), 0, st, feats, t_buf, a, w, b, out, T1max));
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dwconv3x3s2(const T* in, int Tin_max, int Fin, T* out, int Tout_max, int Fout, const PreArgs& a,
                               int n_win, int stage, const float* w, const float* b, cudaStream_t st) {
  CK_LAUNCH(launch_k(dwconv3x3s2_kernel<T>, dim3(dim3(Tout_max, n_win)), dim3(256), 0, st, in, Tin_max, Fin, out, Tout_max, Fout, a, stage, w, b));
  return cudaGetLastError();
}

template cudaError_t launch_conv1<float>(const float*, int64_t, const PreArgs&, int, const float*, const float*, float*, int, cudaStream_t);
template cudaError_t launch_conv1<bf16>(const float*, int64_t, const PreArgs&, int, const float*, const float*, bf16*, int, cudaStream_t);
template cudaError_t launch_dwconv3x3s2<float>(const float*, int, int, float*, int, int, const PreArgs&, int, int, const float*, const float*, cudaStream_t);
template cudaError_t launch_dwconv3x3s2<bf16>(const bf16*, int, int, bf16*, int, int, const PreArgs&, int, int, const float*, const float*, cudaStream_t);

}  // namespace sf
