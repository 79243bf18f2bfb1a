// Log-mel front-end ("Streaming Sortformer Diarizer", Pipeline: 128 mel bins,
// 25 ms window, 10 ms stride; Exported Methods / preprocessor).
//
// Kernel 1 (mel_frames): one CTA = 32 consecutive frames of one clip.  The
// audio span of those frames is staged once in shared memory with the
// preemphasis applied (coalesced loads); each warp then takes one frame at a
// time: windowed samples packed as 256 complex points, radix-2 FFT in shared
// memory, split into the 257 real-FFT bins, power, sparse Slaney filterbank,
// log.  The 32 x 128 log-mel tile is written channels-first with coalesced
// stores, and per-bin (count, shift, shifted sum, M2) of the tile's valid
// frames go to a partial-statistics buffer.
// Kernel 2 (mel_normalize): one CTA per (clip, bin) merges the partials
// (Chan's pairwise update, double) and normalises the row in place; frames
// >= L are zeroed.
#include "common.cuh"
#include "frontend.h"

namespace sf {

constexpr int MEL_FB = 32;                       // frames per CTA
constexpr int MEL_SPAN = (MEL_FB - 1) * 160 + 512;

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

__global__ void __launch_bounds__(256) mel_frames_kernel(const float* __restrict__ audio, int64_t n_max,
                                                          const MelArgs args, const MelTables* __restrict__ tab,
                                                          float* __restrict__ mel, float* __restrict__ part,
                                                          int T_cols, int n_blk) {
  SF_PDL_ENTRY();
  extern __shared__ float4 mel_smem[];
  float* y = reinterpret_cast<float*>(mel_smem);               // [MEL_SPAN]
  float2* tw256 = reinterpret_cast<float2*>(y + MEL_SPAN);      // [128]
  float2* tw512 = tw256 + 128;                                  // [258]
  float* win = reinterpret_cast<float*>(tw512 + 258);           // [512]
  float2* zall = reinterpret_cast<float2*>(win + 512);          // [8][256]
  float (*tile)[MEL_FB + 1] = reinterpret_cast<float (*)[MEL_FB + 1]>(zall + 8 * 256);  // [128][33]

  const int b = blockIdx.y;
  const int blk = blockIdx.x;
  const int t0 = blk * MEL_FB;                    // first column of this tile
  const int64_t len = args.len[b];
  const bool win_mode = args.f0 != nullptr;
  const int64_t fb = win_mode ? args.f0[b] : 0;   // absolute frame of column 0
  const int64_t a0 = win_mode ? args.a0[b] : 0;   // absolute sample of buffer column 0
  const int L = win_mode ? args.nf[b] : (int)(len / 160);
  const float* x = audio + (int64_t)(win_mode ? args.row[b] : b) * n_max - a0;   // indexed by absolute sample
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < 128; i += 256) tw256[i] = tab->tw256[i];
  for (int i = tid; i < 257; i += 256) tw512[i] = tab->tw512[i];   // slot 257 is padding
  for (int i = tid; i < 512; i += 256) win[i] = tab->win[i];
  // span sample i <-> absolute sample n = 160*(fb + t0) - 256 + i
  const int64_t n0 = (int64_t)160 * (fb + t0) - 256;
  for (int i = tid; i < MEL_SPAN; i += 256) {
    int64_t n = n0 + i;
    float v = 0.f;
    if (n >= 0 && n < len) {
      float cur = __ldg(x + n);
      float prev = (n >= 1) ? __ldg(x + n - 1) : 0.f;
      v = (n >= 1) ? fmaf(-0.97f, prev, cur) : cur;
    }
    y[i] = v;
  }
  __syncthreads();

  for (int f = warp; f < MEL_FB; f += 8) {
    const int t = t0 + f;
    float2* z = zall + warp * 256;
    float* pw = reinterpret_cast<float*>(z);   // power spectrum reuses the FFT buffer
    if (t < T_cols) {
      const float* fr = y + f * 160;
      // packed input z[m] = w*y[2m] + i w*y[2m+1], stored at bit-reversed index
      for (int m = lane; m < 256; m += 32) {
        float re = fr[2 * m] * win[2 * m];
        float im = fr[2 * m + 1] * win[2 * m + 1];
        z[__brev(m) >> 24] = make_float2(re, im);
      }
      __syncwarp();
      // radix-2 decimation-in-time, 8 stages
#pragma unroll 1
      for (int s = 0; s < 8; ++s) {
        const int half = 1 << s;
        for (int bf = lane; bf < 128; bf += 32) {
          int grp = bf >> s, pos = bf & (half - 1);
          int i0 = (grp << (s + 1)) + pos, i1 = i0 + half;
          float2 w = tw256[pos << (7 - s)];
          float2 a = z[i0], c = cmul(z[i1], w);
          z[i0] = make_float2(a.x + c.x, a.y + c.y);
          z[i1] = make_float2(a.x - c.x, a.y - c.y);
        }
        __syncwarp();
      }
      // split: A = (Z[k] + conj Z[-k]) / 2, B = (Z[k] - conj Z[-k]) / 2i, X = A + W512^k B
      float pk[9];
#pragma unroll
      for (int j = 0; j < 9; ++j) {
        const int k = lane + 32 * j;
        pk[j] = 0.f;
        if (k <= 256) {
          float2 zk = z[k & 255], zn = z[(256 - k) & 255];
          float2 A = make_float2(0.5f * (zk.x + zn.x), 0.5f * (zk.y - zn.y));
          float2 Bv = make_float2(0.5f * (zk.y + zn.y), -0.5f * (zk.x - zn.x));
          float2 X = cmul(tw512[k], Bv);
          X.x += A.x;
          X.y += A.y;
          pk[j] = X.x * X.x + X.y * X.y;
        }
      }
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 9; ++j) {
        const int k = lane + 32 * j;
        if (k <= 256) pw[k] = pk[j];
      }
      __syncwarp();
      for (int m = lane; m < 128; m += 32) {
        const int k0 = tab->mel_k0[m], nk = tab->mel_nk[m];
        float acc = 0.f;
        for (int j = 0; j < nk; ++j) acc = fmaf(__ldg(tab->mel_w + m * MEL_MAX_NK + j), pw[k0 + j], acc);
        tile[m][f] = logf(acc + 5.9604644775390625e-08f);   // 2^-24
      }
    } else {
      for (int m = lane; m < 128; m += 32) tile[m][f] = 0.f;
    }
    __syncwarp();
  }
  __syncthreads();

  // coalesced channels-first store: for each bin, 32 consecutive frames
  for (int i = tid; i < 128 * MEL_FB; i += 256) {
    int m = i / MEL_FB, f = i % MEL_FB;
    int t = t0 + f;
    if (t < T_cols) mel[((int64_t)(win_mode ? args.row[b] : b) * 128 + m) * T_cols + t] = tile[m][f];
  }
  // per-bin statistics of the valid frames of this tile, shifted by the
  // tile's first value so that a constant bin gives an exact mean
  if (tid < 128) {
    const int nv = max(0, min(MEL_FB, L - t0));
    float c = 0.f, sh = 0.f, m2 = 0.f;
    if (nv > 0) {
      c = tile[tid][0];
      for (int f = 0; f < nv; ++f) sh += tile[tid][f] - c;
      const float mean = c + sh / nv;
      for (int f = 0; f < nv; ++f) {
        float d = tile[tid][f] - mean;
        m2 = fmaf(d, d, m2);
      }
    }
    float* p = part + (((int64_t)b * n_blk + blk) * 128 + tid) * 4;
    p[0] = (float)nv;
    p[1] = c;
    p[2] = sh;
    p[3] = m2;
  }
}

__global__ void __launch_bounds__(256) mel_normalize_kernel(float* __restrict__ mel, const float* __restrict__ part,
                                                            const MelArgs args, int T_cols, int n_blk) {
  SF_PDL_ENTRY();
  const int m = blockIdx.x, b = blockIdx.y;
  const int L = args.nf ? args.nf[b] : (int)(args.len[b] / 160);
  __shared__ float s_mu, s_inv;
  __shared__ double sn[256], smean[256], sm2[256];
  // Chan's pairwise merge of the per-tile (count, mean, M2): each thread
  // merges a strided subset, then a fixed shared-memory tree (deterministic).
  double n = 0, mean = 0, m2 = 0;
  for (int k = threadIdx.x; k < n_blk; k += blockDim.x) {
    const float* p = part + (((int64_t)b * n_blk + k) * 128 + m) * 4;
    const double nb = p[0];
    if (nb <= 0) continue;
    const double mb = (double)p[1] + (double)p[2] / nb, m2b = p[3];
    const double nt = n + nb, d = mb - mean;
    mean += d * nb / nt;
    m2 += m2b + d * d * n * nb / nt;
    n = nt;
  }
  sn[threadIdx.x] = n;
  smean[threadIdx.x] = mean;
  sm2[threadIdx.x] = m2;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      const double na = sn[threadIdx.x], nb = sn[threadIdx.x + w];
      if (nb > 0) {
        const double nt = na + nb, d = smean[threadIdx.x + w] - smean[threadIdx.x];
        smean[threadIdx.x] += d * nb / nt;
        sm2[threadIdx.x] += sm2[threadIdx.x + w] + d * d * na * nb / nt;
        sn[threadIdx.x] = nt;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double sd = (L > 1) ? sqrt(sm2[0] / (double)(L - 1)) : 0.0;
    s_mu = (float)smean[0];
    s_inv = (float)(1.0 / (sd + 1e-5));
  }
  __syncthreads();
  const float mu = s_mu, inv = s_inv;
  float* row = mel + ((int64_t)(args.row ? args.row[b] : b) * 128 + m) * T_cols;
  for (int t = threadIdx.x; t < T_cols; t += blockDim.x) row[t] = (t < L) ? (row[t] - mu) * inv : 0.f;
}

constexpr size_t MEL_SMEM =
    (size_t)MEL_SPAN * 4 + 128 * 8 + 258 * 8 + 512 * 4 + 8 * 256 * 8 + 128 * (MEL_FB + 1) * 4;

cudaError_t frontend_init_attributes() {
  return cudaFuncSetAttribute(mel_frames_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)MEL_SMEM);
}

cudaError_t launch_mel(const float* audio, int B, int64_t n_max, const MelArgs& args, const MelTables* tab,
                       float* mel, float* part, cudaStream_t st) {
  const int T_cols = (int)(1 + n_max / 160);
  const int n_blk = (T_cols + MEL_FB - 1) / MEL_FB;
  const size_t smem = MEL_SMEM;
  static bool attr_set = false;   // first use outside an engine (sf_mel_noalloc)
  if (!attr_set) {
    cudaError_t e = frontend_init_attributes();
    if (e != cudaSuccess) return e;
  }
  attr_set = true;
  CK_LAUNCH(launch_k(mel_frames_kernel, dim3(dim3(n_blk, B)), dim3(256), smem, st, audio, n_max, args, tab, mel, part, T_cols, n_blk));
  CK_LAUNCH(launch_k(mel_normalize_kernel, dim3(dim3(128, B)), dim3(256), 0, st, mel, part, args, T_cols, n_blk));
  return cudaGetLastError();
}

cudaError_t launch_mel_windows(const float* audio, int B, int64_t n_buf, const MelArgs& args, const MelTables* tab,
                               float* mel, float* part, int T_cols, cudaStream_t st) {
  const int n_blk = (T_cols + MEL_FB - 1) / MEL_FB;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = frontend_init_attributes();
    if (e != cudaSuccess) return e;
  }
  attr_set = true;
  CK_LAUNCH(launch_k(mel_frames_kernel, dim3(dim3(n_blk, B)), dim3(256), MEL_SMEM, st, audio, n_buf, args, tab, mel, part,
                     T_cols, n_blk));
  CK_LAUNCH(launch_k(mel_normalize_kernel, dim3(dim3(128, B)), dim3(256), 0, st, mel, part, args, T_cols, n_blk));
  return cudaGetLastError();
}

size_t mel_part_floats(int B, int64_t n_max) {
  const int T_cols = (int)(1 + n_max / 160);
  const int n_blk = (T_cols + MEL_FB - 1) / MEL_FB;
  return (size_t)B * n_blk * 128 * 4;
}

}  // namespace sf

// ---------------------------------------------------------------- host tables
#include <math.h>

namespace sf {

static double hz_to_mel_slaney(double f) {
  const double f_sp = 200.0 / 3.0, logstep = log(6.4) / 27.0;
  return f < 1000.0 ? f / f_sp : 1000.0 / f_sp + log(f / 1000.0) / logstep;
}
static double mel_to_hz_slaney(double m) {
  const double f_sp = 200.0 / 3.0, logstep = log(6.4) / 27.0, m0 = 1000.0 / f_sp;
  return m < m0 ? f_sp * m : 1000.0 * exp(logstep * (m - m0));
}

void build_mel_tables(MelTables* t) {
  const double PI = 3.14159265358979323846;
  for (int k = 0; k < 128; ++k) t->tw256[k] = make_float2((float)cos(2 * PI * k / 256), (float)-sin(2 * PI * k / 256));
  for (int k = 0; k < 257; ++k) t->tw512[k] = make_float2((float)cos(2 * PI * k / 512), (float)-sin(2 * PI * k / 512));
  for (int n = 0; n < 512; ++n) t->win[n] = 0.f;
  for (int n = 0; n < 400; ++n) t->win[56 + n] = (float)(0.5 - 0.5 * cos(2 * PI * n / 399.0));
  double pts[130];
  const double m_lo = hz_to_mel_slaney(0.0), m_hi = hz_to_mel_slaney(8000.0);
  for (int i = 0; i < 130; ++i) pts[i] = mel_to_hz_slaney(m_lo + (m_hi - m_lo) * i / 129.0);
  for (int m = 0; m < 128; ++m) {
    int k0 = -1, nk = 0;
    for (int j = 0; j < MEL_MAX_NK; ++j) t->mel_w[m * MEL_MAX_NK + j] = 0.f;
    for (int k = 0; k <= 256; ++k) {
      const double fk = k * 16000.0 / 512.0;
      const double lo = (fk - pts[m]) / (pts[m + 1] - pts[m]);
      const double hi = (pts[m + 2] - fk) / (pts[m + 2] - pts[m + 1]);
      const double w = fmax(0.0, fmin(lo, hi)) * 2.0 / (pts[m + 2] - pts[m]);
      if (w > 0.0) {
        if (k0 < 0) k0 = k;
        const int j = k - k0;
        if (j < MEL_MAX_NK) t->mel_w[m * MEL_MAX_NK + j] = (float)w;
        nk = j + 1;
      }
    }
    t->mel_k0[m] = k0 < 0 ? 0 : k0;
    t->mel_nk[m] = nk > MEL_MAX_NK ? MEL_MAX_NK : nk;
  }
}

}  // namespace sf
