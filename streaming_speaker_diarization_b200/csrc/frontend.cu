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


// ------------------------------------------------ path 1: register FFT
// mel_frames_reg_kernel: the tiles, staging, output and statistics of
// mel_frames_kernel, with the per-frame transform kept in registers.  Lane l
// holds the packed points z[l + 32 r], r = 0..7 (z[m] = w[2m] y[2m] +
// i w[2m+1] y[2m+1]); 256 = 8 x 32 splits the DFT into an 8-point DFT inside
// each lane (index k1), the twiddle W256^(l k1), and for each k1 a 32-point
// DFT across the lanes (index k2), done as five radix-2 decimation-in-
// frequency stages over xor-shuffles.  Register p of lane l then holds
// Z[brev3(p) + 8 brev5(l)].  The real-FFT split needs Z[256 - k]: for k1 != 0
// it sits in lane l ^ 31, register brev3(8 - k1); for k1 = 0 in register 0 of
// lane brev5(-brev5(l) mod 32).  Power goes to a per-warp shared row padded
// as k + k / 32 (conflict-free stores), which the filterbank reads.
constexpr int MEL_PW = 272;   // padded power row per warp (bins 0..256)

__device__ __forceinline__ int brev3(int x) { return (int)(__brev((unsigned)x) >> 29); }
__device__ __forceinline__ int brev5(int x) { return (int)(__brev((unsigned)x) >> 27); }

// exp(-2 pi i k / 512) for 0 <= k < 512 from the table of k = 0..256
__device__ __forceinline__ float2 w512(const MelTables* __restrict__ tab, int k) {
  const float2 v = __ldg(&tab->tw512[k <= 256 ? k : 512 - k]);
  return k <= 256 ? v : make_float2(v.x, -v.y);
}

__device__ __forceinline__ void cmul_inplace(float& re, float& im, float2 w) {
  const float r = re * w.x - im * w.y;
  im = re * w.y + im * w.x;
  re = r;
}

__global__ void __launch_bounds__(256, 2) mel_frames_reg_kernel(const float* __restrict__ audio, int64_t n_max,
                                                                 const MelArgs args,
                                                                 const MelTables* __restrict__ tab,
                                                                 float* __restrict__ mel, float* __restrict__ part,
                                                                 int T_cols, int n_blk) {
  SF_PDL_ENTRY();
  extern __shared__ float4 mel_smem[];
  float* y = reinterpret_cast<float*>(mel_smem);                                  // [MEL_SPAN]
  float* pw_all = y + MEL_SPAN;                                                   // [8][MEL_PW]
  float (*tile)[MEL_FB + 1] = reinterpret_cast<float (*)[MEL_FB + 1]>(pw_all + 8 * MEL_PW);   // [128][33]
  float* fw = &tile[0][0] + 128 * (MEL_FB + 1);                                   // [128][MEL_MAX_NK] weights
  int* fk = reinterpret_cast<int*>(fw + 128 * MEL_MAX_NK);                        // [128] first bin | count << 16

  const int b = blockIdx.y;
  const int blk = blockIdx.x;
  const int t0 = blk * MEL_FB;
  const int64_t len = args.len[b];
  const bool win_mode = args.f0 != nullptr;
  const int64_t fb = win_mode ? args.f0[b] : 0;
  const int64_t a0 = win_mode ? args.a0[b] : 0;
  const int L = win_mode ? args.nf[b] : (int)(len / 160);
  const float* x = audio + (int64_t)(win_mode ? args.row[b] : b) * n_max - a0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // span sample i <-> absolute sample n = 160*(fb + t0) - 256 + i, preemphasised
  const int64_t n0 = (int64_t)160 * (fb + t0) - 256;
  for (int i = tid; i < MEL_SPAN; i += 256) {
    const int64_t n = n0 + i;
    float v = 0.f;
    if (n >= 0 && n < len) {
      const float cur = __ldg(x + n);
      const float prev = (n >= 1) ? __ldg(x + n - 1) : 0.f;
      v = (n >= 1) ? fmaf(-0.97f, prev, cur) : cur;
    }
    y[i] = v;
  }

  // the filterbank, once per CTA (every frame of the tile reads all of it)
  for (int i = tid; i < 128 * MEL_MAX_NK; i += 256) fw[i] = __ldg(tab->mel_w + i);
  for (int i = tid; i < 128; i += 256) fk[i] = __ldg(&tab->mel_k0[i]) | (__ldg(&tab->mel_nk[i]) << 16);

  // per-lane constants: window pairs, in-lane twiddles, stage twiddles, split twiddles
  float2 wv[8], tA[8], tS[4], t5[8];
  const int q = brev5(lane);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int m = lane + 32 * r;
    wv[r] = make_float2(__ldg(&tab->win[2 * m]), __ldg(&tab->win[2 * m + 1]));
    tA[r] = w512(tab, (2 * lane * brev3(r)) & 511);
    t5[r] = __ldg(&tab->tw512[brev3(r) + 8 * q]);
  }
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int h = 16 >> s;
    tS[s] = (lane & h) ? w512(tab, (lane & (h - 1)) * (256 / h)) : make_float2(1.f, 0.f);
  }
  const int src0 = brev5((32 - q) & 31);
  __syncthreads();

  float* pw = pw_all + warp * MEL_PW;
  const float c8 = 0.70710678118654752f;   // 1 / sqrt(2)
  for (int f = warp; f < MEL_FB; f += 8) {
    const int t = t0 + f;
    if (t < T_cols) {
      const float2* fr2 = reinterpret_cast<const float2*>(y + f * 160);
      float re[8], im[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float2 v = fr2[lane + 32 * r];
        re[r] = v.x * wv[r].x;
        im[r] = v.y * wv[r].y;
      }
      // 8-point DIF over r (span 4, 2, 1); outputs in bit-reversed register order
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float ur = re[r] + re[r + 4], ui = im[r] + im[r + 4];
        float dr = re[r] - re[r + 4], di = im[r] - im[r + 4];
        if (r == 1) { const float a = c8 * (dr + di); di = c8 * (di - dr); dr = a; }        // x W8^1
        if (r == 2) { const float a = di; di = -dr; dr = a; }                               // x W8^2 = -i
        if (r == 3) { const float a = c8 * (di - dr); di = -c8 * (dr + di); dr = a; }       // x W8^3
        re[r] = ur; im[r] = ui; re[r + 4] = dr; im[r + 4] = di;
      }
#pragma unroll
      for (int g = 0; g < 8; g += 4) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int i0 = g + r, i1 = g + r + 2;
          const float ur = re[i0] + re[i1], ui = im[i0] + im[i1];
          float dr = re[i0] - re[i1], di = im[i0] - im[i1];
          if (r == 1) { const float a = di; di = -dr; dr = a; }                             // x W4^1 = -i
          re[i0] = ur; im[i0] = ui; re[i1] = dr; im[i1] = di;
        }
      }
#pragma unroll
      for (int g = 0; g < 8; g += 2) {
        const float ur = re[g] + re[g + 1], ui = im[g] + im[g + 1];
        re[g + 1] = re[g] - re[g + 1];
        im[g + 1] = im[g] - im[g + 1];
        re[g] = ur;
        im[g] = ui;
      }
#pragma unroll
      for (int p = 1; p < 8; ++p) cmul_inplace(re[p], im[p], tA[p]);
      // 32-point DIF across the lanes: lanes with bit h clear keep a + b,
      // lanes with bit h set take (a - b) W_2h^(lane mod h)
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const int h = 16 >> s;
        const float sg = (lane & h) ? -1.f : 1.f;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float pr = __shfl_xor_sync(0xffffffffu, re[p], h);
          const float pi = __shfl_xor_sync(0xffffffffu, im[p], h);
          re[p] = fmaf(sg, re[p], pr);
          im[p] = fmaf(sg, im[p], pi);
          if (s < 4) cmul_inplace(re[p], im[p], tS[s]);
        }
      }
      // real-FFT split: X[k] = A + W512^k B, A = (Z[k] + conj Z[-k]) / 2, B = (Z[k] - conj Z[-k]) / 2i
      float nr[8], ni[8];
      nr[0] = __shfl_sync(0xffffffffu, re[0], src0);
      ni[0] = __shfl_sync(0xffffffffu, im[0], src0);
      constexpr int PP[8] = {0, 1, 3, 2, 7, 6, 5, 4};   // register of Z[256 - k] in lane ^ 31
#pragma unroll
      for (int p = 1; p < 8; ++p) {
        nr[p] = __shfl_xor_sync(0xffffffffu, re[PP[p]], 31);
        ni[p] = __shfl_xor_sync(0xffffffffu, im[PP[p]], 31);
      }
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const float ar = 0.5f * (re[p] + nr[p]), ai = 0.5f * (im[p] - ni[p]);
        const float br = 0.5f * (im[p] + ni[p]), bi = -0.5f * (re[p] - nr[p]);
        const float xr = ar + (t5[p].x * br - t5[p].y * bi);
        const float xi = ai + (t5[p].x * bi + t5[p].y * br);
        const int k = brev3(p) + 8 * q;
        pw[k + (k >> 5)] = xr * xr + xi * xi;
      }
      if (lane == 0) {
        const float d = re[0] - im[0];   // X[256] = Re Z[0] - Im Z[0]
        pw[256 + 8] = d * d;
      }
      __syncwarp();
      // filters lane, 63 - lane, 64 + lane, 127 - lane (narrow and wide paired)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = (i >> 1) * 64 + ((i & 1) ? 63 - lane : lane);
        const int kk = fk[m], k0 = kk & 0xffff, nk = kk >> 16;
        const float* wm = fw + m * MEL_MAX_NK;
        float acc = 0.f;
        for (int j = 0; j < nk; ++j) {
          const int k = k0 + j;
          acc = fmaf(wm[j], pw[k + (k >> 5)], acc);
        }
        // natural log by the hardware log2 (absolute error ~1e-6 here, far
        // inside the 1e-3 feature tolerance)
        tile[m][f] = __logf(acc + 5.9604644775390625e-08f);   // 2^-24
      }
      __syncwarp();
    } else {
      for (int m = lane; m < 128; m += 32) tile[m][f] = 0.f;
    }
  }
  __syncthreads();

  for (int i = tid; i < 128 * MEL_FB; i += 256) {
    const int m = i / MEL_FB, f = i % MEL_FB;
    const int t = t0 + f;
    if (t < T_cols) mel[((int64_t)(win_mode ? args.row[b] : b) * 128 + m) * T_cols + t] = tile[m][f];
  }
  if (tid < 128) {
    const int nv = max(0, min(MEL_FB, L - t0));
    float c = 0.f, sh = 0.f, m2 = 0.f;
    if (nv > 0) {
      c = tile[tid][0];
      for (int f = 0; f < nv; ++f) sh += tile[tid][f] - c;
      const float mean = c + sh / nv;
      for (int f = 0; f < nv; ++f) {
        const float d = tile[tid][f] - mean;
        m2 = fmaf(d, d, m2);
      }
    }
    float* pp = part + (((int64_t)b * n_blk + blk) * 128 + tid) * 4;
    pp[0] = (float)nv;
    pp[1] = c;
    pp[2] = sh;
    pp[3] = m2;
  }
}

// mel_stats_kernel: one CTA per (clip, bin) merges the per-tile partials
// (Chan's pairwise update in double, fixed tree) into the bin's mean and
// 1 / (std + 1e-5), std with the unbiased variance over the L valid frames.
__global__ void __launch_bounds__(256) mel_stats_kernel(const float* __restrict__ part, const MelArgs args,
                                                        int n_blk, float* __restrict__ stats) {
  SF_PDL_ENTRY();
  const int m = blockIdx.x, b = blockIdx.y;
  const int L = args.nf ? args.nf[b] : (int)(args.len[b] / 160);
  __shared__ double sn[256], smean[256], sm2[256];
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
    stats[((int64_t)b * 128 + m) * 2] = (float)smean[0];
    stats[((int64_t)b * 128 + m) * 2 + 1] = (float)(1.0 / (sd + 1e-5));
  }
}

// mel_apply_kernel: normalise in place, 2048 columns of one (clip, bin) row
// per CTA, eight independent loads in flight per thread; columns >= L -> 0.
constexpr int MEL_APPLY_COLS = 2048;

__global__ void __launch_bounds__(256) mel_apply_kernel(float* __restrict__ mel, const float* __restrict__ stats,
                                                        const MelArgs args, int T_cols) {
  SF_PDL_ENTRY();
  const int m = blockIdx.y, b = blockIdx.z;
  const int L = args.nf ? args.nf[b] : (int)(args.len[b] / 160);
  const float mu = stats[((int64_t)b * 128 + m) * 2], inv = stats[((int64_t)b * 128 + m) * 2 + 1];
  float* row = mel + ((int64_t)(args.row ? args.row[b] : b) * 128 + m) * T_cols;
  const int c0 = blockIdx.x * MEL_APPLY_COLS + threadIdx.x;
  float v[MEL_APPLY_COLS / 256];
#pragma unroll
  for (int j = 0; j < MEL_APPLY_COLS / 256; ++j) {
    const int t = c0 + 256 * j;
    v[j] = (t < L) ? row[t] : 0.f;
  }
#pragma unroll
  for (int j = 0; j < MEL_APPLY_COLS / 256; ++j) {
    const int t = c0 + 256 * j;
    if (t < T_cols) row[t] = (t < L) ? (v[j] - mu) * inv : 0.f;
  }
}

constexpr size_t MEL_REG_SMEM = (size_t)MEL_SPAN * 4 + (size_t)8 * MEL_PW * 4 + (size_t)128 * (MEL_FB + 1) * 4 +
                                (size_t)128 * MEL_MAX_NK * 4 + 128 * 4;

constexpr size_t MEL_SMEM =
    (size_t)MEL_SPAN * 4 + 128 * 8 + 258 * 8 + 512 * 4 + 8 * 256 * 8 + 128 * (MEL_FB + 1) * 4;

cudaError_t frontend_init_attributes() {
  cudaError_t e = cudaFuncSetAttribute(mel_frames_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)MEL_SMEM);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(mel_frames_reg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)MEL_REG_SMEM);
}

namespace {

// Both front-end paths over B clips (or windows) of T_cols columns; the
// partials take B * n_blk * 128 * 4 floats of `part`, path 1's per-bin
// (mean, 1 / (std + eps)) the B * 128 * 2 floats after them.
cudaError_t enqueue_mel(const float* audio, int B, int64_t n_buf, const MelArgs& args, const MelTables* tab,
                        float* mel, float* part, int T_cols, int path, cudaStream_t st) {
  // The >48 KB dynamic shared-memory attribute of the frame kernels is a
  // per-device setting made by frontend_init_attributes() with the device
  // current: by sf_create for an engine's device, and by sf_mel_noalloc's
  // one-time set-up for each device it runs on.
  const int n_blk = (T_cols + MEL_FB - 1) / MEL_FB;
  if (path == 1) {
    float* stats = part + (size_t)B * n_blk * 128 * 4;
    CK_LAUNCH(launch_k(mel_frames_reg_kernel, dim3(dim3(n_blk, B)), dim3(256), MEL_REG_SMEM, st, audio, n_buf, args,
                       tab, mel, part, T_cols, n_blk));
    CK_LAUNCH(launch_k(mel_stats_kernel, dim3(dim3(128, B)), dim3(256), 0, st, part, args, n_blk, stats));
    CK_LAUNCH(launch_k(mel_apply_kernel, dim3((T_cols + MEL_APPLY_COLS - 1) / MEL_APPLY_COLS, 128, B), dim3(256), 0,
                       st, mel, stats, args, T_cols));
    return cudaGetLastError();
  }
  CK_LAUNCH(launch_k(mel_frames_kernel, dim3(dim3(n_blk, B)), dim3(256), MEL_SMEM, st, audio, n_buf, args, tab, mel,
                     part, T_cols, n_blk));
  CK_LAUNCH(launch_k(mel_normalize_kernel, dim3(dim3(128, B)), dim3(256), 0, st, mel, part, args, T_cols, n_blk));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mel(const float* audio, int B, int64_t n_max, const MelArgs& args, const MelTables* tab,
                       float* mel, float* part, cudaStream_t st, int path) {
  return enqueue_mel(audio, B, n_max, args, tab, mel, part, (int)(1 + n_max / 160), path, st);
}

cudaError_t launch_mel_windows(const float* audio, int B, int64_t n_buf, const MelArgs& args, const MelTables* tab,
                               float* mel, float* part, int T_cols, cudaStream_t st, int path) {
  return enqueue_mel(audio, B, n_buf, args, tab, mel, part, T_cols, path, st);
}

size_t mel_part_floats(int B, int64_t n_max) {
  const int T_cols = (int)(1 + n_max / 160);
  const int n_blk = (T_cols + MEL_FB - 1) / MEL_FB;
  return (size_t)B * n_blk * 128 * 4 + (size_t)B * 128 * 2;
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
