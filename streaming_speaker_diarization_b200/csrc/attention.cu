// Attention over packed sequences.
//
// Conformer: relative-position MHSA ("Streaming Sortformer Diarizer",
// torch.export Fixes 6 on rel_shift): score(i, j) = ((q_i + u) . k_j +
// (q_i + v) . p_(i-j)) / sqrt(64), softmax over the sequence's keys.
// Transformer: plain MHSA, head dim 24.
//
// bf16 path (flash-style, mma.sync m16n8k16): one CTA = 64 query rows of one
// sequence x one head, 8 warps: two groups of 4 warps (16 query rows each)
// take alternate 64-key tiles and merge their partial softmax state at the
// end.  Per 64-key tile the warp computes
// AC = (Q+u) K^T (16 x 64) and, for the relative term, BD = (Q+v) P^T over
// the 80 relative distances its 16 rows x 64 keys can take; BD goes through
// a per-warp shared tile and is read back along the i - j diagonal.  Online
// softmax in fp32 (exp2 with the scale folded in), P.V from registers.
// fp32 path: one warp per query row (used by the fp32 engine mode).
#include <mutex>
#include "common.cuh"
#include "layers.h"

namespace sf {

// ---------------------------------------------------------------- fp32 path
template <int HD, bool REL>
__global__ void __launch_bounds__(128) attn_f32_kernel(const float* __restrict__ qkv, int D,
                                                       const float* __restrict__ ptab, int R,
                                                       const float* __restrict__ u, const float* __restrict__ vb,
                                                       float* __restrict__ ctx, const SeqTable* __restrict__ seq,
                                                       int M, int s_cap) {
  SF_PDL_ENTRY();
  extern __shared__ float att_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 4 + warp;
  const int h = blockIdx.y;
  float* sc = att_smem + warp * (s_cap + 2 * 64);
  float* qu = sc + s_cap;
  float* qv = qu + 64;
  if (r >= M) return;
  const int s = seq_of_row(seq, r);
  const int sb = seq->off[s], S = seq->off[s + 1] - sb, i = r - sb;
  const int ld = 3 * D;
  const float* q = qkv + (int64_t)r * ld + h * HD;
  for (int d = lane; d < HD; d += 32) {
    qu[d] = q[d] + (REL ? u[h * HD + d] : 0.f);
    if (REL) qv[d] = q[d] + vb[h * HD + d];
  }
  __syncwarp();
  const float scale = 1.0f / sqrtf((float)HD);
  float mx = -INFINITY;
  for (int j = lane; j < S; j += 32) {
    const float* k = qkv + (int64_t)(sb + j) * ld + D + h * HD;
    float a = 0.f;
    for (int d = 0; d < HD; ++d) a = fmaf(qu[d], k[d], a);
    if (REL) {
      const float* p = ptab + (int64_t)(i - j + R - 1) * D + h * HD;
      for (int d = 0; d < HD; ++d) a = fmaf(qv[d], p[d], a);
    }
    a *= scale;
    sc[j] = a;
    mx = fmaxf(mx, a);
  }
  mx = warp_max(mx);
  float sum = 0.f;
  for (int j = lane; j < S; j += 32) {
    const float e = expf(sc[j] - mx);
    sc[j] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  __syncwarp();
  const float inv = 1.f / sum;
  for (int d = lane; d < HD; d += 32) {
    float acc = 0.f;
    const float* v = qkv + (int64_t)sb * ld + 2 * D + h * HD + d;
    for (int j = 0; j < S; ++j) acc = fmaf(sc[j], v[(int64_t)j * ld], acc);
    ctx[(int64_t)r * D + h * HD + d] = acc * inv;
  }
}

// ---------------------------------------------------------------- bf16 path
__device__ __forceinline__ uint32_t s_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void ldsm4t(uint32_t a, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Copy rows [row0, row0 + nrows) x dims [0, HD) of a strided bf16 matrix into
// shared memory (row stride LDS), zero-filling rows outside [lo, hi) and
// dims >= HD up to HDP.
template <int HD, int HDP, int LDS>
__device__ __forceinline__ void load_rows(bf16* dst, const bf16* src, int64_t ld, int row0, int nrows, int lo,
                                          int hi, const float* add) {
  constexpr int CH = HDP / 8;   // 16-byte chunks per row
  for (int e = threadIdx.x; e < nrows * CH; e += blockDim.x) {
    const int rr = e / CH, ch = e % CH;
    const int row = row0 + rr;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (row >= lo && row < hi && ch * 8 < HD) {
      val = *reinterpret_cast<const uint4*>(src + (int64_t)row * ld + ch * 8);
      if (add) {
        bf16* pv = reinterpret_cast<bf16*>(&val);
#pragma unroll
        for (int t = 0; t < 8; ++t) pv[t] = __float2bfloat16_rn(__bfloat162float(pv[t]) + add[ch * 8 + t]);
      }
    }
    *reinterpret_cast<uint4*>(dst + rr * LDS + ch * 8) = val;
  }
}

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool pred) {
  const int sz = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit_() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait_() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Asynchronous version of load_rows (no bias add): rows outside [lo, hi) and
// dims >= HD arrive as zeros.
template <int HD, int HDP, int LDS>
__device__ __forceinline__ void load_rows_async(bf16* dst, const bf16* src, int64_t ld, int row0, int nrows, int lo,
                                                int hi, int tid, int nthr) {
  constexpr int CH = HDP / 8;
  for (int e = tid; e < nrows * CH; e += nthr) {
    const int rr = e / CH, ch = e % CH;
    const int row = row0 + rr;
    const bool ok = row >= lo && row < hi && ch * 8 < HD;
    const bf16* g = ok ? src + (int64_t)row * ld + ch * 8 : src;
    cp_async16_zfill(s_u32(dst + rr * LDS + ch * 8), g, ok);
  }
}

// NG warp groups of 4 warps: group g takes key tiles g, g + NG, g + 2 NG, ...
template <int HD, int HDP, bool REL, int NG = 2>
struct AttCfg {
  static constexpr int LDS = HDP + 8;
  static constexpr int TILE = 64 * LDS;                       // bf16 elements
  static constexpr int NQ = REL ? 2 : 1;
  // Q (+Qv) once; per warp group, K, V and the 128-row relative slice
  // double-buffered; per warp a 16 x 80 fp32 tile of relative scores
  static constexpr int BUF = 2 * TILE + (REL ? 2 * TILE : 0);
  static constexpr int SMEM = (NQ * TILE + NG * 2 * BUF) * 2 + (REL ? 4 * NG * 16 * 80 * 4 : 0);
  static constexpr int MERGE_FLOATS = 128 * (4 + 4 * (HDP / 8));   // a group's (m, l, O) handed to group 0
  static_assert(MERGE_FLOATS * 4 <= 2 * BUF * 2, "merge area fits in one group's buffers");
  static_assert(NG >= 2 && NG <= 8, "2 to 8 warp groups");
};

template <int HD, int HDP, bool REL, int NG = 2>
__global__ void __launch_bounds__(128 * NG) attn_bf16_kernel(const bf16* __restrict__ qkv, int D,
                                                        const bf16* __restrict__ ptab, int R,
                                                        const float* __restrict__ u, const float* __restrict__ vb,
                                                        bf16* __restrict__ ctx, const SeqTable* __restrict__ seq) {
  SF_PDL_ENTRY();
  using C = AttCfg<HD, HDP, REL, NG>;
  constexpr int LDS = C::LDS;
  extern __shared__ float4 att_smem4[];
  bf16* sQu = reinterpret_cast<bf16*>(att_smem4);
  bf16* sQv = sQu + (REL ? C::TILE : 0);
  bf16* sBuf0 = sQu + C::NQ * C::TILE;                        // per group: 2 x [K | V | P(128 rows, REL)]
  float* sBD = reinterpret_cast<float*>(sBuf0 + NG * 2 * C::BUF);

  const int g_tile = blockIdx.x, h = blockIdx.y;
  const int s = seq_of_tile(seq, g_tile);
  const int sb = seq->off[s], S = seq->off[s + 1] - sb;
  const int i0 = (g_tile - seq->tile_off[s]) * 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp >> 2, wq = warp & 3;     // key-tile group, 16-row query slice
  const int gtid = threadIdx.x & 127;
  bf16* sBuf = sBuf0 + grp * 2 * C::BUF;
  const int g = lane >> 2, q = lane & 3;
  const int64_t ld = 3 * D;
  const bf16* Qg = qkv + (int64_t)sb * ld + h * HD;
  const bf16* Kg = Qg + D;
  const bf16* Vg = Qg + 2 * D;

  load_rows<HD, HDP, LDS>(sQu, Qg, ld, i0, 64, 0, S, REL ? u + h * HD : nullptr);
  if (REL) load_rows<HD, HDP, LDS>(sQv, Qg, ld, i0, 64, 0, S, vb + h * HD);
  __syncthreads();
  constexpr int KS = HDP / 16;
  uint32_t aqu[KS][4], aqv[REL ? KS : 1][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int row = wq * 16 + (lane & 15), col = ks * 16 + (lane >> 4) * 8;
    ldsm4(s_u32(sQu + row * LDS + col), aqu[ks]);
    if (REL) ldsm4(s_u32(sQv + row * LDS + col), aqv[ks]);
  }

  constexpr int NO = HDP / 8;
  float o[NO][4];
#pragma unroll
  for (int n = 0; n < NO; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);

  // group `grp` takes key tiles grp, grp + NG, ...; each group double-buffers its own tiles
  auto prefetch = [&](int j0, int buf) {
    bf16* k_ = sBuf + buf * C::BUF;
    load_rows_async<HD, HDP, LDS>(k_, Kg, ld, j0, 64, 0, S, gtid, 128);
    load_rows_async<HD, HDP, LDS>(k_ + C::TILE, Vg, ld, j0, 64, 0, S, gtid, 128);
    if (REL)
      load_rows_async<HD, HDP, LDS>(k_ + 2 * C::TILE, ptab + h * HD, D, i0 - j0 - 63 + R - 1, 128, 0, 2 * R - 1,
                                    gtid, 128);
    cp_async_commit_();
  };
  auto group_sync = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(1 + grp) : "memory"); };
  if (grp * 64 < S) prefetch(grp * 64, 0);
  else cp_async_commit_();
  for (int k = 0;; ++k) {
    const int j0 = (grp + NG * k) * 64;
    if (j0 >= S) break;
    // tile k+1 of this group streams in while tile k is used
    if (j0 + NG * 64 < S) prefetch(j0 + NG * 64, (k + 1) & 1);
    else cp_async_commit_();
    cp_async_wait_<1>();
    group_sync();
    const bf16* sK = sBuf + (k & 1) * C::BUF;
    const bf16* sV = sK + C::TILE;
    const bf16* sP = sK + 2 * C::TILE;
    float sc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        const int nrow = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int col = ks * 16 + ((lane >> 3) & 1) * 8;
        ldsm4(s_u32(sK + nrow * LDS + col), b);
        mma16816(sc[2 * np], aqu[ks], b[0], b[1]);
        mma16816(sc[2 * np + 1], aqu[ks], b[2], b[3]);
      }
    if (REL) {
      float bd[10][4];
#pragma unroll
      for (int n = 0; n < 10; ++n) bd[n][0] = bd[n][1] = bd[n][2] = bd[n][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int np = 0; np < 5; ++np) {
          uint32_t b[4];
          const int nrow = wq * 16 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int col = ks * 16 + ((lane >> 3) & 1) * 8;
          ldsm4(s_u32(sP + nrow * LDS + col), b);
          mma16816(bd[2 * np], aqv[ks], b[0], b[1]);
          mma16816(bd[2 * np + 1], aqv[ks], b[2], b[3]);
        }
      }
      float* wbd = sBD + warp * 16 * 80;
#pragma unroll
      for (int n = 0; n < 10; ++n) {
        wbd[g * 80 + n * 8 + 2 * q] = bd[n][0];
        wbd[g * 80 + n * 8 + 2 * q + 1] = bd[n][1];
        wbd[(g + 8) * 80 + n * 8 + 2 * q] = bd[n][2];
        wbd[(g + 8) * 80 + n * 8 + 2 * q + 1] = bd[n][3];
      }
      __syncwarp();
      // row li, key lj -> relative column li - lj + 63 of this warp's window
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int li = g + ((e >> 1) << 3), lj = n * 8 + 2 * q + (e & 1);
          sc[n][e] += wbd[li * 80 + li - lj + 63];
        }
      __syncwarp();
    }
    // scale, mask keys beyond the sequence, online softmax
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j0 + n * 8 + 2 * q + (e & 1);
        float v = sc[n][e] * sl2;
        if (key >= S) v = -INFINITY;
        sc[n][e] = v;
        if (e < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
      }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float nm0 = fmaxf(m0, mx0), nm1 = fmaxf(m1, mx1);
    const float c0 = exp2f(m0 - nm0), c1 = exp2f(m1 - nm1);
    m0 = nm0;
    m1 = nm1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      sc[n][0] = exp2f(sc[n][0] - m0);
      sc[n][1] = exp2f(sc[n][1] - m0);
      sc[n][2] = exp2f(sc[n][2] - m1);
      sc[n][3] = exp2f(sc[n][3] - m1);
      ps0 += sc[n][0] + sc[n][1];
      ps1 += sc[n][2] + sc[n][3];
    }
    l0 = l0 * c0 + ps0;
    l1 = l1 * c1 + ps1;
#pragma unroll
    for (int n = 0; n < NO; ++n) {
      o[n][0] *= c0; o[n][1] *= c0; o[n][2] *= c1; o[n][3] *= c1;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {       // 16 keys per step
      uint32_t a[4];
      a[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
      a[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
      a[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      a[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
      for (int np = 0; np < NO / 2; ++np) {
        uint32_t b[4];
        const int krow = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = np * 16 + (lane >> 4) * 8;
        ldsm4t(s_u32(sV + krow * LDS + col), b);
        mma16816(o[2 * np], a, b[0], b[1]);
        mma16816(o[2 * np + 1], a, b[2], b[3]);
      }
    }
    group_sync();   // the whole group is done with this buffer before it is refilled
  }
  cp_async_wait_<0>();
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  // groups 1 .. NG-1 hand their running max, sum and unnormalised output to
  // group 0 (same query rows, same lane layout) through their own, now idle,
  // buffers; group 0 merges them in group order
  __syncthreads();
  if (grp > 0) {
    float* mg = reinterpret_cast<float*>(sBuf0 + grp * 2 * C::BUF) + gtid * (4 + 4 * NO);
    mg[0] = m0; mg[1] = m1; mg[2] = l0; mg[3] = l1;
#pragma unroll
    for (int n = 0; n < NO; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) mg[4 + 4 * n + e] = o[n][e];
  }
  __syncthreads();
  if (grp > 0) return;
#pragma unroll 1
  for (int g2 = 1; g2 < NG; ++g2) {
    const float* mg = reinterpret_cast<const float*>(sBuf0 + g2 * 2 * C::BUF) + gtid * (4 + 4 * NO);
    const float mb0 = mg[0], mb1 = mg[1], lb0 = mg[2], lb1 = mg[3];
    const float n0 = fmaxf(m0, mb0), n1 = fmaxf(m1, mb1);   // m0/m1 are finite: group 0 saw key 0
    const float ca0 = exp2f(m0 - n0), cb0 = exp2f(mb0 - n0), ca1 = exp2f(m1 - n1), cb1 = exp2f(mb1 - n1);
    l0 = l0 * ca0 + lb0 * cb0;
    l1 = l1 * ca1 + lb1 * cb1;
#pragma unroll
    for (int n = 0; n < NO; ++n) {
      o[n][0] = o[n][0] * ca0 + mg[4 + 4 * n + 0] * cb0;
      o[n][1] = o[n][1] * ca0 + mg[4 + 4 * n + 1] * cb0;
      o[n][2] = o[n][2] * ca1 + mg[4 + 4 * n + 2] * cb1;
      o[n][3] = o[n][3] * ca1 + mg[4 + 4 * n + 3] * cb1;
    }
    m0 = n0;
    m1 = n1;
  }
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const int r0 = i0 + wq * 16 + g, r1 = r0 + 8;
#pragma unroll
  for (int n = 0; n < NO; ++n) {
    const int d = n * 8 + 2 * q;
    if (d < HD) {
      if (r0 < S)
        *reinterpret_cast<__nv_bfloat162*>(ctx + (int64_t)(sb + r0) * D + h * HD + d) =
            __floats2bfloat162_rn(o[n][0] * inv0, o[n][1] * inv0);
      if (r1 < S)
        *reinterpret_cast<__nv_bfloat162*>(ctx + (int64_t)(sb + r1) * D + h * HD + d) =
            __floats2bfloat162_rn(o[n][2] * inv1, o[n][3] * inv1);
    }
  }
}

// ---------------------------------------------------------------- launchers

template <>
cudaError_t launch_relpos_attention<float>(const float* qkv, const float* ptab, int R, const float* u, const float* v,
                                           float* ctx, const SeqTable* seq, int /*n_tiles*/, int M, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const int s_cap = R;   // no sequence is longer than the position table
  const size_t smem = (size_t)4 * (s_cap + 128) * 4;
  CK_LAUNCH(launch_k(attn_f32_kernel<64, true>, dim3(dim3((M + 3) / 4, 8)), dim3(128), smem, st, qkv, 512, ptab, R, u, v, ctx, seq, M, s_cap));
  return cudaGetLastError();
}

template <>
cudaError_t launch_relpos_attention<bf16>(const bf16* qkv, const bf16* ptab, int R, const float* u, const float* v,
                                          bf16* ctx, const SeqTable* seq, int n_tiles, int M, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  CK_LAUNCH(launch_k(attn_bf16_kernel<64, 64, true>, dim3(dim3(n_tiles, 8)), dim3(256), AttCfg<64, 64, true>::SMEM, st, qkv, 512, ptab, R, u, v,
                                                                                             ctx, seq));
  return cudaGetLastError();
}

template <>
cudaError_t launch_mha<float>(const float* qkv, float* ctx, const SeqTable* seq, int /*n_tiles*/, int M, int R,
                              cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const int s_cap = R;   // no sequence is longer than R rows
  const size_t smem = (size_t)4 * (s_cap + 128) * 4;
  CK_LAUNCH(launch_k(attn_f32_kernel<24, false>, dim3(dim3((M + 3) / 4, 8)), dim3(128), smem, st, qkv, 192, nullptr, 0, nullptr, nullptr, ctx, seq,
                                                                      M, s_cap));
  return cudaGetLastError();
}

template <>
cudaError_t launch_mha<bf16>(const bf16* qkv, bf16* ctx, const SeqTable* seq, int n_tiles, int M, int /*R*/,
                             cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  CK_LAUNCH(launch_k(attn_bf16_kernel<24, 32, false>, dim3(dim3(n_tiles, 8)), dim3(256), AttCfg<24, 32, false>::SMEM, st, 
      qkv, 192, nullptr, 0, nullptr, nullptr, ctx, seq));
  return cudaGetLastError();
}

// fp32 path: one score row of up to R floats per warp (4 warps per CTA).
// The shared-memory limit is a per-kernel attribute of the process, so it
// only ever grows: an engine made for shorter sequences never lowers what
// an earlier engine's launches need.
int attention_f32_max_seq() { return 14000; }   // 4 x (14000 + 128) floats = 221 KB

cudaError_t attention_reserve_f32(int R) {
  static std::mutex mu;
  static int reserved = 0;
  if (R < 1 || R > attention_f32_max_seq()) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lock(mu);
  if (R <= reserved) return cudaSuccess;
  const int smem = 4 * (R + 128) * 4;
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_f32_kernel<24, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) reserved = R;
  return e;
}

cudaError_t attention_init_attributes() {
  cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<64, 64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       AttCfg<64, 64, true>::SMEM);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(attn_bf16_kernel<24, 32, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              AttCfg<24, 32, false>::SMEM);
}

}  // namespace sf
