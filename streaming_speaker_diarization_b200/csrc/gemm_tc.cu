// Blackwell tensor-core GEMM: C[M, N] = A[M, K] . W[N, K]^T, bf16 operands,
// fp32 accumulation in tensor memory, the shared fused epilogues.
//
// One CTA computes one 128 x BN output tile (BN = 64, 128 or 256) with 6
// warps:
//   warp 0  one thread issues TMA loads of 128 x 64 (A) and BN x 64 (W)
//           bf16 tiles, 128-byte swizzled, into a ring of STAGES buffers;
//   warp 1  allocates BN TMEM columns; one thread issues
//           tcgen05.mma.cta_group::1.kind::f16 (M=128, N=BN, K=16) four times
//           per 64-wide k-block and frees each buffer with tcgen05.commit;
//   warps 2-5 wait for the accumulator, read it with tcgen05.ld (each warp
//           its 32-lane TMEM quarter = 32 output rows, thread = row) and
//           apply the epilogue (epilogue_tma.cuh): finished row segments go
//           into swizzled 32-row shared-memory boxes stored by TMA; split-K
//           partials and row-remapped outputs take the staged epilogue
//           (epilogue_tile) instead.
// Full/empty mbarriers order the ring; every wait is bounded by a clock
// budget: a wait that runs out sets ERR_TIMEOUT in the engine's error word,
// raises a CTA-wide abort flag, the producer waits (bounded) for its own
// loads in flight, and TMEM is released before the CTA exits.
// No TMA or bulk load uses cluster multicast: every CTA loads its own
// operand tiles.  The CTA-pair kernel's tcgen05.commit carries the
// .multicast::cluster qualifier only to signal the "stage free" mbarriers
// of both CTAs of the pair on this GPU.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cstring>

#include "common.cuh"
#include "epilogue.cuh"
#include "epilogue_tma.cuh"
#include "layers.h"
#include "tcgen05.cuh"

namespace sf {
namespace {

constexpr int TC_BM = 128, TC_BK = 64;
// Instruction descriptor: bf16 x bf16 -> f32, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TC_BM >> 4) << 24);
}

template <int BN, int STAGES>
struct TcCfg {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int SMEM = 1024 + STAGES * (A_BYTES + B_BYTES) + 256;
  static_assert(STAGES * (A_BYTES + B_BYTES) >= 4 * 32 * 68 * 4 && STAGES * (A_BYTES + B_BYTES) >= 12 * 4096 + 2 * 128 * 8,
                "epilogue staging, TMA boxes and the LayerNorm statistics reuse the pipeline buffers");
};

// Epilogue of one warp's 32 rows: per CW-column chunk (CW = 64 or 32), the
// accumulator block goes TMEM -> registers -> shared tile (row stride CW + 4
// floats: conflict-free 16-byte writes by row and reads by column), then
// each lane writes 4 consecutive columns of one row per step, CW / 4 lanes
// per row (bias preloaded for its columns).  With split-K the raw partial
// tile goes to `part` instead.
template <int EK, int BN, int CW = 64>
__device__ __forceinline__ void epilogue_tile(const Epi& e, uint32_t tmem, float* stage, float* part, int M, int N,
                                              int m0, int n0, int q, int lane, int S, int cbeg = 0, int cend = BN) {
  constexpr int LD = CW + 4;          // staged row stride (floats)
  constexpr int LPR = CW / 4;         // lanes per row
  constexpr int RPI = 32 / LPR;       // rows per store instruction
  constexpr int NI = 32 / RPI;        // store steps per chunk
  const int l4 = lane % LPR, rh = lane / LPR;
#pragma unroll 1
  for (int c0 = cbeg; c0 < cend; c0 += CW) {
    {
      uint32_t v[CW];   // one wide TMEM load (one wait) per chunk
      if (CW == 64) tmem_ld64(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
      else tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
#pragma unroll
      for (int j = 0; j < CW; j += 4)
        *reinterpret_cast<float4*>(stage + lane * LD + j) =
            make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                        __uint_as_float(v[j + 3]));
    }
    __syncwarp();
    const int c = n0 + c0 + 4 * l4;
    if (S == 1 && EK == EPI_RESID) {
      // residual update: NI / 2 loads of x issued before the first store so
      // their latencies overlap (a load after a store to the same array
      // would otherwise wait for it)
      float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e.bias && c < N) bv = *reinterpret_cast<const float4*>(e.bias + c);
      constexpr int NB = NI / 2;
#pragma unroll 1
      for (int i0 = 0; i0 < NI; i0 += NB) {
        float4 xv[NB];
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          const int row = m0 + 32 * q + RPI * (i0 + i) + rh;
          if (row < M && c < N) xv[i] = *reinterpret_cast<const float4*>(epi_f32_ptr(e, row, c));
        }
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          const int rr = RPI * (i0 + i) + rh;
          const int row = m0 + 32 * q + rr;
          const float4 t = *reinterpret_cast<const float4*>(stage + rr * LD + 4 * l4);
          if (row < M && c < N) {
            float4 x = xv[i];
            x.x += e.alpha * (t.x + bv.x); x.y += e.alpha * (t.y + bv.y);
            x.z += e.alpha * (t.z + bv.z); x.w += e.alpha * (t.w + bv.w);
            *reinterpret_cast<float4*>(epi_f32_ptr(e, row, c)) = x;
          }
        }
      }
    } else if (S == 1) {
      float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e.bias && c < N) bv = *reinterpret_cast<const float4*>(e.bias + c);
#pragma unroll 4
      for (int i = 0; i < NI; ++i) {
        const int rr = RPI * i + rh;
        const int row = m0 + 32 * q + rr;
        float4 t = *reinterpret_cast<const float4*>(stage + rr * LD + 4 * l4);
        t.x += bv.x; t.y += bv.y; t.z += bv.z; t.w += bv.w;
        if (row < M && c < N) epi_store4<EK, bf16>(e, row, c, t);
      }
    } else {
#pragma unroll 4
      for (int i = 0; i < NI; ++i) {
        const int rr = RPI * i + rh;
        *reinterpret_cast<float4*>(part + (int64_t)(32 * q + rr) * BN + c0 + 4 * l4) =
            *reinterpret_cast<const float4*>(stage + rr * LD + 4 * l4);
      }
    }
    __syncwarp();
  }
}

// A residual epilogue reads the f32 block it updates: ask L2 for this warp's
// share (rows r0 .. r0 + nrows, columns c0 .. c0 + ncols) while the
// accumulator is still being computed, so the epilogue's loads hit L2.
__device__ __forceinline__ void prefetch_resid(const Epi& e, int M, int N, int r0, int nrows, int c0, int ncols,
                                               int lane) {
  if (e.kind != EPI_RESID) return;
  const int lpr = (ncols + 31) / 32;   // 128-byte lines per row
  for (int k = lane; k < nrows * lpr; k += 32) {
    const int r = r0 + k / lpr, c = c0 + (k % lpr) * 32;
    if (r < M && c < N) asm volatile("prefetch.global.L2 [%0];" ::"l"(epi_f32_ptr(e, r, c)));
  }
}

// Split-K finish: sum the S partial tiles (fixed order z = 0 .. S-1, so the
// result does not depend on which CTA arrives last) and apply the epilogue.
template <int EK, int BN>
__device__ __forceinline__ void reduce_tile(const Epi& e, const float* base, int M, int N, int m0, int n0, int q,
                                            int lane, int S) {
  const int l4 = lane & 15, rh = lane >> 4;
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 64) {
    const int c = n0 + c0 + 4 * l4;
    float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e.bias && c < N) bv = *reinterpret_cast<const float4*>(e.bias + c);
#pragma unroll 1
    for (int i0 = 0; i0 < 16; i0 += 4) {
      float4 acc[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int zz = 0; zz < S; ++zz) {
        float4 t[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int rr = 2 * (i0 + k) + rh;
          t[k] = __ldcg(reinterpret_cast<const float4*>(base + ((int64_t)zz * TC_BM + 32 * q + rr) * BN + c0 + 4 * l4));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc[k].x += t[k].x; acc[k].y += t[k].y; acc[k].z += t[k].z; acc[k].w += t[k].w;
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = m0 + 32 * q + 2 * (i0 + k) + rh;
        float4 t = acc[k];
        t.x += bv.x; t.y += bv.y; t.z += bv.z; t.w += bv.w;
        if (row < M && c < N) epi_store4<EK, bf16>(e, row, c, t);
      }
    }
  }
}

__device__ __forceinline__ void cluster_arrive_wait() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Row statistics of the whole output row from the cluster's partials: rank
// j of the cluster holds (mean, M2) of columns [64 j, 64 j + 64) of local
// row r in its `stat` array.  Chan's pairwise merge of equal-count parts:
// mean = average of the means, M2 = sum(M2_j) + 64 sum((mean_j - mean)^2).
__device__ __forceinline__ void ln_row_stats(const float2* stat, int r, int ncl, int ncols, float& mean,
                                             float& rstd) {
  const uint32_t a0 = su32(stat + r);
  float mj[8], m2j[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {   // all loads issued before any result is used
    mj[j] = 0.f;
    m2j[j] = 0.f;
    if (j < ncl) {
      uint32_t a;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(a0), "r"((uint32_t)j));
      asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(mj[j]), "=f"(m2j[j]) : "r"(a) : "memory");
    }
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < ncl) s += mj[j];
  mean = s / (float)ncl;
  float m2 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < ncl) {
      const float d = mj[j] - mean;
      m2 += m2j[j] + 64.f * d * d;
    }
  }
  rstd = 1.0f / sqrtf(m2 / (float)ncols + 1e-5f);
}

// EPI_RESID_LN epilogue of one warp's 32 rows of a 128 x 64 tile whose CTA
// is rank n0 / 64 of a cluster spanning the row block's N / 64 tiles; thread
// = row, the tile's 64 columns in registers.  x_new = x + alpha (acc + b)
// (x prefetched by the caller into xr); each thread takes (mean, M2) of its
// 64 values; after a cluster barrier every CTA merges the partials of all
// ranks for its rows and normalises its own columns; a second LayerNorm, if
// any, repeats the exchange on the first one's output.  The f32 row and the
// bf16 normalised row go out as three TMA box stores from `boxes` (12 KB).
// Every epilogue thread passes the same cluster barriers
// (n_cluster_barriers(e) of them) whether or not its CTA's accumulator is
// valid (`ok`), so no CTA of the cluster waits for ever; the last barrier
// keeps each CTA's statistics alive until its peers have read them.
__device__ __forceinline__ int n_cluster_barriers(const Epi& e) { return e.ln_g2 ? 3 : 2; }

__device__ __forceinline__ float2 row_stats64(const float* v) {
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < 64; ++k) s += v[k];
  const float mean = s * (1.f / 64.f);
  float m2 = 0.f;
#pragma unroll
  for (int k = 0; k < 64; ++k) {
    const float d = v[k] - mean;
    m2 = fmaf(d, d, m2);
  }
  return make_float2(mean, m2);
}

// Lane-spread epilogue parameters of a 64-column LayerNorm tile (bias, and
// the weights of one or two LayerNorms), read before the accumulator wait.
struct LnParams {
  float2 bias, g, b, g2, b2;
};

__device__ __forceinline__ void layer_norm64(float* v, float2 g, float2 b, float mean, float rstd) {
#pragma unroll
  for (int k = 0; k < 64; ++k) v[k] = (v[k] - mean) * rstd * col64(g, k) + col64(b, k);
}

// 64 f32 values as two 32-column boxes (128-byte rows) at b and b + 4 KB
__device__ __forceinline__ void stage_f32x64(uint32_t b, int lane, const float* v) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float* w = v + 32 * h + 4 * u;
      sts128(sw128_unit(b + h * EPI_BOX_BYTES, lane, u), __float_as_uint(w[0]), __float_as_uint(w[1]),
             __float_as_uint(w[2]), __float_as_uint(w[3]));
    }
}
__device__ __forceinline__ void stage_bf16x64(uint32_t b, int lane, const float* v) {
#pragma unroll
  for (int u = 0; u < 8; ++u)
    sts128(sw128_unit(b, lane, u), pack_bf16(v[8 * u], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
           pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
}

__device__ __forceinline__ void resid_ln_rows(const Epi& e, const CUtensorMap* mx, const CUtensorMap* mh,
                                              uint32_t tmem, uint8_t* boxes, float2* st1, float2* st2, int M, int N,
                                              int m_w, int n0, int q, int lane, bool ok, const float* xr,
                                              const LnParams& lp) {
  const int ncl = N / 64;
  const uint32_t sb = su32(boxes);
  float v[64];
  if (ok) {
    tmem_ld64(tmem + ((uint32_t)(32 * q) << 16), reinterpret_cast<uint32_t*>(v));
#pragma unroll
    for (int k = 0; k < 64; ++k) v[k] = xr[k] + e.alpha * (v[k] + col64(lp.bias, k));
  } else {
#pragma unroll
    for (int k = 0; k < 64; ++k) v[k] = 0.f;
  }
  st1[32 * q + lane] = ok ? row_stats64(v) : make_float2(0.f, 0.f);
  cluster_arrive_wait();
  float mean, rstd;
  ln_row_stats(st1, 32 * q + lane, ncl, N, mean, rstd);
  const bool two = e.ln_g2 != nullptr;
  if (!e.ln_xnorm) stage_f32x64(sb, lane, v);   // out <- x_new
  layer_norm64(v, lp.g, lp.b, mean, rstd);
  if (e.ln_xnorm) stage_f32x64(sb, lane, v);    // out <- LN(x_new)
  if (two) {
    st2[32 * q + lane] = ok ? row_stats64(v) : make_float2(0.f, 0.f);
    cluster_arrive_wait();
    ln_row_stats(st2, 32 * q + lane, ncl, N, mean, rstd);
    layer_norm64(v, lp.g2, lp.b2, mean, rstd);
  }
  stage_bf16x64(sb + 2 * EPI_BOX_BYTES, lane, v);
  fence_async_smem();
  __syncwarp();
  if (lane == 0 && ok && m_w < M) {
    tma_store_2d(mx, boxes, n0, m_w);
    tma_store_2d(mx, boxes + EPI_BOX_BYTES, n0 + 32, m_w);
    tma_store_2d(mh, boxes + 2 * EPI_BOX_BYTES, n0, m_w);
    bulk_commit();
    bulk_wait_read_all();
  }
  __syncwarp();
  cluster_arrive_wait();   // peers have read this CTA's statistics
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(192, 2) gemm_tc_kernel(const __grid_constant__ CUtensorMap ta,
                                                         const __grid_constant__ CUtensorMap tb,
                                                         const __grid_constant__ CUtensorMap mo,
                                                         const __grid_constant__ CUtensorMap mo2, int M, int N, int K,
                                                         Epi e, int* err, float* __restrict__ split_ws,
                                                         int* __restrict__ split_cnt, int tma_epi) {
  using C = TcCfg<BN, STAGES>;
  extern __shared__ uint8_t tc_smem[];
  uint8_t* sm = tc_smem + ((1024 - (su32(tc_smem) & 1023)) & 1023);
  uint8_t* sA = sm;
  uint8_t* sB = sm + STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * C::B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * TC_BM, n0 = blockIdx.x * BN;
  // split-K: this CTA covers k-blocks [kb0, kb1) of the tile's K range
  const int KB_all = (K + TC_BK - 1) / TC_BK;
  const int S = gridDim.z, z = blockIdx.z;
  const int kb0 = (int)((int64_t)KB_all * z / S), kb1 = (int)((int64_t)KB_all * (z + 1) / S);
  const int KB = kb1 - kb0;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&ta)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tb)) : "memory");
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"((uint32_t)BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Set-up above overlaps the previous kernel (programmatic dependent
  // launch).  The weights do not depend on it either: the producer issues
  // the first ring's weight tiles before waiting for the previous kernel's
  // memory; everything else touches global memory only after the wait.
  if (warp != 0) SF_PDL_ENTRY();

  if (warp == 0) {
    if (lane == 0) {
      const int pre = KB < STAGES ? KB : STAGES;   // stages whose empty barrier is free from the start
      for (int kb = 0; kb < pre; ++kb) {
        mbar_expect_tx(&full[kb], C::A_BYTES + C::B_BYTES);
        tma_load_2d(sB + kb * C::B_BYTES, &tb, &full[kb], (kb0 + kb) * TC_BK, n0);
      }
      pdl_wait();
      for (int kb = 0; kb < pre; ++kb) tma_load_2d(sA + kb * C::A_BYTES, &ta, &full[kb], (kb0 + kb) * TC_BK, m0);
      int issued = pre;
      for (int kb = pre; kb < KB; ++kb) {
        const int s = kb % STAGES, r = kb / STAGES;
        if (!mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        mbar_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
        tma_load_2d(sA + s * C::A_BYTES, &ta, &full[s], (kb0 + kb) * TC_BK, m0);
        tma_load_2d(sB + s * C::B_BYTES, &tb, &full[s], (kb0 + kb) * TC_BK, n0);
        ++issued;
      }
      if (*abort_flag) {   // let this CTA's own loads land before the shared memory is released
        for (int kb = issued - STAGES > 0 ? issued - STAGES : 0; kb < issued; ++kb) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&full[kb % STAGES], (kb / STAGES) & 1) && clock64() - t0 < WAIT_CYCLES) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BN);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES, r = kb / STAGES;
        if (!mbar_wait(&full[s], r & 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t ad = sw128_desc(su32(sA + s * C::A_BYTES));
        const uint64_t bd = sw128_desc(su32(sB + s * C::B_BYTES));
#pragma unroll
        for (int k = 0; k < TC_BK / 16; ++k)   // +32 bytes along K per MMA (encoded >> 4)
          umma_bf16(tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, (kb | k) != 0);
        umma_commit(&empty[s]);
      }
      umma_commit(accf);   // arrives once every MMA issued above has completed
      pdl_trigger();
    }
  } else if (e.kind == EPI_RESID_LN) {
    // thread = row: the residual row segment is read while the main loop runs
    const int q = warp & 3, m_w = m0 + 32 * q, row = m_w + lane;
    float2* st1 = reinterpret_cast<float2*>(sm + 4 * 3 * EPI_BOX_BYTES);
    float xr[64];
    load_resid32(e, row, M, n0, N, xr);
    load_resid32(e, row, M, n0 + 32, N, xr + 32);
    LnParams lp;
    lp.bias = lane_param64(e.bias, n0, N, lane);
    lp.g = lane_param64(e.ln_g, n0, N, lane);
    lp.b = lane_param64(e.ln_b, n0, N, lane);
    lp.g2 = lane_param64(e.ln_g2, n0, N, lane);
    lp.b2 = lane_param64(e.ln_b2, n0, N, lane);
    // warp-uniform: tcgen05.ld is a warp-wide instruction
    const bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, abort_flag) && !*abort_flag);
    if (!ok) *abort_flag = 1;
    tc_fence_after();
    resid_ln_rows(e, &mo, &mo2, tmem, sm + q * 3 * EPI_BOX_BYTES, st1, st1 + 128, M, N, m_w, n0, q, lane, ok, xr, lp);
  } else if (tma_epi) {
    // thread = row, TMA box stores; the pipeline buffers are free once the
    // accumulator is complete, so the boxes reuse them
    const int q = warp & 3, m_w = m0 + 32 * q;
    float xr[32];
    float2 b2;
    epi_prefetch<true, BN>(e, M, N, m_w, n0, 0, lane, xr, b2);
    if (__all_sync(0xffffffffu, mbar_wait(accf, 0, abort_flag) && !*abort_flag)) {
      tc_fence_after();
      BoxRing ring{sm + q * 2 * EPI_BOX_BYTES, 0};
      row_epilogue_any<BN, true>(e, &mo, &mo2, tmem + ((uint32_t)(32 * q) << 16), ring, M, N, m_w, n0, 0, 1, lane, xr,
                                 b2);
      ring.drain(lane);
    } else {
      *abort_flag = 1;
    }
  } else {
    // Staged epilogue (split-K partials, row-remapped or unaligned outputs):
    // per 64-column chunk, each warp copies its 32 x 64 accumulator block
    // from TMEM to a padded shared tile (thread = row), then writes it out
    // with lanes along the columns (one contiguous row segment per store
    // instruction).  The pipeline buffers are free once the accumulator is
    // complete, so the tiles reuse them.
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    float* stage = reinterpret_cast<float*>(sm) + q * (32 * 68);
    volatile int* last_flag = abort_flag + 1;
    prefetch_resid(e, M, N, m0 + 32 * q, 32, n0, BN, lane);
    if (mbar_wait(accf, 0, abort_flag) && !*abort_flag) {
      tc_fence_after();
      const int tile = blockIdx.y * gridDim.x + blockIdx.x;
      float* part = split_ws + ((int64_t)tile * S + z) * TC_BM * BN;
      switch (e.kind) {
        case EPI_BIAS: epilogue_tile<EPI_BIAS, BN>(e, tmem, stage, part, M, N, m0, n0, q, lane, S); break;
        case EPI_BIAS_RELU: epilogue_tile<EPI_BIAS_RELU, BN>(e, tmem, stage, part, M, N, m0, n0, q, lane, S); break;
        case EPI_BIAS_SWISH: epilogue_tile<EPI_BIAS_SWISH, BN>(e, tmem, stage, part, M, N, m0, n0, q, lane, S); break;
        case EPI_BIAS_GLU: epilogue_tile<EPI_BIAS_GLU, BN>(e, tmem, stage, part, M, N, m0, n0, q, lane, S); break;
        case EPI_RESID: epilogue_tile<EPI_RESID, BN>(e, tmem, stage, part, M, N, m0, n0, q, lane, S); break;
        case EPI_F32: epilogue_tile<EPI_F32, BN>(e, tmem, stage, part, M, N, m0, n0, q, lane, S); break;
        default: epilogue_tile<EPI_F32_AND_T, BN>(e, tmem, stage, part, M, N, m0, n0, q, lane, S); break;
      }
      if (S > 1) {
        // the last CTA of the tile to arrive sums the partials in split order
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 64) {
          const int prev = atomicAdd(&split_cnt[tile], 1);
          *last_flag = (prev == S - 1) ? 1 : 0;
          if (prev == S - 1) split_cnt[tile] = 0;   // ready for the next launch
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (*last_flag) {
          __threadfence();
          const float* base = split_ws + (int64_t)tile * S * TC_BM * BN;
          switch (e.kind) {
            case EPI_BIAS: reduce_tile<EPI_BIAS, BN>(e, base, M, N, m0, n0, q, lane, S); break;
            case EPI_BIAS_RELU: reduce_tile<EPI_BIAS_RELU, BN>(e, base, M, N, m0, n0, q, lane, S); break;
            case EPI_BIAS_SWISH: reduce_tile<EPI_BIAS_SWISH, BN>(e, base, M, N, m0, n0, q, lane, S); break;
            case EPI_BIAS_GLU: reduce_tile<EPI_BIAS_GLU, BN>(e, base, M, N, m0, n0, q, lane, S); break;
            case EPI_RESID: reduce_tile<EPI_RESID, BN>(e, base, M, N, m0, n0, q, lane, S); break;
            case EPI_F32: reduce_tile<EPI_F32, BN>(e, base, M, N, m0, n0, q, lane, S); break;
            default: reduce_tile<EPI_F32_AND_T, BN>(e, base, M, N, m0, n0, q, lane, S); break;
          }
        }
      }
    } else {
      *abort_flag = 1;
    }
  }
  if (e.kind == EPI_RESID_LN && warp < 2) {   // the epilogue warps' cluster barriers, for the whole CTA
    __syncwarp();
    for (int i = 0; i < n_cluster_barriers(e); ++i) cluster_arrive_wait();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)BN) : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag) set_err(err, ERR_TIMEOUT);
}


// Persistent variant for GEMMs with more tiles than SMs: each CTA walks the
// tiles blockIdx.x, blockIdx.x + gridDim.x, ... (n fastest, so co-running CTAs
// share A rows in L2).  Two TMEM accumulators of BN columns alternate between
// tiles, so the epilogue of tile i overlaps the mainloop of tile i + 1; the
// producer's ring of stages runs on across tiles.  Warps: 0 TMA producer,
// 1 MMA issuer, 2-9 epilogue (two warps per TMEM lane quarter, each draining
// half of the columns).  acc_full[a] is committed by the MMA thread;
// acc_empty[a] collects one arrival per epilogue warp.
template <int BN, int STAGES>
struct TcpCfg {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE_FLOATS = 8 * 2 * EPI_BOX_BYTES / 4;   // per epilogue warp two TMA boxes (or a 32 x 36 tile)
  // + barriers: STAGES full / empty, two accumulator pairs, two residual
  // loads per epilogue warp, the TMEM slot and the abort flag
  static constexpr int SMEM = 1024 + STAGES * (A_BYTES + B_BYTES) + STAGE_FLOATS * 4 + 512;
  // two accumulators, rounded up to a power of two
  static constexpr uint32_t TMEM_COLS = 2 * BN <= 256 ? 256u : 512u;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert((STAGES * (A_BYTES + B_BYTES)) % 1024 == 0, "box buffers stay 1024-byte aligned");
  static_assert((2 * STAGES + 4 + 16) * 8 + 8 <= 512, "barrier area");
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(320, 1) gemm_tcp_kernel(const __grid_constant__ CUtensorMap ta,
                                                          const __grid_constant__ CUtensorMap tb,
                                                          const __grid_constant__ CUtensorMap mo,
                                                          const __grid_constant__ CUtensorMap mo2, int M, int N, int K,
                                                          Epi e, int* err, int tma_epi) {
  using C = TcpCfg<BN, STAGES>;
  extern __shared__ uint8_t tc_smem[];
  uint8_t* sm = tc_smem + ((1024 - (su32(tc_smem) & 1023)) & 1023);
  uint8_t* sA = sm;
  uint8_t* sB = sm + STAGES * C::A_BYTES;
  float* stg = reinterpret_cast<float*>(sB + STAGES * C::B_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + C::STAGE_FLOATS);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;     // [2]
  uint64_t* acce = accf + 2;           // [2]
  uint64_t* rbar = acce + 2;           // [8][2] residual box loads of the epilogue warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (N + BN - 1) / BN;
  const int tiles = ((M + TC_BM - 1) / TC_BM) * tiles_n;
  const int KB = (K + TC_BK - 1) / TC_BK;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&ta)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tb)) : "memory");
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 8);
    }
    for (int b = 0; b < 16; ++b) mbar_init(&rbar[b], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  SF_PDL_ENTRY();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < tiles && !*abort_flag; tile += gridDim.x) {
        const int m0 = (tile / tiles_n) * TC_BM, n0 = (tile % tiles_n) * BN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag)) {
            *abort_flag = 1;
            break;
          }
          mbar_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
          tma_load_2d(sA + s * C::A_BYTES, &ta, &full[s], kb * TC_BK, m0);
          tma_load_2d(sB + s * C::B_BYTES, &tb, &full[s], kb * TC_BK, n0);
        }
      }
      if (*abort_flag) {   // let this CTA's own loads land before the shared memory is released
        for (int k = it - STAGES > 0 ? it - STAGES : 0; k < it; ++k) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&full[k % STAGES], (k / STAGES) & 1) && clock64() - t0 < WAIT_CYCLES) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BN);
      int it = 0, i = 0;
      for (int tile = blockIdx.x; tile < tiles && !*abort_flag; tile += gridDim.x, ++i) {
        const int a = i & 1, u = i >> 1;
        if (!mbar_wait(&acce[a], (u & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(a * BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&full[s], r & 1, abort_flag)) {
            *abort_flag = 1;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(su32(sA + s * C::A_BYTES));
          const uint64_t bd = sw128_desc(su32(sB + s * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k)
            umma_bf16(acc, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, (kb | k) != 0);
          umma_commit(&empty[s]);
        }
        umma_commit(&accf[a]);
      }
      pdl_trigger();
    }
  } else {
    const int q = warp & 3, hc = (warp - 2) >> 2;   // TMEM lane quarter, column half
    float* stage = stg + (warp - 2) * (32 * 36);
    BoxRing ring{reinterpret_cast<uint8_t*>(stg) + (warp - 2) * 2 * EPI_BOX_BYTES, 0};
    ResidTma rt{rbar + 2 * (warp - 2), 0u, 0u};
    const bool resid_tma = tma_epi && e.kind == EPI_RESID;
    float xr[32];
    float2 b2 = make_float2(0.f, 0.f);
    int i = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++i) {
      const int a = i & 1, u = i >> 1;
      const int m0 = (tile / tiles_n) * TC_BM, n0 = (tile % tiles_n) * BN;
      if (!tma_epi) prefetch_resid(e, M, N, m0 + 32 * q, 32, n0 + hc * BN / 2, BN / 2, lane);
      else if (resid_tma) resid_tma_prologue<BN>(e, &mo, ring, rt, M, N, m0 + 32 * q, n0, hc, 2, lane);
      else epi_prefetch<false, BN>(e, M, N, m0 + 32 * q, n0, hc, lane, xr, b2);
      if (__any_sync(0xffffffffu, !mbar_wait(&accf[a], u & 1, abort_flag) || *abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(a * BN);
      if (resid_tma) {
        if (!resid_tma_rows<BN>(e, &mo, acc + ((uint32_t)(32 * q) << 16), ring, rt, M, N, m0 + 32 * q, n0, hc, 2, lane,
                                abort_flag))
          *abort_flag = 1;
      } else if (tma_epi) {   // chunks alternate between the two warps of a lane quarter
        row_epilogue_any<BN, false>(e, &mo, &mo2, acc + ((uint32_t)(32 * q) << 16), ring, M, N, m0 + 32 * q, n0, hc, 2, lane,
                             xr, b2);
      } else {
        const int cb = hc * BN / 2, ce = cb + BN / 2;
        switch (e.kind) {
          case EPI_BIAS: epilogue_tile<EPI_BIAS, BN, 32>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
          case EPI_BIAS_RELU: epilogue_tile<EPI_BIAS_RELU, BN, 32>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
          case EPI_BIAS_SWISH: epilogue_tile<EPI_BIAS_SWISH, BN, 32>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
          case EPI_BIAS_GLU: epilogue_tile<EPI_BIAS_GLU, BN, 32>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
          case EPI_RESID: epilogue_tile<EPI_RESID, BN, 32>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
          case EPI_F32: epilogue_tile<EPI_F32, BN, 32>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
          default: epilogue_tile<EPI_F32_AND_T, BN, 32>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[a]);   // this warp is done reading accumulator a
    }
    if (lane == 0) resid_tma_drain(rt);
    ring.drain(lane);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                 : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag) set_err(err, ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------
// CTA-pair variant (tcgen05 cta_group::2): a cluster of two CTAs on two SMs
// computes one 256 x BN tile.  Each CTA loads its own 128 rows of A and its
// own BN/2 rows of W per k-block; the even CTA (rank 0) issues M = 256
// MMAs that read both CTAs' shared tiles, and each CTA's TMEM receives its
// 128 rows x BN accumulator.  Per output element each SM moves 2/3 of the
// operand bytes of the single-CTA 128 x 256 tile, so the same shared memory
// holds half again as many k-blocks in flight.
//   rank 0 warp 0 / rank 1 warp 0: TMA producers; both signal rank 0's
//     full[s] (rank 0 arms it with both CTAs' bytes);
//   rank 0 warp 1: MMA issuer; tcgen05.commit multicast frees empty[s] and
//     publishes acc_full[a] in both CTAs;
//   warps 2-9 of both CTAs: epilogue of their own 128 rows; each warp
//     arrives on rank 0's acc_empty[a] (16 arrivals per phase).
// Waits are bounded like the single-CTA kernels.  If either CTA gave up, both
// hold their shared memory ~200 us after the closing cluster barrier so that
// copies and MMAs still in flight land before it is released.  The loads
// carry no multicast.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory whose completion is signalled on an
// mbarrier that may live in the peer CTA (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier at this offset in both CTAs of the pair when
// every MMA issued so far has completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          su32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

constexpr int PAIR_BM = 256;

template <int BN, int STAGES>
struct Tc2Cfg {
  static constexpr int CW = 32;        // epilogue chunk width (columns) of the staged fallback epilogue
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = (BN / 2) * TC_BK * 2;
  static constexpr int STAGE_FLOATS = 8 * 2 * EPI_BOX_BYTES / 4;   // per epilogue warp two TMA boxes
  static_assert(STAGE_FLOATS >= 8 * 32 * (CW + 4), "fallback staging fits the box buffers");
  static constexpr int SMEM = 1024 + STAGES * (A_BYTES + B_BYTES) + STAGE_FLOATS * 4 + 512;
  static_assert((2 * STAGES + 4 + 16) * 8 + 16 <= 512, "barrier area");
  // TMEM columns: two accumulators, rounded up to a power of two
  static constexpr uint32_t TMEM_COLS = 2 * BN <= 256 ? 256u : 512u;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert(BN % 64 == 0 && BN <= 256 && (BN / 2) % 32 == 0, "pair tile width");
  static_assert(B_BYTES % 1024 == 0, "stage buffers stay 1024-byte aligned for the 128-byte swizzle");
};

// M = 256 instruction descriptor (bf16 x bf16 -> f32, K-major operands).
__host__ __device__ constexpr uint32_t idesc_bf16_m256(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(PAIR_BM >> 4) << 24);
}

template <int BN, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                    const __grid_constant__ CUtensorMap mo, const __grid_constant__ CUtensorMap mo2, int M, int N,
                    int K, Epi e, int* err, int tma_epi) {
  using C = Tc2Cfg<BN, STAGES>;
  extern __shared__ uint8_t tc_smem[];
  uint8_t* sm = tc_smem + ((1024 - (su32(tc_smem) & 1023)) & 1023);
  uint8_t* sA = sm;
  uint8_t* sB = sm + STAGES * C::A_BYTES;
  float* stg = reinterpret_cast<float*>(sB + STAGES * C::B_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + C::STAGE_FLOATS);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;     // [2]
  uint64_t* acce = accf + 2;           // [2], used in rank 0
  uint64_t* rbar = acce + 2;           // [8][2] residual box loads of the epilogue warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* peer_abort = abort_flag + 1;   // written by the other CTA at teardown

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int tiles_n = (N + BN - 1) / BN;
  const int tiles = ((M + PAIR_BM - 1) / PAIR_BM) * tiles_n;
  const int KB = (K + TC_BK - 1) / TC_BK;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&ta)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tb)) : "memory");
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 16);
    }
    for (int b = 0; b < 16; ++b) mbar_init(&rbar[b], 1);
    *abort_flag = 0;
    *peer_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  SF_PDL_ENTRY();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int tile = pair; tile < tiles && !*abort_flag; tile += npairs) {
        const int m0 = (tile / tiles_n) * PAIR_BM + TC_BM * (int)rank;
        const int n0 = (tile % tiles_n) * BN + (BN / 2) * (int)rank;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag)) {
            *abort_flag = 1;
            break;
          }
          if (rank == 0) mbar_expect_tx(&full[s], 2 * (C::A_BYTES + C::B_BYTES));
          const uint32_t fb = mapa_shared(su32(&full[s]), 0);
          tma_load_2d_pair(sA + s * C::A_BYTES, &ta, fb, kb * TC_BK, m0);
          tma_load_2d_pair(sB + s * C::B_BYTES, &tb, fb, kb * TC_BK, n0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_m256(BN);
      int it = 0, i = 0;
      for (int tile = pair; tile < tiles && !*abort_flag; tile += npairs, ++i) {
        const int a = i & 1, u = i >> 1;
        if (!mbar_wait(&acce[a], (u & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(a * BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&full[s], r & 1, abort_flag)) {
            *abort_flag = 1;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(su32(sA + s * C::A_BYTES));
          const uint64_t bd = sw128_desc(su32(sB + s * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k)
            umma_bf16_pair(acc, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, (kb | k) != 0);
          umma_commit_pair(&empty[s]);
        }
        umma_commit_pair(&accf[a]);
      }
      pdl_trigger();
    }
  } else {
    const int q = warp & 3, hc = (warp - 2) >> 2;   // TMEM lane quarter, column half
    float* stage = stg + (warp - 2) * (32 * (C::CW + 4));
    BoxRing ring{reinterpret_cast<uint8_t*>(stg) + (warp - 2) * 2 * EPI_BOX_BYTES, 0};
    ResidTma rt{rbar + 2 * (warp - 2), 0u, 0u};
    const bool resid_tma = tma_epi && e.kind == EPI_RESID;
    float xr[32];
    float2 b2 = make_float2(0.f, 0.f);
    int i = 0;
    for (int tile = pair; tile < tiles; tile += npairs, ++i) {
      const int a = i & 1, u = i >> 1;
      const int m0 = (tile / tiles_n) * PAIR_BM + TC_BM * (int)rank, n0 = (tile % tiles_n) * BN;
      if (!tma_epi) prefetch_resid(e, M, N, m0 + 32 * q, 32, n0 + hc * BN / 2, BN / 2, lane);
      else if (resid_tma) resid_tma_prologue<BN>(e, &mo, ring, rt, M, N, m0 + 32 * q, n0, hc, 2, lane);
      else epi_prefetch<false, BN>(e, M, N, m0 + 32 * q, n0, hc, lane, xr, b2);
      if (__any_sync(0xffffffffu, !mbar_wait(&accf[a], u & 1, abort_flag) || *abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(a * BN);
      const int cb = hc * BN / 2, ce = cb + BN / 2;
      if (resid_tma) {
        if (!resid_tma_rows<BN>(e, &mo, acc + ((uint32_t)(32 * q) << 16), ring, rt, M, N, m0 + 32 * q, n0, hc, 2, lane,
                                abort_flag))
          *abort_flag = 1;
      } else if (tma_epi) {
        row_epilogue_any<BN, false>(e, &mo, &mo2, acc + ((uint32_t)(32 * q) << 16), ring, M, N, m0 + 32 * q, n0, hc, 2, lane,
                             xr, b2);
      } else switch (e.kind) {
        case EPI_BIAS: epilogue_tile<EPI_BIAS, BN, C::CW>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
        case EPI_BIAS_RELU: epilogue_tile<EPI_BIAS_RELU, BN, C::CW>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
        case EPI_BIAS_SWISH: epilogue_tile<EPI_BIAS_SWISH, BN, C::CW>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
        case EPI_BIAS_GLU: epilogue_tile<EPI_BIAS_GLU, BN, C::CW>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
        case EPI_RESID: epilogue_tile<EPI_RESID, BN, C::CW>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
        case EPI_F32: epilogue_tile<EPI_F32, BN, C::CW>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
        default: epilogue_tile<EPI_F32_AND_T, BN, C::CW>(e, acc, stage, nullptr, M, N, m0, n0, q, lane, 1, cb, ce); break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(su32(&acce[a]), 0));   // accumulator a drained here
    }
    if (lane == 0) resid_tma_drain(rt);
    ring.drain(lane);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) st_cluster_u32(mapa_shared(su32((const void*)peer_abort), rank ^ 1u), 1u);
  __syncwarp();
  cluster_sync_all();   // no CTA leaves while its peer may still signal its barriers
  if (*abort_flag || *peer_abort) {
    // a wait gave up: copies or MMAs may still be in flight into either CTA
    uint64_t t0, t1;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    do {
      __nanosleep(10000);
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
    } while (t1 - t0 < 200000ull);
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                 : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag) set_err(err, ERR_TIMEOUT);
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

cudaError_t get_encoder() {
  if (g_encode) return cudaSuccess;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess) return e;
  if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

// 2-D bf16 tensor map over a row-major [rows x cols] matrix with row stride
// ld elements; box = box_rows x 64 columns, 128-byte swizzle, zero fill.
cudaError_t make_map(CUtensorMap* m, const void* base, int rows, int cols, int ld, int box_rows) {
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((int64_t)ld * 2) % 16) return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)TC_BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2-D output tensor map for the TMA box stores of the row-per-thread
// epilogue: 32-row boxes of box_cols elements, rows of 128 bytes (128-byte
// swizzle) or 64 bytes (64-byte swizzle).
bool make_out_map(CUtensorMap* m, const void* base, bool f32, int rows, int cols, int64_t ld, int box_cols) {
  const int esz = f32 ? 4 : 2;
  if (!base || (reinterpret_cast<uintptr_t>(base) & 15) || (ld * esz) % 16 || rows <= 0 || cols <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * esz)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, 32u};
  cuuint32_t estr[2] = {1, 1};
  const int row_bytes = box_cols * esz;
  CUresult r = g_encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output maps of an epilogue (row_epilogue / resid_ln_rows); false where the
// staged epilogue has to run instead (row remap, unaligned outputs).
bool make_epi_maps(const Epi& e, int M, int N, CUtensorMap* mo, CUtensorMap* mo2) {
  memset(mo, 0, sizeof(*mo));
  memset(mo2, 0, sizeof(*mo2));
  if (e.rpg) return false;
  switch (e.kind) {
    case EPI_BIAS:
    case EPI_BIAS_RELU:
    case EPI_BIAS_SWISH: return make_out_map(mo, e.out, false, M, N, e.ldo, 64);
    case EPI_BIAS_GLU: return make_out_map(mo, e.out, false, M, N / 2, e.ldo, 32);
    case EPI_RESID:
    case EPI_F32: return make_out_map(mo, e.out, true, M, N, e.ldo, 32);
    case EPI_F32_AND_T:
      return make_out_map(mo, e.out, true, M, N, e.ldo, 32) && make_out_map(mo2, e.out2, false, M, N, e.ldo2, 32);
    case EPI_RESID_LN:
      return make_out_map(mo, e.out, true, M, N, e.ldo, 32) && make_out_map(mo2, e.ln_h, false, M, N, e.ldh, 64);
    default: return false;
  }
}

template <int BN, int STAGES>
cudaError_t launch_tc(const bf16* A, int lda, const bf16* W, int M, int N, int K, int splits, const Epi& e,
                      const TcScratch& sc, cudaStream_t st) {
  CUtensorMap ta, tb, mo, mo2;
  cudaError_t r = make_map(&ta, A, M, K, lda, TC_BM);
  if (r != cudaSuccess) return r;
  r = make_map(&tb, W, N, K, K, BN);
  if (r != cudaSuccess) return r;
  const int te = (splits == 1 && make_epi_maps(e, M, N, &mo, &mo2)) ? 1 : 0;
  dim3 grid((N + BN - 1) / BN, (M + TC_BM - 1) / TC_BM, splits);
  CK_LAUNCH(launch_k(gemm_tc_kernel<BN, STAGES>, dim3(grid), dim3(192), TcCfg<BN, STAGES>::SMEM, st, ta, tb, mo, mo2, M,
                     N, K, e, sc.err, sc.ws, sc.cnt, te));
  return cudaGetLastError();
}

int g_num_sms = 148;
int g_ln_clusters[9] = {};   // co-resident clusters of n CTAs of gemm_tc_kernel<64, 8> (0: unusable)

// EPI_RESID_LN: 128 x 64 tiles, one cluster of N / 64 CTAs per row block.
template <int STAGES>
cudaError_t launch_tc_ln_s(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e,
                           const TcScratch& sc, cudaStream_t st) {
  constexpr int BN = 64;
  CUtensorMap ta, tb, mo, mo2;
  cudaError_t r = make_map(&ta, A, M, K, lda, TC_BM);
  if (r != cudaSuccess) return r;
  r = make_map(&tb, W, N, K, K, BN);
  if (r != cudaSuccess) return r;
  if (!make_epi_maps(e, M, N, &mo, &mo2)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(N / BN, (M + TC_BM - 1) / TC_BM, 1);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = TcCfg<BN, STAGES>::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = N / BN;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (g_launch_pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  CK_LAUNCH(cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, STAGES>, ta, tb, mo, mo2, M, N, K, e, sc.err,
                               (float*)nullptr, (int*)nullptr, 1));
  return cudaGetLastError();
}

// With programmatic dependent launch the single-wave GEMMs run with half
// the operand ring (96 KB of shared memory), so that a CTA of the next
// kernel fits on the same SM and starts its set-up and weight loads while
// this one finishes.
cudaError_t launch_tc_ln(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e,
                         const TcScratch& sc, cudaStream_t st) {
  if (g_launch_pdl) return launch_tc_ln_s<4>(A, lda, W, M, N, K, e, sc, st);
  return launch_tc_ln_s<8>(A, lda, W, M, N, K, e, sc, st);
}

template <int BN, int STAGES>
cudaError_t launch_tcp(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e, const TcScratch& sc,
                       cudaStream_t st) {
  CUtensorMap ta, tb, mo, mo2;
  cudaError_t r = make_map(&ta, A, M, K, lda, TC_BM);
  if (r != cudaSuccess) return r;
  r = make_map(&tb, W, N, K, K, BN);
  if (r != cudaSuccess) return r;
  const int te = make_epi_maps(e, M, N, &mo, &mo2) ? 1 : 0;
  const int tiles = ((M + TC_BM - 1) / TC_BM) * ((N + BN - 1) / BN);
  const int grid = tiles < g_num_sms ? tiles : g_num_sms;
  CK_LAUNCH(launch_k(gemm_tcp_kernel<BN, STAGES>, dim3(grid), dim3(320), TcpCfg<BN, STAGES>::SMEM, st, ta, tb, mo, mo2,
                     M, N, K, e, sc.err, te));
  return cudaGetLastError();
}

int g_max_pairs = 0;   // co-resident CTA pairs of gemm_tc2_kernel (0: not queried)

template <int BN, int STAGES>
cudaError_t launch_tc2(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e, const TcScratch& sc,
                       cudaStream_t st) {
  CUtensorMap ta, tb, mo, mo2;
  cudaError_t r = make_map(&ta, A, M, K, lda, TC_BM);
  if (r != cudaSuccess) return r;
  r = make_map(&tb, W, N, K, K, BN / 2);
  if (r != cudaSuccess) return r;
  const int te = make_epi_maps(e, M, N, &mo, &mo2) ? 1 : 0;
  const int tiles = ((M + PAIR_BM - 1) / PAIR_BM) * ((N + BN - 1) / BN);
  const int cap = g_max_pairs > 0 ? g_max_pairs : g_num_sms / 2;
  const int pairs = tiles < cap ? tiles : cap;
  CK_LAUNCH(launch_k(gemm_tc2_kernel<BN, STAGES>, dim3(2 * pairs), dim3(320), Tc2Cfg<BN, STAGES>::SMEM, st, ta, tb, mo,
                     mo2, M, N, K, e, sc.err, te));
  return cudaGetLastError();
}

}  // namespace

// 2-D bf16 tensor map (row-major [rows x cols], row stride ld elements), box
// box_rows x 64 columns, 128-byte swizzle, zero fill outside the matrix.
cudaError_t make_bf16_map_sw128(CUtensorMap* m, const void* base, int rows, int cols, int ld, int box_rows) {
  cudaError_t r = get_encoder();
  if (r != cudaSuccess) return r;
  return make_map(m, base, rows, cols, ld, box_rows);
}

int g_gemm_pairs = 1;
int g_gemm_pair_bn = 0;

// Pair tile width for a multi-wave GEMM on the CTA-pair kernel: the fewest
// estimated microseconds over BN = 256 / 192 / 128, counting whole rounds of
// tiles over the co-resident pairs (the last round is as long as a full one)
// and per tile a fixed ~1 us plus a per-k-block time that shrinks with BN.
int gemm_pair_plan(int M, int N, int K) {
  const int pairs = g_max_pairs > 0 ? g_max_pairs : g_num_sms / 2;
  const int tm = (M + PAIR_BM - 1) / PAIR_BM, KB = (K + TC_BK - 1) / TC_BK;
  double best = 1e30;
  int bb = 256;
  for (int bn : {256, 192, 128}) {
    const int tiles = tm * ((N + bn - 1) / bn);
    const int rounds = (tiles + pairs - 1) / pairs;
    const double t = rounds * (1.0 + KB * (bn == 256 ? 0.40 : bn == 192 ? 0.33 : 0.27));
    if (t < best * 0.98) {
      best = t;
      bb = bn;
    }
  }
  return bb;
}

// Tile width BN and split count S from a cost model of this kernel on 148
// SMs, calibrated with per-phase timestamps on B200 (with the staged
// epilogue; the TMA-store epilogue is shorter, by about the same amount for
// every choice): per CTA ~1.4 us of set-up and first-load latency, ~0.28 us
// per 64-wide k-block (bounded by loads in flight, nearly independent of
// BN), and an epilogue of ~1.4 / 2.1 / 3.8 us for BN = 64 / 128 / 256; a
// split-K partial round trip costs about (BN / 64) x (1.5 + 0.9 S) us.
// Splits need scratch and at most 2 waves.
void gemm_tc_plan(int M, int N, int K, const TcScratch& sc, int* bn_out, int* s_out) {
  const int tm = (M + TC_BM - 1) / TC_BM;
  const int KB = (K + TC_BK - 1) / TC_BK;
  double best = 1e30;
  int bb = 64, bs = 1;
  for (int bn : {256, 128, 64}) {
    const int tiles = tm * ((N + bn - 1) / bn);
    for (int sp : {1, 2, 3, 4}) {
      if (sp > 1 && (!sc.ws || !sc.cnt || sp > KB || (int64_t)tiles * sp > 2 * 148 ||
                     (size_t)tiles * sp * TC_BM * bn * 4 > sc.ws_bytes || tiles > sc.cnt_len))
        continue;
      const int waves = (tiles * sp + 147) / 148;
      const int kb_per = (KB + sp - 1) / sp;
      const double epi = sp == 1 ? (bn == 64 ? 1.4 : bn == 128 ? 2.1 : 3.8) : (bn / 64.0) * (1.5 + 0.9 * sp);
      const double t = waves * (1.4 + 0.28 * kb_per + epi);
      if (t < best * 0.97) {
        best = t;
        bb = bn;
        bs = sp;
      }
    }
  }
  *bn_out = bb;
  *s_out = bs;
}

bool gemm_ln_fusable(int M, int N, int K) {
  if (M <= 0 || K % 8 || N % 64 || N / 64 > 8) return false;
  return (M + TC_BM - 1) / TC_BM <= g_ln_clusters[N / 64];
}

cudaError_t gemm_bf16_tc(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e,
                         const TcScratch& sc, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  if (N % 16 || K % 8) return cudaErrorInvalidValue;
  cudaError_t r = get_encoder();
  if (r != cudaSuccess) return r;
  if (e.kind == EPI_RESID_LN) {
    if (!gemm_ln_fusable(M, N, K) || !e.ln_g || !e.ln_b || !e.ln_h || (e.ln_g2 && (!e.ln_b2 || !e.ln_xnorm)) ||
        e.rpg || (reinterpret_cast<uintptr_t>(e.out) & 15) || (reinterpret_cast<uintptr_t>(e.ln_h) & 15) ||
        e.ldo % 4 || e.ldh % 8)
      return cudaErrorInvalidValue;
    return launch_tc_ln(A, lda, W, M, N, K, e, sc, st);
  }
  int bn, sp;
  gemm_tc_plan(M, N, K, sc, &bn, &sp);
  // more tiles than SMs: the persistent kernel overlaps each tile's epilogue
  // with the next tile's mainloop
  if (sp == 1 && N >= 128 && ((M + TC_BM - 1) / TC_BM) * ((N + bn - 1) / bn) > g_num_sms) {
    // CTA pairs: every such GEMM in mode 2; in mode 1 those with K >= 1024
    // and N >= 256, where the pair kernel's deeper operand ring wins (the
    // single-CTA kernel leads on shorter K, whose time goes to the epilogue)
    if (g_gemm_pairs == 2 || (g_gemm_pairs == 1 && K >= 1024 && N >= 256)) {
      switch (g_gemm_pair_bn ? g_gemm_pair_bn : gemm_pair_plan(M, N, K)) {
        case 256: return launch_tc2<256, 5>(A, lda, W, M, N, K, e, sc, st);
        case 192: return launch_tc2<192, 5>(A, lda, W, M, N, K, e, sc, st);
        default: return launch_tc2<128, 6>(A, lda, W, M, N, K, e, sc, st);
      }
    }
    // whole tiles where N allows: 192 columns for N = 192 or 576 (the
    // d 192 Transformer), else 256 or 128
    if (N % 256 && N % 192 == 0) return launch_tcp<192, 3>(A, lda, W, M, N, K, e, sc, st);
    if (N >= 256) return launch_tcp<256, 3>(A, lda, W, M, N, K, e, sc, st);
    return launch_tcp<128, 4>(A, lda, W, M, N, K, e, sc, st);
  }
  if (g_launch_pdl) {   // lean rings: two CTAs per SM (see launch_tc_ln)
    switch (bn) {
      case 256: return launch_tc<256, 4>(A, lda, W, M, N, K, sp, e, sc, st);
      case 128: return launch_tc<128, 3>(A, lda, W, M, N, K, sp, e, sc, st);
      default: return launch_tc<64, 4>(A, lda, W, M, N, K, sp, e, sc, st);
    }
  }
  switch (bn) {
    case 256: return launch_tc<256, 4>(A, lda, W, M, N, K, sp, e, sc, st);
    case 128: return launch_tc<128, 6>(A, lda, W, M, N, K, sp, e, sc, st);
    default: return launch_tc<64, 8>(A, lda, W, M, N, K, sp, e, sc, st);
  }
}

cudaError_t gemm_tc_init_attributes() {
  cudaError_t r = get_encoder();
  if (r != cudaSuccess) return r;
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) ==
                                                 cudaSuccess && n_sm > 0)
    g_num_sms = n_sm;
  r = cudaFuncSetAttribute(gemm_tc2_kernel<256, 5>, cudaFuncAttributeMaxDynamicSharedMemorySize, Tc2Cfg<256, 5>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc2_kernel<192, 5>, cudaFuncAttributeMaxDynamicSharedMemorySize, Tc2Cfg<192, 5>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc2_kernel<128, 6>, cudaFuncAttributeMaxDynamicSharedMemorySize, Tc2Cfg<128, 6>::SMEM);
  if (r != cudaSuccess) return r;
  {   // every configuration holds one CTA per SM: the same number of co-resident pairs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (g_num_sms / 2));
    cfg.blockDim = dim3(320);
    cfg.dynamicSmemBytes = Tc2Cfg<256, 5>::SMEM;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<256, 5>, &cfg) == cudaSuccess && n > 0) g_max_pairs = n;
    cudaGetLastError();
  }
  r = cudaFuncSetAttribute(gemm_tcp_kernel<256, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcpCfg<256, 3>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tcp_kernel<128, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcpCfg<128, 4>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tcp_kernel<192, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcpCfg<192, 3>::SMEM);
  if (r != cudaSuccess) return r;
  r = cudaFuncSetAttribute(gemm_tc_kernel<256, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TcCfg<256, 4>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc_kernel<128, 6>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<128, 6>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc_kernel<64, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<64, 8>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc_kernel<128, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<128, 3>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc_kernel<64, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<64, 4>::SMEM);
  if (r != cudaSuccess) return r;
  for (int n = 1; n <= 8; ++n) {   // clusters of n CTAs for the LayerNorm-fused epilogue
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n, 1, 1);
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = TcCfg<64, 8>::SMEM;
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeClusterDimension;
    a.val.clusterDim.x = n;
    a.val.clusterDim.y = 1;
    a.val.clusterDim.z = 1;
    cfg.attrs = &a;
    cfg.numAttrs = 1;
    int n_cl = 0;
    g_ln_clusters[n] = cudaOccupancyMaxActiveClusters(&n_cl, gemm_tc_kernel<64, 8>, &cfg) == cudaSuccess ? n_cl : 0;
    cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace sf
