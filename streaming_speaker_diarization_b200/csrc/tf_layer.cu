// One post-LN Transformer layer after its attention, fused ("Streaming
// Sortformer Diarizer", Pipeline: 18-layer Transformer encoder, d_model 192,
// 8 heads, FFN 768 with ReLU, post-LN):
//   x  <- LN1(x + ctx Wo^T + bo)
//   x  <- LN2(x + relu(x W1^T + b1) W2^T + b2)
//   qkv <- x Wqkv'^T + bqkv'   (the next layer's projection), or h <- act(x)
// over one 128-row block per cluster of four CTAs.  Rank j of the cluster
// owns columns [48 j, 48 j + 48) of x, hidden columns [192 j, 192 j + 192)
// and qkv columns [144 j, 144 j + 144):
//   O    acc (128 x 48)  = ctx . Wo[48 j ..]^T             K = 192, TMEM [0, 48)
//        + bias + x, LayerNorm statistics exchanged over the cluster, y1 =
//        LN1 written to x and, as bf16, into every rank's A operand buffer Y
//   F1   acc (128 x 192) = Y . W1[192 j ..]^T               K = 192, TMEM [64, 256)
//        relu(+ b1) as bf16 into the local buffer H
//   F2   acc (128 x 192) = H . W2[:, 192 j ..]^T            K = 192 (this rank's
//        hidden slice), TMEM [256, 448): a partial sum of all 192 outputs;
//        the four partials are summed for each rank's own 48 columns over
//        distributed shared memory (rank order), + b2 + y1, LayerNorm as
//        above, y2 to x and into every rank's Y
//   Q    acc (128 x 144) = Y . Wqkv'[144 j ..]^T            K = 192, TMEM [0, 144)
//        + bias, bf16 to qkv (or, after the last layer, y2 as bf16 to h)
// Warps: 0 TMA loads (ctx into its own buffer, the weight tiles through a
// three-stage ring), 1 the MMAs (one thread), 2-5 the epilogues (thread =
// row = TMEM lane).  All 192 threads pass the same six cluster barriers:
// every wait between two barriers depends only on work that some thread
// does before reaching the next barrier, so the barriers cannot deadlock;
// every mbarrier wait is bounded (a wait that runs out raises ERR_TIMEOUT,
// skips the CTA's remaining work and still passes the barriers).
#include "common.cuh"
#include "layers.h"
#include "tcgen05.cuh"
#include "attn_common.cuh"

namespace sf {
namespace {

constexpr int TL_E = 192, TL_F = 768, TL_R = 128, TL_C = 4;
constexpr int TL_EJ = TL_E / TL_C;       // 48
constexpr int TL_FJ = TL_F / TL_C;       // 192
constexpr int TL_QJ = 3 * TL_E / TL_C;   // 144
constexpr int TL_KB = TL_E / 64;         // 3 k-blocks of 64 for every product
constexpr int TL_RING = 3;

struct TlSmem {
  static constexpr int KB_A = TL_R * 64 * 2;          // 16 KB: 128 rows x 64 bf16, 128-byte swizzle
  static constexpr int STAGE = TL_FJ * 64 * 2;        // 24 KB: the widest weight tile
  static constexpr int OFF_CTX = 0;                   // 3 x 16 KB
  static constexpr int OFF_Y = OFF_CTX + TL_KB * KB_A;
  static constexpr int OFF_H = OFF_Y + TL_KB * KB_A;
  static constexpr int OFF_RING = OFF_H + TL_KB * KB_A;
  static constexpr int OFF_ST = OFF_RING + TL_RING * STAGE;   // 2 x 128 float2 statistics
  static constexpr int OFF_PAR = OFF_ST + 2 * TL_R * 8;      // this rank's biases and LayerNorm weights
  static constexpr int N_PAR = 6 * TL_EJ + TL_FJ + TL_QJ;     // bo, ln1 g/b, b2, ln2 g/b (48 each), b1, bq
  static constexpr int OFF_BAR = OFF_PAR + N_PAR * 4;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert(TL_E * TL_R * 4 == 2 * TL_KB * KB_A, "F2 partial staging (f32 [192][128]) fills CTX and H");
};

// tmem column bases
constexpr uint32_t TM_O = 0, TM_F1 = 64, TM_F2 = 256, TM_Q = 0;

__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cl_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cl_map(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t a, uint4 v) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Row statistics of the whole 192-column row from the four ranks' (mean,
// M2) over 48 columns each (Chan's merge of equal-count parts).
__device__ __forceinline__ void tl_row_stats(const float2* st, int r, float& mean, float& rstd) {
  const uint32_t a0 = su32(st + r);
  float mj[TL_C], m2j[TL_C];
#pragma unroll
  for (int j = 0; j < TL_C; ++j)
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(mj[j]), "=f"(m2j[j]) : "r"(cl_map(a0, j)) : "memory");
  mean = 0.25f * ((mj[0] + mj[1]) + (mj[2] + mj[3]));
  float m2 = 0.f;
#pragma unroll
  for (int j = 0; j < TL_C; ++j) {
    const float d = mj[j] - mean;
    m2 += m2j[j] + (float)TL_EJ * d * d;
  }
  rstd = 1.0f / sqrtf(m2 / (float)TL_E + 1e-5f);
}
__device__ __forceinline__ float2 tl_local_stats(const float* v) {
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < TL_EJ; ++c) s += v[c];
  const float mean = s * (1.f / TL_EJ);
  float m2 = 0.f;
#pragma unroll
  for (int c = 0; c < TL_EJ; ++c) {
    const float d = v[c] - mean;
    m2 = fmaf(d, d, m2);
  }
  return make_float2(mean, m2);
}

// bf16 copy of this rank's 48 columns of row r into the Y buffer of every
// rank of the cluster (K-major, 128-byte swizzle, k-block = column / 64).
__device__ __forceinline__ void tl_broadcast(uint32_t y_base, int r, int j, const float* v) {
#pragma unroll
  for (int g = 0; g < TL_EJ / 8; ++g) {
    const int col = TL_EJ * j + 8 * g;
    const uint4 w = make_uint4(pack_bf16(v[8 * g], v[8 * g + 1]), pack_bf16(v[8 * g + 2], v[8 * g + 3]),
                               pack_bf16(v[8 * g + 4], v[8 * g + 5]), pack_bf16(v[8 * g + 6], v[8 * g + 7]));
    const uint32_t off = (uint32_t)((col >> 6) * TlSmem::KB_A) + sw128_off(r, (col & 63) >> 3);
#pragma unroll
    for (int rk = 0; rk < TL_C; ++rk) st_cluster_v4(cl_map(y_base + off, rk), w);
  }
}

__global__ void __launch_bounds__(192, 1) tf_layer_kernel(
    const __grid_constant__ CUtensorMap t_ctx, const __grid_constant__ CUtensorMap t_wo,
    const __grid_constant__ CUtensorMap t_w1, const __grid_constant__ CUtensorMap t_w2,
    const __grid_constant__ CUtensorMap t_wq, TfLayerArgs a, int M, int* err) {
  using L = TlSmem;
  extern __shared__ uint8_t tl_smem[];
  uint8_t* sm = tl_smem + ((1024 - (su32(tl_smem) & 1023)) & 1023);
  uint8_t* sCtx = sm + L::OFF_CTX;
  uint8_t* sY = sm + L::OFF_Y;
  uint8_t* sH = sm + L::OFF_H;
  uint8_t* sRing = sm + L::OFF_RING;
  float2* st1 = reinterpret_cast<float2*>(sm + L::OFF_ST);
  float2* st2 = st1 + TL_R;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);   // [TL_RING]
  uint64_t* empty = full + TL_RING;                                 // [TL_RING]
  uint64_t* ctx_full = empty + TL_RING;
  uint64_t* o_done = ctx_full + 1;
  uint64_t* f1_done = o_done + 1;
  uint64_t* h_ready = f1_done + 1;
  uint64_t* f2_done = h_ready + 1;
  uint64_t* q_done = f2_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = (int)cl_rank();
  const int m0 = blockIdx.y * TL_R;
  const bool has_next = a.bq != nullptr;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&t_ctx)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&t_wo)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&t_w1)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&t_w2)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&t_wq)) : "memory");
    for (int s = 0; s < TL_RING; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(ctx_full, 1);
    mbar_init(o_done, 1);
    mbar_init(f1_done, 1);
    mbar_init(h_ready, 4);
    mbar_init(f2_done, 1);
    mbar_init(q_done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)), "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loads
    // Ring items: Wo k-blocks 0-2, W1 0-2 (before barrier A), W2 0-2 (after
    // B: their slots free when F1's MMAs complete), Wqkv' 0-2 (their slots
    // free when F2's MMAs complete, before barrier C).
    int item = 0;
    auto load_w = [&](const CUtensorMap* t, int x, int y, int rows) -> bool {
      const int s = item % TL_RING, r = item / TL_RING;
      ++item;
      if (!mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag)) return false;
      mbar_expect_tx(&full[s], (uint32_t)rows * 128);
      tma_load_2d(sRing + s * L::STAGE, t, &full[s], x, y);
      return true;
    };
    bool ok = true;
    if (lane == 0) {
      for (int kb = 0; ok && kb < TL_KB; ++kb) ok = load_w(&t_wo, 64 * kb, TL_EJ * j, TL_EJ);   // weights first
      pdl_wait();   // the previous kernel's ctx and x
      if (ok) {
        mbar_expect_tx(ctx_full, TL_KB * L::KB_A);
        for (int kb = 0; kb < TL_KB; ++kb) tma_load_2d(sCtx + kb * L::KB_A, &t_ctx, ctx_full, 64 * kb, m0);
      }
      for (int kb = 0; ok && kb < TL_KB; ++kb) ok = load_w(&t_w1, 64 * kb, TL_FJ * j, TL_FJ);
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
    cl_sync();   // A
    cl_sync();   // B
    if (lane == 0) {
      for (int kb = 0; ok && !*abort_flag && kb < TL_KB; ++kb) ok = load_w(&t_w2, TL_FJ * j + 64 * kb, 0, TL_E);
      if (has_next)
        for (int kb = 0; ok && !*abort_flag && kb < TL_KB; ++kb) ok = load_w(&t_wq, 64 * kb, TL_QJ * j, TL_QJ);
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
    cl_sync();   // C
    cl_sync();   // D
    cl_sync();   // E
    if (lane == 0 && *abort_flag) {   // let this CTA's own loads land before its shared memory is released
      for (int k = item - TL_RING > 0 ? item - TL_RING : 0; k < item; ++k) {
        const long long c0 = clock64();
        while (!mbar_try_wait(&full[k % TL_RING], (k / TL_RING) & 1) && clock64() - c0 < WAIT_CYCLES) {
        }
      }
      const long long c0 = clock64();
      while (!mbar_try_wait(ctx_full, 0) && clock64() - c0 < WAIT_CYCLES) {
      }
    }
    __syncwarp();
    cl_sync();   // F
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMAs
    int item = 0;
    // one product: A = three 16 KB k-blocks at a_base, B = the next three ring items
    auto product = [&](uint8_t* a_base, uint32_t tm, int n, uint64_t* done) -> bool {
      const uint32_t idesc = idesc_bf16_mn(TL_R, n, false);
      for (int kb = 0; kb < TL_KB; ++kb) {
        const int s = item % TL_RING, r = item / TL_RING;
        ++item;
        if (!mbar_wait(&full[s], r & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t ad = sw128_desc(su32(a_base + kb * L::KB_A));
        const uint64_t bd = sw128_desc(su32(sRing + s * L::STAGE));
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_bf16(tmem + tm, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, (kb | k) != 0);
        umma_commit(&empty[s]);
      }
      umma_commit(done);
      return true;
    };
    bool ok = true;
    if (lane == 0) {
      ok = mbar_wait(ctx_full, 0, abort_flag);
      if (ok) ok = product(sCtx, TM_O, TL_EJ, o_done);
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
    cl_sync();   // A
    cl_sync();   // B: Y holds y1 in every rank
    if (lane == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (ok && !*abort_flag) ok = product(sY, TM_F1, TL_FJ, f1_done);
      if (ok && !*abort_flag) ok = mbar_wait(h_ready, 0, abort_flag);
      if (ok && !*abort_flag) {
        tc_fence_after();
        ok = product(sH, TM_F2, TL_E, f2_done);
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
    cl_sync();   // C
    cl_sync();   // D
    cl_sync();   // E: Y holds y2 in every rank
    if (lane == 0 && has_next && ok && !*abort_flag) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (!product(sY, TM_Q, TL_QJ, q_done)) *abort_flag = 1;
    }
    if (lane == 0) pdl_trigger();
    __syncwarp();
    cl_sync();   // F
  } else {
    // ------------------------------------------------------------ epilogues
    const int q = warp & 3, r = 32 * q + lane, row = m0 + r;
    const bool valid = row < M;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    // this rank's slices of the biases and LayerNorm weights, once, into
    // shared memory (read there by every epilogue below)
    float* par = reinterpret_cast<float*>(sm + L::OFF_PAR);
    float* p_bo = par;
    float* p_g1 = p_bo + TL_EJ;
    float* p_be1 = p_g1 + TL_EJ;
    float* p_b2 = p_be1 + TL_EJ;
    float* p_g2 = p_b2 + TL_EJ;
    float* p_be2 = p_g2 + TL_EJ;
    float* p_b1 = p_be2 + TL_EJ;   // TL_FJ
    float* p_bq = p_b1 + TL_FJ;    // TL_QJ
    static_assert(6 * TL_EJ + TL_FJ + TL_QJ == L::N_PAR, "parameter block layout");
    {
      const int t = threadIdx.x - 64;   // 0 .. 127
      for (int i = t; i < TL_EJ; i += 128) {
        p_bo[i] = a.bo[TL_EJ * j + i];
        p_g1[i] = a.ln1_g[TL_EJ * j + i];
        p_be1[i] = a.ln1_b[TL_EJ * j + i];
        p_b2[i] = a.b2[TL_EJ * j + i];
        p_g2[i] = a.ln2_g[TL_EJ * j + i];
        p_be2[i] = a.ln2_b[TL_EJ * j + i];
      }
      for (int i = t; i < TL_FJ; i += 128) p_b1[i] = a.b1[TL_FJ * j + i];
      if (has_next)
        for (int i = t; i < TL_QJ; i += 128) p_bq[i] = a.bq[TL_QJ * j + i];
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    pdl_wait();   // x and the outputs belong to the previous kernels' stream order
    auto wait_all = [&](uint64_t* bar) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, 0, abort_flag)) && !*abort_flag;
    };
    float y1[TL_EJ];
    // --- E1: O projection + bias + residual, LN1
    float v[TL_EJ];
    {   // the residual row is loaded while the O product is computed
      const float* xr = a.x + (int64_t)row * TL_E + TL_EJ * j;
#pragma unroll
      for (int c = 0; c < TL_EJ; c += 4) {
        const float4 xv = valid ? *reinterpret_cast<const float4*>(xr + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        v[c] = xv.x; v[c + 1] = xv.y; v[c + 2] = xv.z; v[c + 3] = xv.w;
      }
    }
    bool ok = wait_all(o_done);
    {
      if (ok) {
        tc_fence_after();
        uint32_t u[48];
        tmem_ld32(tmem + lane_base + TM_O, u);
        tmem_ld16(tmem + lane_base + TM_O + 32, u + 32);
#pragma unroll
        for (int c = 0; c < TL_EJ; ++c) v[c] += __uint_as_float(u[c]) + p_bo[c];
      } else {
#pragma unroll
        for (int c = 0; c < TL_EJ; ++c) v[c] = 0.f;
      }
      st1[r] = tl_local_stats(v);
      cl_sync();   // A
      float mean, rstd;
      tl_row_stats(st1, r, mean, rstd);
#pragma unroll
      for (int c = 0; c < TL_EJ; ++c) y1[c] = (v[c] - mean) * rstd * p_g1[c] + p_be1[c];
      if (!valid || !ok) {
#pragma unroll
        for (int c = 0; c < TL_EJ; ++c) y1[c] = 0.f;   // rows past M feed zeros to the products
      }
      tl_broadcast(su32(sY), r, j, y1);
      asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
      cl_sync();   // B
    }
    // --- E2: F1 + bias, ReLU, bf16 into H
    ok = ok && wait_all(f1_done);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < TL_FJ; c0 += 64) {
        uint32_t u[64];
        tmem_ld64(tmem + lane_base + TM_F1 + c0, u);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int col = c0 + 8 * g;
          const float4 b0 = *reinterpret_cast<const float4*>(p_b1 + col);
          const float4 b1 = *reinterpret_cast<const float4*>(p_b1 + col + 4);
          float h[8] = {__uint_as_float(u[8 * g]) + b0.x,     __uint_as_float(u[8 * g + 1]) + b0.y,
                        __uint_as_float(u[8 * g + 2]) + b0.z, __uint_as_float(u[8 * g + 3]) + b0.w,
                        __uint_as_float(u[8 * g + 4]) + b1.x, __uint_as_float(u[8 * g + 5]) + b1.y,
                        __uint_as_float(u[8 * g + 6]) + b1.z, __uint_as_float(u[8 * g + 7]) + b1.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) h[k] = fmaxf(h[k], 0.f);
          *reinterpret_cast<uint4*>(sH + (col >> 6) * L::KB_A + sw128_off(r, (col & 63) >> 3)) =
              make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]), pack_bf16(h[4], h[5]), pack_bf16(h[6], h[7]));
        }
      }
      tc_fence_before();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(h_ready);   // also on failure, so the MMA thread's wait ends
    // --- E3: F2 partials summed over the cluster, + b2 + y1, LN2
    ok = ok && wait_all(f2_done);
    // partial f32 [192][128] (column-major, row fastest): columns 0-95 in
    // the ctx buffer, 96-191 in H (both free once F2's MMAs completed)
    float* pst_lo = reinterpret_cast<float*>(sCtx);
    float* pst_hi = reinterpret_cast<float*>(sH);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < TL_E; c0 += 64) {
        uint32_t u[64];
        tmem_ld64(tmem + lane_base + TM_F2 + c0, u);
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const int c = c0 + k;
          (c < 96 ? pst_lo + c * TL_R : pst_hi + (c - 96) * TL_R)[r] = __uint_as_float(u[k]);
        }
      }
    }
    cl_sync();   // C
    {
#pragma unroll
      for (int c = 0; c < TL_EJ; ++c) v[c] = 0.f;
      if (ok) {
#pragma unroll 1
        for (int rk = 0; rk < TL_C; rk += 2) {   // fixed rank order: the sum does not depend on timing
          float t0[TL_EJ], t1[TL_EJ];
#pragma unroll
          for (int c = 0; c < TL_EJ; ++c) {   // two ranks' loads in flight before the sums
            const int col = TL_EJ * j + c;
            const uint32_t p = su32((col < 96 ? pst_lo + col * TL_R : pst_hi + (col - 96) * TL_R) + r);
            t0[c] = ld_cluster_f32(cl_map(p, (uint32_t)rk));
            t1[c] = ld_cluster_f32(cl_map(p, (uint32_t)rk + 1));
          }
#pragma unroll
          for (int c = 0; c < TL_EJ; ++c) v[c] = (v[c] + t0[c]) + t1[c];
        }
#pragma unroll
        for (int c = 0; c < TL_EJ; ++c) v[c] = y1[c] + (v[c] + p_b2[c]);
      }
      st2[r] = tl_local_stats(v);
      cl_sync();   // D
      float mean, rstd;
      tl_row_stats(st2, r, mean, rstd);
      float y2[TL_EJ];
#pragma unroll
      for (int c = 0; c < TL_EJ; ++c) y2[c] = (v[c] - mean) * rstd * p_g2[c] + p_be2[c];
      if (ok && valid) {
        float* xr = a.x + (int64_t)row * TL_E + TL_EJ * j;
#pragma unroll
        for (int c = 0; c < TL_EJ; c += 4) *reinterpret_cast<float4*>(xr + c) = make_float4(y2[c], y2[c + 1], y2[c + 2], y2[c + 3]);
        if (!has_next) {   // last layer: the head's input as bf16
          bf16* hr = a.h + (int64_t)row * TL_E + TL_EJ * j;
#pragma unroll
          for (int c = 0; c < TL_EJ; c += 8)
            *reinterpret_cast<uint4*>(hr + c) = make_uint4(pack_bf16(y2[c], y2[c + 1]), pack_bf16(y2[c + 2], y2[c + 3]),
                                                           pack_bf16(y2[c + 4], y2[c + 5]), pack_bf16(y2[c + 6], y2[c + 7]));
        }
      }
      if (has_next) {
        if (!valid || !ok) {
#pragma unroll
          for (int c = 0; c < TL_EJ; ++c) y2[c] = 0.f;
        }
        tl_broadcast(su32(sY), r, j, y2);
        asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
      }
      cl_sync();   // E
    }
    // --- E4: next layer's Q | K | V columns of this rank + bias, bf16
    if (has_next && ok && wait_all(q_done)) {
      tc_fence_after();
      bf16* qr = a.qkv + (int64_t)row * (3 * TL_E) + TL_QJ * j;
      const float* bq = p_bq;
      auto store16 = [&](const uint32_t* uu, int c0) {
        float f[16];
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
          const float4 bv = *reinterpret_cast<const float4*>(bq + c0 + k);
          f[k] = __uint_as_float(uu[k]) + bv.x;
          f[k + 1] = __uint_as_float(uu[k + 1]) + bv.y;
          f[k + 2] = __uint_as_float(uu[k + 2]) + bv.z;
          f[k + 3] = __uint_as_float(uu[k + 3]) + bv.w;
        }
        if (valid) {
          uint4* d = reinterpret_cast<uint4*>(qr + c0);
          d[0] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
          d[1] = make_uint4(pack_bf16(f[8], f[9]), pack_bf16(f[10], f[11]), pack_bf16(f[12], f[13]),
                            pack_bf16(f[14], f[15]));
        }
      };
      {
        uint32_t u[64];
        tmem_ld64(tmem + lane_base + TM_Q, u);
#pragma unroll
        for (int k = 0; k < 64; k += 16) store16(u + k, k);
      }
      {
        uint32_t u[64];
        tmem_ld64(tmem + lane_base + TM_Q + 64, u);
#pragma unroll
        for (int k = 0; k < 64; k += 16) store16(u + k, 64 + k);
      }
      {
        uint32_t u[16];
        tmem_ld16(tmem + lane_base + TM_Q + 128, u);
        store16(u, 128);
      }
    } else if (has_next && !ok) {
      *abort_flag = 1;
    }
    if (!ok) *abort_flag = 1;
    cl_sync();   // F: peers are done with this CTA's shared memory
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u) : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag) set_err(err, ERR_TIMEOUT);
}

int g_tl_clusters = 0;   // co-resident clusters of tf_layer_kernel

}  // namespace

cudaError_t launch_tf_layer(const bf16* ctx, const TfLayerW& w, const TfLayerW* next, float* x, bf16* qkv, bf16* h,
                            int M, int* err, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  if (!ctx || !x || !w.wo || !w.w1 || !w.w2 || (next ? (!qkv || !next->wqkv) : !h)) return cudaErrorInvalidValue;
  CUtensorMap t_ctx, t_wo, t_w1, t_w2, t_wq;
  cudaError_t r = make_bf16_map_sw128(&t_ctx, ctx, M, TL_E, TL_E, TL_R);
  if (r == cudaSuccess) r = make_bf16_map_sw128(&t_wo, w.wo, TL_E, TL_E, TL_E, TL_EJ);
  if (r == cudaSuccess) r = make_bf16_map_sw128(&t_w1, w.w1, TL_F, TL_E, TL_E, TL_FJ);
  if (r == cudaSuccess) r = make_bf16_map_sw128(&t_w2, w.w2, TL_E, TL_F, TL_F, TL_E);
  if (r == cudaSuccess)
    r = next ? make_bf16_map_sw128(&t_wq, next->wqkv, 3 * TL_E, TL_E, TL_E, TL_QJ) : make_bf16_map_sw128(&t_wq, w.wo, TL_E, TL_E, TL_E, TL_QJ);
  if (r != cudaSuccess) return r;
  TfLayerArgs a{};
  a.x = x;
  a.bo = w.bo;
  a.ln1_g = w.ln1_g;
  a.ln1_b = w.ln1_b;
  a.b1 = w.b1;
  a.b2 = w.b2;
  a.ln2_g = w.ln2_g;
  a.ln2_b = w.ln2_b;
  a.bq = next ? next->bqkv : nullptr;
  a.qkv = qkv;
  a.h = h;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(TL_C, (M + TL_R - 1) / TL_R, 1);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = TlSmem::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = TL_C;
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
  CK_LAUNCH(cudaLaunchKernelEx(&cfg, tf_layer_kernel, t_ctx, t_wo, t_w1, t_w2, t_wq, a, M, err));
  return cudaGetLastError();
}

int tf_layer_max_rows() { return g_tl_clusters * TL_R; }

cudaError_t tf_layer_init_attributes() {
  cudaError_t r = cudaFuncSetAttribute(tf_layer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TlSmem::SMEM);
  if (r != cudaSuccess) return r;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(TL_C, 1, 1);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = TlSmem::SMEM;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeClusterDimension;
  at.val.clusterDim.x = TL_C;
  at.val.clusterDim.y = 1;
  at.val.clusterDim.z = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  int n = 0;
  g_tl_clusters = cudaOccupancyMaxActiveClusters(&n, tf_layer_kernel, &cfg) == cudaSuccess ? n : 0;
  cudaGetLastError();
  return cudaSuccess;
}

}  // namespace sf
