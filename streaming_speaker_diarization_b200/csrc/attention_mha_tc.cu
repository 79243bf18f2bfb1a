// Plain multi-head self-attention of the Transformer encoder on the
// Blackwell tensor cores (tcgen05 MMA with TMEM accumulators, TMA loads),
// bf16 operands, fp32 scores and softmax: d_model 192, 8 heads of 24
// ("Streaming Sortformer Diarizer" model card: 18-layer Transformer encoder
// after the FastConformer):
//   out_i = sum_j softmax_j(q_i . k_j / sqrt(24)) v_j   over the keys of i's sequence.
//
// One CTA = 128 query rows [i0, i0 + 128) of one sequence x one head.  The
// head dimension is carried as 64 so that every operand has the 128-byte
// rows of the swizzle the tensor cores read: Q is written by the softmax
// warps with dims 24-63 set to zero, so the 40 neighbouring columns that the
// 64-column TMA boxes of K bring along add nothing to Q K^T; the P V product
// yields 64 columns of which the first 24 are the head's output.  Per
// 64-key tile [j0, j0 + 64):
//   S   = Q K^T   M 128, N 64, K 64   TMEM columns [0, 64)
//   O_t = P V     M 128, N 64, K 64   TMEM columns 64 + 64 (t % 2)
// Warps: 0 loads K and V (three-stage ring) with TMA; 1 issues the MMAs (one
// thread); 2-5 run the softmax, thread = query row = TMEM lane: online
// softmax in the exp2 domain (scale folded in), P to shared memory as bf16,
// O accumulated in registers.  Shared memory ~97 KB and 256 TMEM columns, so
// two CTAs share an SM.  Every wait is bounded: a wait that runs out raises
// ERR_TIMEOUT, the CTA drains its own copies and frees its TMEM.
// When the (query tile, head) units are fewer than the SMs (one long
// sequence), each unit's key tiles are split over a cluster of 2 or 4 CTAs:
// each CTA leaves the softmax state (O, m, l) of its key range in its own
// shared memory and the cluster's rank 0 merges them in rank order over
// distributed shared memory.
#include "common.cuh"
#include "layers.h"
#include "tcgen05.cuh"
#include "attn_common.cuh"

namespace sf {
namespace {

constexpr int MQ = 128;     // query rows per CTA
constexpr int MK = 64;      // keys per tile
constexpr int MHP = 64;     // head dim as carried (zero-padded in Q when the head is narrower)
constexpr int MNB = 3;      // K / V ring stages

struct MhaTc {
  static constexpr int Q_BYTES = MQ * MHP * 2;     // 16 KB
  static constexpr int K_BYTES = MK * MHP * 2;     //  8 KB
  static constexpr int V_BYTES = MK * MHP * 2;     //  8 KB (MN-major B operand)
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int P_BYTES = MQ * MK * 2;      // 16 KB
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = Q_BYTES;
  static constexpr int OFF_P = OFF_RING + MNB * STAGE;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  static_assert(STAGE % 1024 == 0 && OFF_P % 1024 == 0 && OFF_RING % 1024 == 0, "swizzled tiles 1024-aligned");
  // key split: row r's partial state O[head dim], m, l (+2 pad, 16-byte
  // rows) goes to the K/V ring once the last P.V product has completed
  static_assert(MQ * (MHP + 4) * 4 <= MNB * STAGE, "partials fit in the ring");
};

}  // namespace

// MHD: the head dimension (24 for the Sortformer Transformer, 64 for the
// Nemotron-3 variant); E = 8 x MHD is a runtime argument.
template <int MHD>
__global__ void __launch_bounds__(192, 2) attn_mha_tc_kernel(const __grid_constant__ CUtensorMap t_qkv,
                                                             const bf16* __restrict__ qkv, int E,
                                                             bf16* __restrict__ ctx,
                                                             const SeqTable* __restrict__ seq, int* err,
                                                             int ks) {
  using L = MhaTc;
  extern __shared__ uint8_t mh_smem[];
  uint8_t* sm = mh_smem + ((1024 - (su32(mh_smem) & 1023)) & 1023);
  uint8_t* sQ = sm + L::OFF_Q;
  uint8_t* sRing = sm + L::OFF_RING;
  uint8_t* sP = sm + L::OFF_P;
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);   // [MNB]
  uint64_t* kv_empty = kv_full + MNB;                                  // [MNB]
  uint64_t* s_full = kv_empty + MNB;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;                                       // [2]
  uint64_t* pv_full = p_full + 2;                                      // [2]
  uint64_t* q_ready = pv_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int s = seq_of_tile2(seq, blockIdx.x);
  const int sb = seq->off[s], S = seq->off[s + 1] - sb;
  const int i0 = (blockIdx.x - seq->tile2_off[s]) * MQ;
  const int T = (S + MK - 1) / MK;   // key tiles of the sequence
  // key split: this CTA takes key tiles [t0, t0 + Tl) (blockIdx.z of ks);
  // ring stages and barrier phases count local tiles
  const int t0 = (int)((int64_t)T * blockIdx.z / ks);
  const int Tl = (int)((int64_t)T * (blockIdx.z + 1) / ks) - t0;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&t_qkv)) : "memory");
    for (int b = 0; b < MNB; ++b) {
      mbar_init(&kv_full[b], 1);
      mbar_init(&kv_empty[b], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&p_full[b], 4);
      mbar_init(&pv_full[b], 1);
    }
    mbar_init(q_ready, 4);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"(256u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  SF_PDL_ENTRY();

  if (warp == 0) {
    // ---------------------------------------------------------------- loads
    if (lane == 0) {
      int t = 0;
      for (; t < Tl && !*abort_flag; ++t) {
        const int b = t % MNB, r = t / MNB, j0 = (t0 + t) * MK;
        if (!mbar_wait(&kv_empty[b], (r & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        uint8_t* st = sRing + b * L::STAGE;
        mbar_expect_tx(&kv_full[b], L::STAGE);
        tma_load_2d(st, &t_qkv, &kv_full[b], E + h * MHD, sb + j0);                    // K rows j0 .. (+40 cols)
        tma_load_2d(st + L::K_BYTES, &t_qkv, &kv_full[b], 2 * E + h * MHD, sb + j0);   // V rows j0 .. (+40 cols)
      }
      if (*abort_flag) {   // let this CTA's own loads land before its shared memory is released
        for (int k = t - MNB > 0 ? t - MNB : 0; k < t; ++k) {
          const long long c0 = clock64();
          while (!mbar_try_wait(&kv_full[k % MNB], (k / MNB) & 1) && clock64() - c0 < WAIT_CYCLES) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMAs
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_mn(MQ, MK, false);
      constexpr uint32_t id_pv = idesc_bf16_mn(MQ, MHP, true);
      const uint64_t dq = sw128_desc(su32(sQ));
      bool ok = mbar_wait(q_ready, 0, abort_flag);
      auto issue_pv = [&](int t) -> bool {
        const int pb = t & 1, b = t % MNB;
        if (!mbar_wait(&p_full[pb], (t >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dp = sw128_desc(su32(sP + pb * L::P_BYTES));
        const uint64_t dv = sw128_desc_mn(su32(sRing + b * L::STAGE + L::K_BYTES));
#pragma unroll
        for (int k = 0; k < MK / 16; ++k)   // keys 16 at a time: +32 bytes in P, +16 rows (2048 bytes) in V
          umma_bf16(tmem + 64 + 64 * pb, dp + (uint64_t)(2 * k), dv + (uint64_t)(128 * k), id_pv, k != 0);
        umma_commit(&pv_full[pb]);
        umma_commit(&kv_empty[b]);   // K and V of tile t are no longer read
        return true;
      };
      for (int t = 0; ok && t < Tl; ++t) {
        const int b = t % MNB;
        if (!mbar_wait(&kv_full[b], (t / MNB) & 1, abort_flag)) { ok = false; break; }
        if (t > 0 && !mbar_wait(s_free, (t - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dk = sw128_desc(su32(sRing + b * L::STAGE));
#pragma unroll
        for (int k = 0; k < MHP / 16; ++k) umma_bf16(tmem, dq + (uint64_t)(2 * k), dk + (uint64_t)(2 * k), id_s, k != 0);
        umma_commit(s_full);
        if (t > 0 && !issue_pv(t - 1)) { ok = false; break; }
      }
      if (ok && Tl > 0) ok = issue_pv(Tl - 1);
      if (!ok) *abort_flag = 1;
      pdl_trigger();   // the next kernel may launch and set up; it waits for this grid's memory
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int q = warp & 3;                        // TMEM lane quarter of this warp
    const int r = 32 * q + lane;                   // query row in the tile = TMEM lane
    const int i = i0 + r;
    const bool row_ok = i < S;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    // Q row (24 dims, rounded as loaded) and 40 zero dims into the swizzled A tile
    {
      const bf16* qrow = qkv + (int64_t)(sb + (row_ok ? i : 0)) * (3 * E) + h * MHD;
#pragma unroll
      for (int c = 0; c < MHP / 8; ++c) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row_ok && c < MHD / 8) {   // 24 or 64 dims = 3 or 8 16-byte chunks, 16-byte aligned
          v = *reinterpret_cast<const uint4*>(qrow + 8 * c);
        }
        *reinterpret_cast<uint4*>(sQ + sw128_off(r, c)) = v;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }

    static_assert(MHD == 24 || MHD == 64, "head dims of the two Transformers");
    constexpr float inv_sqrt_hd = MHD == 64 ? 0.125f : 0.20412414523193151f;
    const float sl2 = 1.4426950408889634f * inv_sqrt_hd;   // log2(e) / sqrt(head dim)
    float m_run = -INFINITY, l_run = 0.f;
    float o[MHD];
#pragma unroll
    for (int d = 0; d < MHD; ++d) o[d] = 0.f;
    bool ok = true;
    for (int t = 0; t < Tl; ++t) {
      const int j0 = (t0 + t) * MK;
      if (!warp_wait(s_full, t & 1)) { ok = false; break; }
      tc_fence_after();
      float sc[MK];
      {
        uint32_t v[MK];
        tmem_ld64(tmem + lane_base, v);
#pragma unroll
        for (int k = 0; k < MK; ++k) sc[k] = __uint_as_float(v[k]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);   // S of tile t read out of TMEM
      // the running maximum over the raw scores (the scale is positive), then
      // p = 2^(s sl2 - m) with one packed FMA per two keys
      const bool full = j0 + MK <= S;
      if (!full) {   // last tile: keys past the sequence end get no weight
#pragma unroll
        for (int c = 0; c < MK; ++c)
          if (j0 + c >= S) sc[c] = -INFINITY;
      }
      // row maximum and sum as 8 / 4 independent partial chains (one warp per
      // scheduler: a single serial chain would expose every latency)
      float mp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mp[k] = sc[k];
#pragma unroll
      for (int c = 8; c < MK; ++c) mp[c & 7] = fmaxf(mp[c & 7], sc[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      const float m_new = fmaxf(m_run, mx * sl2);   // finite: key j0 < S (every local tile starts inside S)
      const float alpha = ex2_approx(m_run - m_new);
      const float2 s2 = make_float2(sl2, sl2), nm2 = make_float2(-m_new, -m_new);
      float2 ps2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) ps2[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < MK; c += 2) {
        const float2 x = __ffma2_rn(make_float2(sc[c], sc[c + 1]), s2, nm2);
        float2 pe;
        pe.x = ex2_approx(x.x);
        pe.y = ex2_approx(x.y);
        sc[c] = pe.x;
        sc[c + 1] = pe.y;
        ps2[(c >> 1) & 3] = __fadd2_rn(ps2[(c >> 1) & 3], pe);
      }
      const float2 pt2 = __fadd2_rn(__fadd2_rn(ps2[0], ps2[1]), __fadd2_rn(ps2[2], ps2[3]));
      l_run = l_run * alpha + (pt2.x + pt2.y);
      m_run = m_new;
      // P row as bf16 into the swizzled A tile of P.V (buffer t % 2; its
      // previous tile's P.V completed before iteration t - 1 read its result)
      uint8_t* pt = sP + (t & 1) * L::P_BYTES;
#pragma unroll
      for (int ch = 0; ch < MK / 8; ++ch) {
        uint32_t w4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 hp = __floats2bfloat162_rn(sc[8 * ch + 2 * k], sc[8 * ch + 2 * k + 1]);
          w4[k] = *reinterpret_cast<uint32_t*>(&hp);
        }
        *reinterpret_cast<uint4*>(pt + sw128_off(r, ch)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t & 1]);
      // O (relative to m_(t-1)) += P_(t-1) V_(t-1), then rescale to m_t
      if (t > 0) {
        const int pb = (t - 1) & 1;
        if (!warp_wait(&pv_full[pb], ((t - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[64];
        if (MHD <= 32) tmem_ld32(tmem + lane_base + (uint32_t)(64 + 64 * pb), v);   // the head's columns
        else tmem_ld64(tmem + lane_base + (uint32_t)(64 + 64 * pb), v);
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int k = 0; k < MHD; k += 2) {
          const float2 t = __fmul2_rn(__fadd2_rn(make_float2(o[k], o[k + 1]),
                                                 make_float2(__uint_as_float(v[k]), __uint_as_float(v[k + 1]))),
                                      a2);
          o[k] = t.x;
          o[k + 1] = t.y;
        }
      }
    }
    if (ok && Tl > 0) {
      const int pb = (Tl - 1) & 1;
      if (warp_wait(&pv_full[pb], ((Tl - 1) >> 1) & 1)) {
        tc_fence_after();
        uint32_t v[64];
        if (MHD <= 32) tmem_ld32(tmem + lane_base + (uint32_t)(64 + 64 * pb), v);
        else tmem_ld64(tmem + lane_base + (uint32_t)(64 + 64 * pb), v);
#pragma unroll
        for (int k = 0; k < MHD; ++k) o[k] += __uint_as_float(v[k]);
      } else {
        ok = false;
      }
    }
    auto store_row = [&](const float* ov, float l) {
      const float inv = 1.f / l;
      uint4* dst = reinterpret_cast<uint4*>(ctx + (int64_t)(sb + i) * E + h * MHD);   // 2 x MHD h bytes: 16-byte aligned
#pragma unroll
      for (int c = 0; c < MHD / 8; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 ho = __floats2bfloat162_rn(ov[8 * c + 2 * k] * inv, ov[8 * c + 2 * k + 1] * inv);
          w4[k] = *reinterpret_cast<uint32_t*>(&ho);
        }
        dst[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    };
    if (!ok) {
      *abort_flag = 1;
    } else if (ks == 1) {
      if (row_ok) store_row(o, l_run);
    } else {
      // Key split: (O, m, l) of this CTA's key range into row r's slot of
      // the K/V ring.  Every K/V tile landed and was consumed: this warp saw
      // the last P.V product complete, which follows every product that read
      // the ring.  A CTA with no key tiles leaves m = -inf, l = 0 (weight 0
      // in the merge).
      constexpr int PSTR = MHD + 4;
      float* mine = reinterpret_cast<float*>(sRing) + r * PSTR;
#pragma unroll
      for (int d = 0; d < MHD; d += 4)
        *reinterpret_cast<float4*>(mine + d) = make_float4(o[d], o[d + 1], o[d + 2], o[d + 3]);
      mine[MHD] = m_run;
      mine[MHD + 1] = l_run;
    }
  }
  if (ks > 1) {
    // every thread of every CTA of the cluster meets here (also after a failed wait)
    __syncthreads();
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    uint32_t crank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(crank));
    if (crank == 0 && warp >= 2 && !*abort_flag) {
      const int q = warp & 3, r = 32 * q + lane, i = i0 + r;
      constexpr int PSTR = MHD + 4;
      const uint32_t row_addr = su32(reinterpret_cast<float*>(sRing) + r * PSTR);
      float mz[4], lz[4];
#pragma unroll
      for (int zz = 0; zz < 4; ++zz) {
        mz[zz] = -INFINITY;
        lz[zz] = 0.f;
        if (zz < ks) {
          uint32_t a;
          asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(row_addr + 4u * MHD), "r"((uint32_t)zz));
          asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(mz[zz]), "=f"(lz[zz]) : "r"(a) : "memory");
        }
      }
      const float m = fmaxf(fmaxf(mz[0], mz[1]), fmaxf(mz[2], mz[3]));   // finite: some rank has a key tile
      float acc[MHD], l = 0.f;
#pragma unroll
      for (int d = 0; d < MHD; ++d) acc[d] = 0.f;
#pragma unroll
      for (int zz = 0; zz < 4; ++zz) {
        if (zz >= ks) break;
        const float wz = ex2_approx(mz[zz] - m);   // an empty key range has m = -inf: weight 0
        l += wz * lz[zz];
#pragma unroll
        for (int d = 0; d < MHD; d += 4) {
          uint32_t a;
          asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(row_addr + 4u * d), "r"((uint32_t)zz));
          float4 v4;
          asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(v4.x), "=f"(v4.y), "=f"(v4.z), "=f"(v4.w)
                       : "r"(a)
                       : "memory");
          acc[d] += wz * v4.x; acc[d + 1] += wz * v4.y; acc[d + 2] += wz * v4.z; acc[d + 3] += wz * v4.w;
        }
      }
      if (i < S) {
        const float inv = 1.f / l;
        uint4* dst = reinterpret_cast<uint4*>(ctx + (int64_t)(sb + i) * E + h * MHD);
#pragma unroll
        for (int c = 0; c < MHD / 8; ++c) {
          uint32_t w4[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 ho = __floats2bfloat162_rn(acc[8 * c + 2 * k] * inv, acc[8 * c + 2 * k + 1] * inv);
            w4[k] = *reinterpret_cast<uint32_t*>(&ho);
          }
          dst[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
    // no CTA leaves while rank 0 may still read its shared memory
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256u) : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag) set_err(err, ERR_TIMEOUT);
}

namespace {
int g_mha_sms = 148;
int g_mha_clusters[2][3] = {{1, 0, 0}, {1, 0, 0}};   // [head dim 24 / 64]: co-resident clusters of 1, 2, 4 CTAs

template <int MHD>
cudaError_t launch_mha_tc_t(const bf16* qkv, bf16* ctx, const SeqTable* seq, int n_tiles2, int M, int max_len, int E,
                            int* err, cudaStream_t st) {
  if (M <= 0 || n_tiles2 <= 0) return cudaSuccess;
  if (E != 8 * MHD) return cudaErrorInvalidValue;
  CUtensorMap t_qkv;
  cudaError_t r = make_bf16_map_sw128(&t_qkv, qkv, M, 3 * E, 3 * E, MK);
  if (r != cudaSuccess) return r;
  // fewer (query tile, head) units than the two CTAs per SM hold: split
  // each unit's keys over a cluster of 2 or 4 CTAs (no more splits than key
  // tiles of the longest sequence), but only as far as every cluster is
  // co-resident (one wave: a second wave would double the time)
  const int* cl = g_mha_clusters[MHD == 64 ? 1 : 0];
  const int units = n_tiles2 * 8;
  int ks = 1;
  if (units < 2 * g_mha_sms) {
    const int want = 2 * g_mha_sms / units, tmax = (max_len + MK - 1) / MK;
    if (want >= 4 && tmax >= 4 && units <= cl[2]) ks = 4;
    else if (want >= 2 && tmax >= 2 && units <= cl[1]) ks = 2;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles2, 8, ks);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = MhaTc::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = 1;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = ks;
  ++na;
  if (g_launch_pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  CK_LAUNCH(cudaLaunchKernelEx(&cfg, attn_mha_tc_kernel<MHD>, t_qkv, (const bf16*)qkv, E, ctx, seq, err, ks));
  return cudaGetLastError();
}

template <int MHD>
cudaError_t init_mha_tc() {
  cudaError_t r =
      cudaFuncSetAttribute(attn_mha_tc_kernel<MHD>, cudaFuncAttributeMaxDynamicSharedMemorySize, MhaTc::SMEM);
  if (r != cudaSuccess) return r;
  for (int j = 1; j < 3; ++j) {   // can clusters of 2 and 4 CTAs be scheduled at all, and how many at once?
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1 << j);
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = MhaTc::SMEM;
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeClusterDimension;
    a.val.clusterDim.x = 1;
    a.val.clusterDim.y = 1;
    a.val.clusterDim.z = 1 << j;
    cfg.attrs = &a;
    cfg.numAttrs = 1;
    int n_cl = 0;
    g_mha_clusters[MHD == 64 ? 1 : 0][j] =
        cudaOccupancyMaxActiveClusters(&n_cl, attn_mha_tc_kernel<MHD>, &cfg) == cudaSuccess ? n_cl : 0;
    cudaGetLastError();
  }
  return cudaSuccess;
}
}  // namespace

cudaError_t launch_mha_tc(const bf16* qkv, bf16* ctx, const SeqTable* seq, int n_tiles2, int M, int max_len,
                          int* err, cudaStream_t st) {
  return launch_mha_tc_t<24>(qkv, ctx, seq, n_tiles2, M, max_len, 192, err, st);
}

cudaError_t launch_mha_tc_hd64(const bf16* qkv, bf16* ctx, const SeqTable* seq, int n_tiles2, int M, int max_len,
                               int E, int* err, cudaStream_t st) {
  return launch_mha_tc_t<64>(qkv, ctx, seq, n_tiles2, M, max_len, E, err, st);
}

cudaError_t attention_mha_tc_init_attributes() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
      n > 0)
    g_mha_sms = n;
  cudaError_t r = init_mha_tc<24>();
  if (r != cudaSuccess) return r;
  return init_mha_tc<64>();
}

}  // namespace sf
