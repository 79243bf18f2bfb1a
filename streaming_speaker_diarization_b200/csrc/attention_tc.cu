// Relative-position MHSA on the Blackwell tensor cores (tcgen05 MMA with TMEM
// accumulators, TMA loads), bf16 operands, fp32 scores and softmax, head dim
// 64.  Same arithmetic as the FastConformer attention of the "Streaming
// Sortformer Diarizer" model (relative-position MHSA):
//   score(i, j) = ((q_i + u) . k_j + (q_i + v) . p_(i-j)) / sqrt(64),
//   out_i = sum_j softmax_j(score(i, .)) v_j   over the keys of i's sequence.
//
// One CTA = 128 query rows [i0, i0 + 128) of one sequence x one head.  Per
// 64-key tile [j0, j0 + 64):
//   AC = (Q+u) K^T    M 128, N  64, K 64   TMEM columns [0, 64)
//   BD = (Q+v) Pw^T   M 128, N 192, K 64   TMEM columns [64, 256)
//        Pw = position-table rows for distances i0 - j0 - 63 .. i0 - j0 + 128,
//        i.e. every i - j of the tile (row r, key c: BD column r - c + 63),
//        as three 64-row blocks; consecutive key tiles share two of them, so
//        each tile loads one new block (three N = 64 MMAs, one per block)
//   O_t = P V         M 128, N  64, K 64   TMEM columns 256 + 64 (t % 2)
// Warps: 0 loads K and V (three-stage ring) and the position blocks (five-
// slot ring) with TMA; 1 issues the MMAs (one thread); 2-5 run the softmax,
// thread = query row = TMEM lane.  A
// warp's 32 rows need a 96-column band of BD; it is staged in shared memory
// (row stride 100 floats: conflict-free by rows and along the diagonal) and
// read back at column r - c + 63.  The softmax is online in the exp2 domain
// (scale folded in); P goes to shared memory as bf16 (the A operand of P.V);
// O accumulates in registers, rescaled before each tile's P.V is added.
// With fewer (query tile, head) units than SMs (one long sequence), each
// unit's key tiles are split over a cluster of 2 or 4 CTAs; each keeps its
// softmax state (O, m, l) in shared memory and the cluster's rank 0 merges
// them in rank order over distributed shared memory.
// Every wait is bounded: a wait that runs out raises ERR_TIMEOUT, the CTA
// drains its own copies and frees its TMEM.
#include "common.cuh"
#include "layers.h"
#include "tcgen05.cuh"
#include "attn_common.cuh"

namespace sf {
namespace {

constexpr int AQ = 128;      // query rows per CTA
constexpr int AK = 64;       // keys per tile
constexpr int AHD = 64;      // head dim
constexpr int ANB = 3;       // K / V ring stages
constexpr int NPW = ANB + 2; // 64-row position blocks held (tile t reads blocks t - 2 .. t)
constexpr int BD_LD = 100;   // staged BD row stride (floats)
constexpr int PSTR = AHD + 4; // key-split partial row: O[64], m, l, 2 pad (16-byte aligned rows)

struct AttTc {
  static constexpr int Q_BYTES = AQ * AHD * 2;      // 16 KB, K-major, 128-byte swizzle
  static constexpr int K_BYTES = AK * AHD * 2;      //  8 KB
  static constexpr int V_BYTES = AK * AHD * 2;      //  8 KB (MN-major B operand)
  static constexpr int PB_BYTES = 64 * AHD * 2;     //  8 KB position block (one of the 192 distances of a tile)
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int P_BYTES = AQ * AK * 2;       // 16 KB
  static constexpr int OFF_QU = 0;
  static constexpr int OFF_QV = Q_BYTES;
  static constexpr int OFF_RING = 2 * Q_BYTES;
  static constexpr int OFF_PW = OFF_RING + ANB * STAGE;
  static constexpr int OFF_P = OFF_PW + NPW * PB_BYTES;
  static constexpr int OFF_BD = OFF_P + 2 * P_BYTES;
  static constexpr int BD_BYTES = 4 * 32 * BD_LD * 4;
  static constexpr int OFF_BAR = OFF_BD + BD_BYTES;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  static_assert(STAGE % 1024 == 0 && OFF_P % 1024 == 0 && OFF_PW % 1024 == 0, "swizzled tiles 1024-aligned");
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

}  // namespace

__global__ void __launch_bounds__(192, 1) attn_relpos_tc_kernel(const __grid_constant__ CUtensorMap t_qkv,
                                                                const __grid_constant__ CUtensorMap t_pos,
                                                                const bf16* __restrict__ qkv, int D, int R,
                                                                const float* __restrict__ u,
                                                                const float* __restrict__ vb, bf16* __restrict__ ctx,
                                                                const SeqTable* __restrict__ seq, int* err, int ks) {
  using L = AttTc;
  extern __shared__ uint8_t at_smem[];
  uint8_t* sm = at_smem + ((1024 - (su32(at_smem) & 1023)) & 1023);
  uint8_t* sQu = sm + L::OFF_QU;
  uint8_t* sQv = sm + L::OFF_QV;
  uint8_t* sRing = sm + L::OFF_RING;
  uint8_t* sP = sm + L::OFF_P;
  float* sBD = reinterpret_cast<float*>(sm + L::OFF_BD);
  uint8_t* sPw = sm + L::OFF_PW;
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);   // [ANB] K, V (+ new position blocks)
  uint64_t* kv_empty = kv_full + ANB;                                  // [ANB]
  uint64_t* pw_empty = kv_empty + ANB;                                 // [NPW]
  uint64_t* s_full = pw_empty + NPW;
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
  const int i0 = (blockIdx.x - seq->tile2_off[s]) * AQ;
  const int T = (S + AK - 1) / AK;   // key tiles of the sequence
  // key split: this CTA takes key tiles [t0, t0 + Tl) (blockIdx.z of ks);
  // ring stages and barrier phases count local tiles tt = t - t0
  const int t0 = (int)((int64_t)T * blockIdx.z / ks);
  const int Tl = (int)((int64_t)T * (blockIdx.z + 1) / ks) - t0;

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&t_qkv)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&t_pos)) : "memory");
    for (int b = 0; b < ANB; ++b) {
      mbar_init(&kv_full[b], 1);
      mbar_init(&kv_empty[b], 1);
    }
    for (int b = 0; b < NPW; ++b) mbar_init(&pw_empty[b], 1);
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
                 "r"(512u)
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
      int tt = 0;
      for (; tt < Tl && !*abort_flag; ++tt) {
        const int t = t0 + tt, b = tt % ANB, r = tt / ANB, j0 = t * AK;
        if (!mbar_wait(&kv_empty[b], (r & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        // position block k = distances i0 - 64k - 63 .. i0 - 64k; local index
        // lb = k - t0 + 2, slot lb % NPW; the first tile brings blocks
        // t0 - 2 .. t0, later tiles block t
        const int lb_lo = tt == 0 ? 0 : tt + 2, lb_hi = tt + 2;
        bool got = true;
        for (int lb = lb_lo; lb <= lb_hi && got; ++lb)
          got = mbar_wait(&pw_empty[lb % NPW], ((lb / NPW) & 1) ^ 1, abort_flag);
        if (!got) {
          *abort_flag = 1;
          break;
        }
        uint8_t* st = sRing + b * L::STAGE;
        mbar_expect_tx(&kv_full[b], L::STAGE + (lb_hi - lb_lo + 1) * L::PB_BYTES);
        tma_load_2d(st, &t_qkv, &kv_full[b], D + h * AHD, sb + j0);                       // K rows j0 ..
        tma_load_2d(st + L::K_BYTES, &t_qkv, &kv_full[b], 2 * D + h * AHD, sb + j0);      // V rows j0 ..
        for (int lb = lb_lo; lb <= lb_hi; ++lb)
          tma_load_2d(sPw + (lb % NPW) * L::PB_BYTES, &t_pos, &kv_full[b], h * AHD,
                      i0 - 64 * (lb + t0 - 2) - (AK - 1) + R - 1);
      }
      if (*abort_flag) {   // let this CTA's own loads land before its shared memory is released
        for (int k = tt - ANB > 0 ? tt - ANB : 0; k < tt; ++k) {
          const long long c0 = clock64();
          while (!mbar_try_wait(&kv_full[k % ANB], (k / ANB) & 1) && clock64() - c0 < WAIT_CYCLES) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMAs
    if (lane == 0 && Tl > 0) {
      constexpr uint32_t id_s = idesc_bf16_mn(AQ, AK, false);
      constexpr uint32_t id_bd = idesc_bf16_mn(AQ, 64, false);
      constexpr uint32_t id_pv = idesc_bf16_mn(AQ, AHD, true);
      const uint32_t tm_s = tmem, tm_bd = tmem + AK;
      const uint64_t dqu = sw128_desc(su32(sQu)), dqv = sw128_desc(su32(sQv));
      bool ok = mbar_wait(q_ready, 0, abort_flag);
      auto issue_pv = [&](int tt) -> bool {
        const int pb = tt & 1, b = tt % ANB;
        if (!mbar_wait(&p_full[pb], (tt >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dp = sw128_desc(su32(sP + pb * L::P_BYTES));
        const uint64_t dv = sw128_desc_mn(su32(sRing + b * L::STAGE + L::K_BYTES));
#pragma unroll
        for (int k = 0; k < AK / 16; ++k)   // K (keys) 16 at a time: +32 bytes in P, +16 rows (2048 bytes) in V
          umma_bf16(tmem + 256 + 64 * pb, dp + (uint64_t)(2 * k), dv + (uint64_t)(128 * k), id_pv, k != 0);
        umma_commit(&pv_full[pb]);
        umma_commit(&kv_empty[b]);   // K, V and Pw of tile t are no longer read
        return true;
      };
      for (int tt = 0; ok && tt < Tl; ++tt) {
        const int b = tt % ANB;
        if (!mbar_wait(&kv_full[b], (tt / ANB) & 1, abort_flag)) { ok = false; break; }
        if (tt > 0 && !mbar_wait(s_free, (tt - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint8_t* st = sRing + b * L::STAGE;
        const uint64_t dk = sw128_desc(su32(st));
#pragma unroll
        for (int k = 0; k < AHD / 16; ++k) umma_bf16(tm_s, dqu + (uint64_t)(2 * k), dk + (uint64_t)(2 * k), id_s, k != 0);
        // BD columns 64 m .. 64 m + 63 <- position block t - m (local index tt + 2 - m)
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          const uint64_t dpw = sw128_desc(su32(sPw + ((tt + 2 - m) % NPW) * L::PB_BYTES));
#pragma unroll
          for (int k = 0; k < AHD / 16; ++k)
            umma_bf16(tm_bd + 64 * m, dqv + (uint64_t)(2 * k), dpw + (uint64_t)(2 * k), id_bd, k != 0);
        }
        umma_commit(s_full);
        umma_commit(&pw_empty[tt % NPW]);   // block t - 2 (local tt) is read for the last time by tile t
        if (tt > 0 && !issue_pv(tt - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(Tl - 1);
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
    // bounded wait with a warp-uniform outcome (the tcgen05.ld that follow are warp-collective)
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    // (Q + u) and (Q + v) rows, rounded to bf16, into the swizzled A tiles
    if (Tl > 0) {
      const bf16* qrow = qkv + (int64_t)(sb + (row_ok ? i : 0)) * (3 * D) + h * AHD;
      const float* uh = u + h * AHD;
      const float* vh = vb + h * AHD;
#pragma unroll
      for (int c = 0; c < AHD / 8; ++c) {
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (row_ok) raw = *reinterpret_cast<const uint4*>(qrow + 8 * c);
        const bf16* qv8 = reinterpret_cast<const bf16*>(&raw);
        uint32_t wu[4], wv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int d = 8 * c + 2 * k;
          const float a0 = __bfloat162float(qv8[2 * k]), a1 = __bfloat162float(qv8[2 * k + 1]);
          __nv_bfloat162 hu = __floats2bfloat162_rn(row_ok ? a0 + uh[d] : 0.f, row_ok ? a1 + uh[d + 1] : 0.f);
          __nv_bfloat162 hv = __floats2bfloat162_rn(row_ok ? a0 + vh[d] : 0.f, row_ok ? a1 + vh[d + 1] : 0.f);
          wu[k] = *reinterpret_cast<uint32_t*>(&hu);
          wv[k] = *reinterpret_cast<uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(sQu + sw128_off(r, c)) = make_uint4(wu[0], wu[1], wu[2], wu[3]);
        *reinterpret_cast<uint4*>(sQv + sw128_off(r, c)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }

    float* stg = sBD + (warp - 2) * 32 * BD_LD;
    const float sl2 = 1.4426950408889634f * 0.125f;   // log2(e) / sqrt(64)
    float m_run = -INFINITY, l_run = 0.f;
    float o[AHD];
#pragma unroll
    for (int d = 0; d < AHD; ++d) o[d] = 0.f;
    bool ok = true;
    for (int tt = 0; tt < Tl; ++tt) {
      const int j0 = (t0 + tt) * AK;
      if (!warp_wait(s_full, tt & 1)) { ok = false; break; }
      tc_fence_after();
      float sc[AK];
      {
        // this warp's BD band: columns 32q .. 32q + 95 of BD, one row per lane
        // (wide TMEM loads: one wait per load instruction)
        uint32_t v[64];
        tmem_ld64(tmem + lane_base + (uint32_t)(AK + 32 * q), v);
#pragma unroll
        for (int k = 0; k < 64; k += 4)
          *reinterpret_cast<float4*>(stg + lane * BD_LD + k) =
              make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]), __uint_as_float(v[k + 2]),
                          __uint_as_float(v[k + 3]));
        tmem_ld32(tmem + lane_base + (uint32_t)(AK + 32 * q + 64), v);
#pragma unroll
        for (int k = 0; k < 32; k += 4)
          *reinterpret_cast<float4*>(stg + lane * BD_LD + 64 + k) =
              make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]), __uint_as_float(v[k + 2]),
                          __uint_as_float(v[k + 3]));
        tmem_ld64(tmem + lane_base, v);
#pragma unroll
        for (int k = 0; k < AK; ++k) sc[k] = __uint_as_float(v[k]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);   // AC / BD of tile t read out of TMEM
      // key c of row r: BD column r - c + 63 = staged column lane + 63 - c.
      // AC + BD as packed adds, the running maximum over the unscaled sums
      // (the scale is positive), then p = 2^(s sl2 - m) as one packed FMA per
      // two keys
      const float* bdr = stg + lane * (BD_LD + 1) + (AK - 1);
#pragma unroll
      for (int c = 0; c < AK; c += 2) {
        const float2 t = __fadd2_rn(make_float2(sc[c], sc[c + 1]), make_float2(bdr[-c], bdr[-c - 1]));
        sc[c] = t.x;
        sc[c + 1] = t.y;
      }
      const bool full = j0 + AK <= S;
      if (!full) {   // last tile: keys past the sequence end get no weight
#pragma unroll
        for (int c = 0; c < AK; ++c)
          if (j0 + c >= S) sc[c] = -INFINITY;
      }
      // row maximum and sum as 8 / 4 independent partial chains (one warp per
      // scheduler: a single serial chain would expose every latency)
      float mp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mp[k] = sc[k];
#pragma unroll
      for (int c = 8; c < AK; ++c) mp[c & 7] = fmaxf(mp[c & 7], sc[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      const float m_new = fmaxf(m_run, mx * sl2);   // finite: key j0 < S
      const float alpha = ex2_approx(m_run - m_new);
      const float2 s2 = make_float2(sl2, sl2), nm2 = make_float2(-m_new, -m_new);
      float2 ps2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) ps2[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < AK; c += 2) {
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
      uint8_t* pt = sP + (tt & 1) * L::P_BYTES;
#pragma unroll
      for (int ch = 0; ch < AK / 8; ++ch) {
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
      if (lane == 0) mbar_arrive(&p_full[tt & 1]);
      // O (relative to m_(t-1)) += P_(t-1) V_(t-1), then rescale to m_t
      if (tt > 0) {
        const int pb = (tt - 1) & 1;
        if (!warp_wait(&pv_full[pb], ((tt - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[AHD];
        tmem_ld64(tmem + lane_base + (uint32_t)(256 + 64 * pb), v);
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int k = 0; k < AHD; k += 2) {
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
        uint32_t v[AHD];
        tmem_ld64(tmem + lane_base + (uint32_t)(256 + 64 * pb), v);
#pragma unroll
        for (int k = 0; k < AHD; ++k) o[k] += __uint_as_float(v[k]);
      } else {
        ok = false;
      }
    }
    if (!ok) *abort_flag = 1;
    auto store_row = [&](const float* ov, float l) {
      const float inv = 1.f / l;
      uint4* dst = reinterpret_cast<uint4*>(ctx + (int64_t)(sb + i) * D + h * AHD);
#pragma unroll
      for (int c = 0; c < AHD / 8; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 ho = __floats2bfloat162_rn(ov[8 * c + 2 * k] * inv, ov[8 * c + 2 * k + 1] * inv);
          w4[k] = *reinterpret_cast<uint32_t*>(&ho);
        }
        dst[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    };
    if (ks == 1) {
      if (ok && row_ok) store_row(o, l_run);
    } else {
      // Key split: the ks CTAs of a (query tile, head) form a cluster; each
      // leaves (O, m, l) of its key range in its own shared memory (the BD
      // staging area, free now) and the cluster's rank 0 merges them in rank
      // order over distributed shared memory after the cluster barrier.
      // Row r's slot overlaps another warp's BD band: all four softmax warps
      // finish their last tile before any slot is written.
      asm volatile("bar.sync 1, 128;" ::: "memory");
      float* mine = sBD + r * PSTR;
#pragma unroll
      for (int d = 0; d < AHD; d += 4)
        *reinterpret_cast<float4*>(mine + d) = make_float4(o[d], o[d + 1], o[d + 2], o[d + 3]);
      mine[AHD] = m_run;
      mine[AHD + 1] = l_run;
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
      const uint32_t row_addr = su32(sBD + r * PSTR);
      auto ld_peer = [&](uint32_t rank, int off) -> float {
        uint32_t a;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(row_addr + 4u * off), "r"(rank));
        float v;
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
        return v;
      };
      float mz[4], lz[4];
#pragma unroll
      for (int zz = 0; zz < 4; ++zz) {
        mz[zz] = zz < ks ? ld_peer(zz, AHD) : -INFINITY;
        lz[zz] = zz < ks ? ld_peer(zz, AHD + 1) : 0.f;
      }
      const float m = fmaxf(fmaxf(mz[0], mz[1]), fmaxf(mz[2], mz[3]));
      float acc[AHD], l = 0.f;
#pragma unroll
      for (int d = 0; d < AHD; ++d) acc[d] = 0.f;
#pragma unroll
      for (int zz = 0; zz < 4; ++zz) {
        if (zz >= ks) break;
        const float wz = ex2_approx(mz[zz] - m);   // an empty key range has m = -inf: weight 0
        l += wz * lz[zz];
#pragma unroll
        for (int d = 0; d < AHD; d += 4) {
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
        uint4* dst = reinterpret_cast<uint4*>(ctx + (int64_t)(sb + i) * D + h * AHD);
#pragma unroll
        for (int c = 0; c < AHD / 8; ++c) {
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u) : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag) set_err(err, ERR_TIMEOUT);
}

namespace {
int g_att_sms = 148;
int g_att_clusters[3] = {1, 0, 0};   // co-resident clusters of 1, 2, 4 CTAs (0: that split is off)
}

cudaError_t launch_relpos_attention_tc(const bf16* qkv, const bf16* ptab, int R, const float* u, const float* v,
                                       bf16* ctx, const SeqTable* seq, int n_tiles2, int M, int max_len,
                                       const TcScratch& sc, cudaStream_t st) {
  if (M <= 0 || n_tiles2 <= 0) return cudaSuccess;
  constexpr int D = 512;
  CUtensorMap t_qkv, t_pos;
  cudaError_t r = make_bf16_map_sw128(&t_qkv, qkv, M, 3 * D, 3 * D, AK);
  if (r != cudaSuccess) return r;
  r = make_bf16_map_sw128(&t_pos, ptab, 2 * R - 1, D, D, 64);
  if (r != cudaSuccess) return r;
  // fewer (query tile, head) units than SMs: split each unit's keys over a
  // cluster of 2 or 4 CTAs (no more splits than key tiles of the longest
  // sequence, and only while every cluster is co-resident), merged in the
  // cluster's shared memory
  const int units = n_tiles2 * 8;
  int ks = 1;
  if (units < g_att_sms) {
    const int want = g_att_sms / units, tmax = (max_len + AK - 1) / AK;
    if (want >= 4 && tmax >= 4 && units <= g_att_clusters[2]) ks = 4;
    else if (want >= 2 && tmax >= 2 && units <= g_att_clusters[1]) ks = 2;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles2, 8, ks);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = AttTc::SMEM;
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
  CK_LAUNCH(cudaLaunchKernelEx(&cfg, attn_relpos_tc_kernel, t_qkv, t_pos, qkv, D, R, u, v, ctx, seq, sc.err, ks));
  return cudaGetLastError();
}

cudaError_t attention_tc_init_attributes() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
      n > 0)
    g_att_sms = n;
  cudaError_t r = cudaFuncSetAttribute(attn_relpos_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AttTc::SMEM);
  if (r != cudaSuccess) return r;
  for (int j = 1; j < 3; ++j) {   // can clusters of 2 and 4 CTAs be scheduled at all?
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1 << j);
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = AttTc::SMEM;
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeClusterDimension;
    a.val.clusterDim.x = 1;
    a.val.clusterDim.y = 1;
    a.val.clusterDim.z = 1 << j;
    cfg.attrs = &a;
    cfg.numAttrs = 1;
    int n_cl = 0;
    g_att_clusters[j] = cudaOccupancyMaxActiveClusters(&n_cl, attn_relpos_tc_kernel, &cfg) == cudaSuccess ? n_cl : 0;
    cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace sf
