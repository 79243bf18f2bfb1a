// Row-per-thread GEMM epilogues with TMA bulk stores (sm_100a).
//
// An epilogue warp owns 32 accumulator rows (its TMEM lane quarter): thread
// = row.  Per chunk of columns it reads its row's accumulators with one
// tcgen05.ld, applies bias / activation / residual in registers, writes the
// finished row segment into a shared-memory box laid out as the tensor map's
// swizzle expects (rows of 128 or 64 bytes; the 16-byte units of row r
// permuted by r), and one lane stores the 32-row box with
// cp.async.bulk.tensor.  The TMA engine clips rows >= M and columns past the
// matrix; the threads never wait for global stores.  Residual rows are read
// before the accumulator is complete, so their latency hides behind the main
// loop: into registers in the single-wave kernel, as TMA boxes into the box
// buffers in the persistent kernels (resid_tma_*).
//
// Box buffers: each warp alternates between its buffers; before rewriting a
// buffer, lane 0 waits until at most one earlier store group still reads
// shared memory (cp.async.bulk.wait_group.read 1), and before the CTA's
// shared memory is released or reused it waits until all of its stores have
// read their boxes.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "common.cuh"
#include "layers.h"
#include "tcgen05.cuh"

namespace sf {

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(su32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most one committed store group may still be reading shared memory
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// every committed store group has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Logistic sigmoid through one special-function operation: sigmoid(x) =
// (1 + tanh(x / 2)) / 2 with the hardware tanh approximation (absolute error
// about 2^-11, below the rounding of the bf16 outputs it feeds), where the
// exp-and-reciprocal form takes two.
__device__ __forceinline__ float sigmoid_t(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Row r's 16-byte unit u of a box with 128-byte rows, 128-byte swizzle
// (buffer 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128_unit(uint32_t base, int r, int u) {
  return base + (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4));
}
// Row r's 16-byte unit u of a box with 64-byte rows, 64-byte swizzle.
__device__ __forceinline__ uint32_t sw64_unit(uint32_t base, int r, int u) {
  return base + (uint32_t)(r * 64 + ((u ^ ((r >> 1) & 3)) << 4));
}

constexpr int EPI_BOX_BYTES = 4096;   // 32 rows x 128 bytes

// Per-warp box ring: two 4 KB buffers; `n` counts the stores issued so far.
struct BoxRing {
  uint8_t* base;
  int n;
  __device__ __forceinline__ uint8_t* next(int lane) {
    uint8_t* b = base + (n & 1) * EPI_BOX_BYTES;
    if (lane == 0 && n >= 2) bulk_wait_read1();
    __syncwarp();
    return b;
  }
  // publish the box written by this warp's threads and store it at (x, y)
  __device__ __forceinline__ void store(const CUtensorMap* map, const uint8_t* b, int x, int y, bool valid, int lane) {
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (valid) tma_store_2d(map, b, x, y);
      bulk_commit();   // an empty group keeps the buffer count in step
    }
    ++n;
  }
  __device__ __forceinline__ void drain(int lane) {
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
  }
};

// Epilogue parameters (bias, LayerNorm weights) are read before the
// accumulator is complete and kept spread over the warp's lanes: for a
// 64-column chunk lane l holds columns 2l and 2l + 1, for a 32-column chunk
// column l; a warp shuffle hands each thread (row) the value of column k.
// Zeros past N or for a null vector.
__device__ __forceinline__ float2 lane_param64(const float* p, int c, int N, int lane) {
  if (!p || c + 2 * lane >= N) return make_float2(0.f, 0.f);
  return __ldg(reinterpret_cast<const float2*>(p + c + 2 * lane));
}
__device__ __forceinline__ float lane_param32(const float* p, int c, int N, int lane) {
  if (!p || c + lane >= N) return 0.f;
  return __ldg(p + c + lane);
}
__device__ __forceinline__ float col64(float2 p, int k) {
  return __shfl_sync(0xffffffffu, (k & 1) ? p.y : p.x, k >> 1);
}
// bias[c + j] added to v[j] (columns below N) with loads every lane makes
// at the same address
template <int NV>
__device__ __forceinline__ void add_bias_bcast(float* v, const float* bias, int c, int N) {
  if (!bias) return;
#pragma unroll
  for (int j = 0; j < NV; j += 4) {
    if (c + j < N) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(bias + c + j));
      v[j] += b.x; v[j + 1] += b.y; v[j + 2] += b.z; v[j + 3] += b.w;
    }
  }
}
// Ask L1 for a tile's bias (BN floats from column n0) ahead of its epilogue.
__device__ __forceinline__ void prefetch_bias_l1(const float* bias, int n0, int BN, int N, int lane) {
  const int c = n0 + 32 * lane;
  if (bias && 32 * lane < BN && c < N) asm volatile("prefetch.global.L1 [%0];" ::"l"(bias + c));
}

// Columns per chunk: 64 for the kinds that write bf16 (one 128-byte box row,
// or 64 bytes after the gated linear unit), 32 for those that write f32.
__host__ __device__ constexpr int row_epi_chunk(int kind) {
  return (kind == EPI_BIAS || kind == EPI_BIAS_RELU || kind == EPI_BIAS_SWISH || kind == EPI_BIAS_GLU) ? 64 : 32;
}

// The residual row segment (32 f32 columns at c) of this thread's row, or
// zeros past the matrix.
__device__ __forceinline__ void load_resid32(const Epi& e, int row, int M, int c, int N, float* x) {
  const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(e.out) + (int64_t)row * e.ldo + c);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < M && c + 4 * j < N) t = p[j];
    x[4 * j] = t.x; x[4 * j + 1] = t.y; x[4 * j + 2] = t.z; x[4 * j + 3] = t.w;
  }
}

// One warp's share of a tile's epilogue: rows m_w .. m_w + 31 (this warp's
// TMEM lane quarter at accumulator column base `acc`), chunks j = first,
// first + step, ... of the tile's columns [n0, n0 + BN).  The caller reads
// the first chunk's bias (epi_prefetch) and, for EPI_RESID, its residual
// into `bias2` / `xr` before waiting for the accumulator.
template <int EK, int BN, bool LANE_BIAS>
__device__ __forceinline__ void row_epilogue(const Epi& e, const CUtensorMap* mo, const CUtensorMap* mo2, uint32_t acc,
                                             BoxRing& ring, int M, int N, int m_w, int n0, int first, int step,
                                             int lane, float* xr, float2& bias2) {
  constexpr int CW = row_epi_chunk(EK);
  constexpr int NCH = BN / CW;
  const int row = m_w + lane;
  const bool rows_in = m_w < M;
#pragma unroll 1
  for (int j = first; j < NCH; j += step) {
    const int c = n0 + j * CW;
    // LANE_BIAS: this chunk's bias was read lane-spread by the caller or the
    // previous chunk, and the next chunk's is in flight meanwhile; else each
    // thread reads the chunk's bias with broadcast loads (cached in L1)
    const float2 bc = bias2;
    if (LANE_BIAS && j + step < NCH) {
      if (CW == 64) bias2 = lane_param64(e.bias, c + step * CW, N, lane);
      else bias2.x = lane_param32(e.bias, c + step * CW, N, lane);
    }
    if (CW == 64) {
      float v[64];
      tmem_ld64(acc + (uint32_t)(j * CW), reinterpret_cast<uint32_t*>(v));
      if (LANE_BIAS) {
#pragma unroll
        for (int k = 0; k < 64; ++k) v[k] += col64(bc, k);
      } else {
        add_bias_bcast<64>(v, e.bias, c, N);
      }
      if (EK == EPI_BIAS_RELU) {
#pragma unroll
        for (int k = 0; k < 64; ++k) v[k] = fmaxf(v[k], 0.f);
      }
      if (EK == EPI_BIAS_SWISH) {
#pragma unroll
        for (int k = 0; k < 64; ++k) v[k] *= sigmoid_t(v[k]);
      }
      uint8_t* b = ring.next(lane);
      const uint32_t sb = su32(b);
      if (EK == EPI_BIAS_GLU) {   // interleaved (value, gate) pairs -> 32 outputs, 64-byte rows
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t w[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int k = 16 * u + 4 * t;
            w[t] = pack_bf16(v[k] * sigmoid_t(v[k + 1]), v[k + 2] * sigmoid_t(v[k + 3]));
          }
          sts128(sw64_unit(sb, lane, u), w[0], w[1], w[2], w[3]);
        }
        ring.store(mo, b, c >> 1, m_w, rows_in && c < N, lane);
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u)
          sts128(sw128_unit(sb, lane, u), pack_bf16(v[8 * u], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                 pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
        ring.store(mo, b, c, m_w, rows_in && c < N, lane);
      }
    } else {
      float v[32];
      tmem_ld32(acc + (uint32_t)(j * CW), reinterpret_cast<uint32_t*>(v));
      if (LANE_BIAS) {
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] += __shfl_sync(0xffffffffu, bc.x, k);
      } else {
        add_bias_bcast<32>(v, e.bias, c, N);
      }
      if (EK == EPI_RESID) {
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = xr[k] + e.alpha * v[k];
        // the next chunk's residual: in flight while this chunk is stored
        if (j + step < NCH) load_resid32(e, row, M, c + step * CW, N, xr);
      }
      uint8_t* b = ring.next(lane);
      const uint32_t sb = su32(b);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        sts128(sw128_unit(sb, lane, u), __float_as_uint(v[4 * u]), __float_as_uint(v[4 * u + 1]),
               __float_as_uint(v[4 * u + 2]), __float_as_uint(v[4 * u + 3]));
      ring.store(mo, b, c, m_w, rows_in && c < N, lane);
      if (EK == EPI_F32_AND_T) {   // the bf16 copy: 32 columns, 64-byte rows
        uint8_t* b2 = ring.next(lane);
        const uint32_t sb2 = su32(b2);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          sts128(sw64_unit(sb2, lane, u), pack_bf16(v[8 * u], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                 pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
        ring.store(mo2, b2, c, m_w, rows_in && c < N, lane);
      }
    }
  }
}

// Parameters of a warp's first chunk, read while the main loop still runs:
// the bias (lane-spread, or the tile's bias lines requested into L1) and,
// for EPI_RESID, this thread's residual row segment.  The single-wave kernel
// meets each layer's bias cold and spreads it over the lanes; the persistent
// kernels reuse it across tiles from L1, where broadcast loads are cheaper
// than the shuffles.
template <bool LANE_BIAS, int BN>
__device__ __forceinline__ void epi_prefetch(const Epi& e, int M, int N, int m_w, int n0, int first, int lane,
                                             float* xr, float2& bias2) {
  const int cw = row_epi_chunk(e.kind);
  const int c = n0 + first * cw;
  if (LANE_BIAS) {
    if (cw == 64) bias2 = lane_param64(e.bias, c, N, lane);
    else bias2 = make_float2(lane_param32(e.bias, c, N, lane), 0.f);
  } else {
    prefetch_bias_l1(e.bias, n0, BN, N, lane);
  }
  if (e.kind == EPI_RESID) load_resid32(e, m_w + lane, M, c, N, xr);
}

// EPI_RESID in the persistent kernels: the residual comes into the warp's
// two box buffers as 32 x 32 f32 boxes by TMA loads through the output map
// itself, each thread reads its row segment back from shared memory, adds
// alpha (acc + bias) in place, and the box goes out by the TMA store.  Per
// thread that replaces eight 16-byte global loads per chunk, each touching
// 32 rows in a warp, by conflict-free shared-memory reads.  A tile's first
// two chunks are requested before its accumulator wait; the buffer of chunk
// t is reloaded with chunk t + 2 as soon as chunk t's store has read it, so
// that load runs while chunk t + 1 is processed.  Warps whose 32 rows start
// past M load and store nothing.
struct ResidTma {
  uint64_t* bar;       // the warp's two mbarriers (one per box buffer)
  uint32_t phase;      // bit b: parity of buffer b's next load completion
  uint32_t pending;    // bit b: a load into buffer b is not yet waited for
};

__device__ __forceinline__ void lds128(uint32_t addr, float* v) {
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
               : "r"(addr)
               : "memory");
}

// Request the residual box (columns c .., rows m_w ..) into buffer b; the
// caller has made sure no store still reads that buffer.
__device__ __forceinline__ void resid_tma_request(const CUtensorMap* mo, const BoxRing& ring, ResidTma& rt, int b, int c,
                                                  int m_w, int M, int N, int lane) {
  if (m_w >= M || c >= N) return;   // uniform over the warp
  if (lane == 0) {
    mbar_expect_tx(&rt.bar[b], EPI_BOX_BYTES);
    tma_load_2d(ring.base + b * EPI_BOX_BYTES, mo, &rt.bar[b], c, m_w);
  }
  rt.pending |= 1u << b;
}

// Before a tile's accumulator wait: the tile's bias lines into L1, every
// earlier store of this warp done reading its buffer, the first two
// residual boxes requested.
template <int BN>
__device__ __forceinline__ void resid_tma_prologue(const Epi& e, const CUtensorMap* mo, const BoxRing& ring,
                                                   ResidTma& rt, int M, int N, int m_w, int n0, int first, int step,
                                                   int lane) {
  prefetch_bias_l1(e.bias, n0, BN, N, lane);
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int j = first + t * step;
    if (j < BN / 32) resid_tma_request(mo, ring, rt, t, n0 + j * 32, m_w, M, N, lane);
  }
}

// The warp's chunks j = first, first + step, ... of the tile; false when a
// residual load was not seen within the wait bound (or the kernel aborted).
template <int BN>
__device__ __forceinline__ bool resid_tma_rows(const Epi& e, const CUtensorMap* mo, uint32_t acc, BoxRing& ring,
                                               ResidTma& rt, int M, int N, int m_w, int n0, int first, int step,
                                               int lane, volatile int* abort_flag) {
  constexpr int NCH = BN / 32;
  int t = 0;
#pragma unroll 1
  for (int j = first; j < NCH; j += step, ++t) {
    const int c = n0 + j * 32, b = t & 1;
    const bool valid = m_w < M && c < N;
    float v[32];
    tmem_ld32(acc + (uint32_t)(j * 32), reinterpret_cast<uint32_t*>(v));
    add_bias_bcast<32>(v, e.bias, c, N);
    uint8_t* box = ring.base + b * EPI_BOX_BYTES;
    const uint32_t sb = su32(box);
    if (valid) {
      if (__any_sync(0xffffffffu, !mbar_wait(&rt.bar[b], (rt.phase >> b) & 1u, abort_flag))) return false;
      rt.phase ^= 1u << b;
      rt.pending &= ~(1u << b);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float x[4];
        const uint32_t a = sw128_unit(sb, lane, u);
        lds128(a, x);
        sts128(a, __float_as_uint(x[0] + e.alpha * v[4 * u]), __float_as_uint(x[1] + e.alpha * v[4 * u + 1]),
               __float_as_uint(x[2] + e.alpha * v[4 * u + 2]), __float_as_uint(x[3] + e.alpha * v[4 * u + 3]));
      }
    }
    ring.store(mo, box, c, m_w, valid, lane);
    if (j + 2 * step < NCH) {
      if (lane == 0) bulk_wait_read_all();   // the store just issued has read the buffer
      __syncwarp();
      resid_tma_request(mo, ring, rt, b, n0 + (j + 2 * step) * 32, m_w, M, N, lane);
    }
  }
  return true;
}

// Before the shared memory is released: loads that were requested but not
// waited for (only after an abort) land first, within the wait bound.
__device__ __forceinline__ void resid_tma_drain(ResidTma& rt) {
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    if (!(rt.pending >> b & 1u)) continue;
    const long long t0 = clock64();
    while (!mbar_try_wait(&rt.bar[b], (rt.phase >> b) & 1u) && clock64() - t0 < WAIT_CYCLES) {
    }
  }
  rt.pending = 0;
}

// Dispatch on the epilogue kind (after epi_prefetch).
template <int BN, bool LANE_BIAS>
__device__ __forceinline__ void row_epilogue_any(const Epi& e, const CUtensorMap* mo, const CUtensorMap* mo2,
                                                 uint32_t acc, BoxRing& ring, int M, int N, int m_w, int n0, int first,
                                                 int step, int lane, float* xr, float2& bias2) {
  switch (e.kind) {
    case EPI_BIAS: row_epilogue<EPI_BIAS, BN, LANE_BIAS>(e, mo, mo2, acc, ring, M, N, m_w, n0, first, step, lane, xr, bias2); break;
    case EPI_BIAS_RELU: row_epilogue<EPI_BIAS_RELU, BN, LANE_BIAS>(e, mo, mo2, acc, ring, M, N, m_w, n0, first, step, lane, xr, bias2); break;
    case EPI_BIAS_SWISH: row_epilogue<EPI_BIAS_SWISH, BN, LANE_BIAS>(e, mo, mo2, acc, ring, M, N, m_w, n0, first, step, lane, xr, bias2); break;
    case EPI_BIAS_GLU: row_epilogue<EPI_BIAS_GLU, BN, LANE_BIAS>(e, mo, mo2, acc, ring, M, N, m_w, n0, first, step, lane, xr, bias2); break;
    case EPI_RESID: row_epilogue<EPI_RESID, BN, LANE_BIAS>(e, mo, mo2, acc, ring, M, N, m_w, n0, first, step, lane, xr, bias2); break;
    case EPI_F32: row_epilogue<EPI_F32, BN, LANE_BIAS>(e, mo, mo2, acc, ring, M, N, m_w, n0, first, step, lane, xr, bias2); break;
    default: row_epilogue<EPI_F32_AND_T, BN, LANE_BIAS>(e, mo, mo2, acc, ring, M, N, m_w, n0, first, step, lane, xr, bias2); break;
  }
}

}  // namespace sf
