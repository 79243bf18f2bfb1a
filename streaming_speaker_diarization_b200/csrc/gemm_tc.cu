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
//           its 32-lane TMEM quarter = 32 output rows) and apply the epilogue.
// Full/empty mbarriers order the ring; every wait is bounded by a clock
// budget: a wait that runs out sets ERR_TIMEOUT in the engine's error word,
// raises a CTA-wide abort flag, the producer waits (bounded) for its own
// loads in flight, and TMEM is released before the CTA exits.
// No cluster multicast is used anywhere.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "layers.h"

namespace sf {
namespace {

constexpr int TC_BM = 128, TC_BK = 64;
constexpr long long WAIT_CYCLES = 4000000000LL;   // ~2 s at 2 GHz

__device__ __forceinline__ uint32_t su32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase of the given parity; false on timeout or abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag) {
  const long long t0 = clock64();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(b, parity)) return true;
    if ((i & 63) == 63) {
      if (*abort_flag) return false;
      if (clock64() - t0 > WAIT_CYCLES) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Shared-memory matrix descriptor: K-major tile whose rows are 128 bytes,
// 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);   // start address, bits [0, 14)
  d |= (uint64_t)1 << 16;                    // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset, bits [32, 46)
  d |= (uint64_t)1 << 46;                    // descriptor version, bits [46, 48)
  d |= (uint64_t)2 << 61;                    // 128-byte swizzle, bits [61, 64)
  return d;
}

// Instruction descriptor: bf16 x bf16 -> f32, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TC_BM >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int BN, int STAGES>
struct TcCfg {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int SMEM = 1024 + STAGES * (A_BYTES + B_BYTES) + 256;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(192, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap ta,
                                                         const __grid_constant__ CUtensorMap tb, int M, int N, int K,
                                                         Epi e, int* err) {
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
  const int KB = (K + TC_BK - 1) / TC_BK;

  if (threadIdx.x == 0) {
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

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES, r = kb / STAGES;
        if (!mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        mbar_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
        tma_load_2d(sA + s * C::A_BYTES, &ta, &full[s], kb * TC_BK, m0);
        tma_load_2d(sB + s * C::B_BYTES, &tb, &full[s], kb * TC_BK, n0);
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
    }
  } else {
    // Epilogue: per 64-column chunk, each warp copies its 32 x 64 accumulator
    // block from TMEM to a padded shared tile (thread = row), then writes it
    // out with lanes along the columns (one contiguous row segment per store
    // instruction).  The pipeline buffers are free once the accumulator is
    // complete, so the tiles reuse them.
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    float* stage = reinterpret_cast<float*>(sm) + q * (32 * 65);
    if (mbar_wait(accf, 0, abort_flag) && !*abort_flag) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 64) {
        uint32_t v[16];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(c0 + 16 * h), v);
#pragma unroll
          for (int j = 0; j < 16; ++j) stage[lane * 65 + 16 * h + j] = __uint_as_float(v[j]);
        }
        __syncwarp();
        const int c = n0 + c0 + 2 * lane;
#pragma unroll 4
        for (int rr = 0; rr < 32; ++rr) {
          const int row = m0 + 32 * q + rr;
          if (row < M && c < N) epi_store2<bf16>(e, row, c, stage[rr * 65 + 2 * lane], stage[rr * 65 + 2 * lane + 1]);
        }
        __syncwarp();
      }
    } else {
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)BN) : "memory");
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

template <int BN, int STAGES>
cudaError_t launch_tc(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e, int* err,
                      cudaStream_t st) {
  CUtensorMap ta, tb;
  cudaError_t r = make_map(&ta, A, M, K, lda, TC_BM);
  if (r != cudaSuccess) return r;
  r = make_map(&tb, W, N, K, K, BN);
  if (r != cudaSuccess) return r;
  dim3 grid((N + BN - 1) / BN, (M + TC_BM - 1) / TC_BM);
  gemm_tc_kernel<BN, STAGES><<<grid, 192, TcCfg<BN, STAGES>::SMEM, st>>>(ta, tb, M, N, K, e, err);
  return cudaGetLastError();
}

}  // namespace

// Tile width: the widest of 256 / 128 / 64 that does not cost extra waves of
// 148 SMs (cost ~ waves x (BN + 32), 32 standing for the per-tile A traffic).
int gemm_tc_pick_bn(int M, int N) {
  const int tm = (M + TC_BM - 1) / TC_BM;
  int best = 64;
  double best_cost = 1e30;
  for (int bn : {256, 128, 64}) {
    const int tiles = tm * ((N + bn - 1) / bn);
    const int waves = (tiles + 147) / 148;
    const double cost = (double)waves * (bn + 32);
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

cudaError_t gemm_bf16_tc(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e, int* err,
                         cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  if (N % 16 || K % 8) return cudaErrorInvalidValue;
  cudaError_t r = get_encoder();
  if (r != cudaSuccess) return r;
  switch (gemm_tc_pick_bn(M, N)) {
    case 256: return launch_tc<256, 4>(A, lda, W, M, N, K, e, err, st);
    case 128: return launch_tc<128, 6>(A, lda, W, M, N, K, e, err, st);
    default: return launch_tc<64, 8>(A, lda, W, M, N, K, e, err, st);
  }
}

cudaError_t gemm_tc_init_attributes() {
  cudaError_t r = get_encoder();
  if (r != cudaSuccess) return r;
  r = cudaFuncSetAttribute(gemm_tc_kernel<256, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TcCfg<256, 4>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc_kernel<128, 6>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<128, 6>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc_kernel<64, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<64, 8>::SMEM);
  return r;
}

}  // namespace sf
