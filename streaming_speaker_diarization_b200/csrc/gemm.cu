// Dense projections: C[M, N] = A[M, K] . W[N, K]^T with fused epilogues
// (bias, ReLU, swish, GLU on interleaved column pairs, scaled residual add
// into the fp32 stream, fp32 and dual fp32/act stores, row remapping).
//
// gemm_simt: fp32 FFMA tiles (64 x 64 x 16), used by the fp32 engine mode
//            whose tolerance (1e-4 on probabilities) rules out reduced-
//            precision tensor-core inputs.
// gemm_mma:  bf16 tensor-core tiles (128 x 128 x 32, mma.sync m16n8k16,
//            ldmatrix, 3-stage cp.async pipeline); the portable tensor-core
//            path, kept as the cross-check of the tcgen05 kernel.
#include "common.cuh"
#include "layers.h"
#include "epilogue.cuh"

namespace sf {

// ------------------------------------------------------------- fp32 SIMT
__global__ void __launch_bounds__(256) gemm_simt_kernel(const float* __restrict__ A, int lda,
                                                        const float* __restrict__ W, int M, int N, int K, Epi e) {
  SF_PDL_ENTRY();
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    {
      const int row = tid / 4, kk = (tid % 4) * 4;
      float4 va = make_float4(0, 0, 0, 0), vb = make_float4(0, 0, 0, 0);
      if (m0 + row < M) va = *reinterpret_cast<const float4*>(A + (int64_t)(m0 + row) * lda + k0 + kk);
      if (n0 + row < N) vb = *reinterpret_cast<const float4*>(W + (int64_t)(n0 + row) * K + k0 + kk);
      As[kk + 0][row] = va.x; As[kk + 1][row] = va.y; As[kk + 2][row] = va.z; As[kk + 3][row] = va.w;
      Bs[kk + 0][row] = vb.x; Bs[kk + 1][row] = vb.y; Bs[kk + 2][row] = vb.z; Bs[kk + 3][row] = vb.w;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[k][ty * 4 + i]; b[i] = Bs[k][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      const int c = n0 + tx * 4 + j;
      if (c < N) epi_store2<float>(e, r, c, acc[i][j], acc[i][j + 1]);
    }
  }
}

// ------------------------------------------------------------- bf16 mma.sync
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  const int sz = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int MM_BM = 128, MM_BN = 128, MM_BK = 32, MM_LD = 40, MM_STAGES = 3;
constexpr int MM_SMEM = MM_STAGES * (MM_BM + MM_BN) * MM_LD * 2;

__global__ void __launch_bounds__(256) gemm_mma_kernel(const bf16* __restrict__ A, int lda,
                                                       const bf16* __restrict__ W, int M, int N, int K, Epi e) {
  SF_PDL_ENTRY();
  extern __shared__ float4 mm_smem[];
  bf16* sA = reinterpret_cast<bf16*>(mm_smem);
  bf16* sB = sA + MM_STAGES * MM_BM * MM_LD;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 2, wn = warp & 3;          // 2 x 4 warps, warp tile 64 x 32
  const int m0 = blockIdx.y * MM_BM, n0 = blockIdx.x * MM_BN;
  const int KT = K / MM_BK;

  auto load_tile = [&](int stage, int kt) {
    const int k0 = kt * MM_BK;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int ch = tid + j * 256;            // 512 16-byte chunks per operand tile
      const int row = ch >> 2, kc = (ch & 3) * 8;
      const bool pa = (m0 + row) < M, pb = (n0 + row) < N;
      const bf16* ga = A + (int64_t)(pa ? m0 + row : 0) * lda + k0 + kc;
      const bf16* gb = W + (int64_t)(pb ? n0 + row : 0) * K + k0 + kc;
      cp_async16(smem_u32(sA + (stage * MM_BM + row) * MM_LD + kc), ga, pa);
      cp_async16(smem_u32(sB + (stage * MM_BN + row) * MM_LD + kc), gb, pb);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.f;

#pragma unroll
  for (int s = 0; s < MM_STAGES - 1; ++s) {
    if (s < KT) load_tile(s, s);
    cp_async_commit();
  }
  for (int kt = 0; kt < KT; ++kt) {
    cp_async_wait<MM_STAGES - 2>();
    __syncthreads();
    {
      const int nk = kt + MM_STAGES - 1;
      if (nk < KT) load_tile(nk % MM_STAGES, nk);
      cp_async_commit();
    }
    const int st = kt % MM_STAGES;
    const bf16* tA = sA + st * MM_BM * MM_LD;
    const bf16* tB = sB + st * MM_BN * MM_LD;
#pragma unroll
    for (int kk = 0; kk < MM_BK; kk += 16) {
      uint32_t af[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int row = wm * 64 + mt * 16 + (lane & 15);
        const int col = kk + (lane >> 4) * 8;
        ldsm_x4(smem_u32(tA + row * MM_LD + col), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
      }
      uint32_t bfr[4][2];
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int nrow = wn * 32 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int col = kk + ((lane >> 3) & 1) * 8;
        ldsm_x4(smem_u32(tB + nrow * MM_LD + col), bfr[np * 2][0], bfr[np * 2][1], bfr[np * 2 + 1][0],
                bfr[np * 2 + 1][1]);
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_bf16(acc[mt][nt], af[mt], bfr[nt][0], bfr[nt][1]);
    }
  }
  cp_async_wait<0>();

  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int r = m0 + wm * 64 + mt * 16 + g;
      const int c = n0 + wn * 32 + nt * 8 + q * 2;
      if (c < N) {
        if (r < M) epi_store2<bf16>(e, r, c, acc[mt][nt][0], acc[mt][nt][1]);
        if (r + 8 < M) epi_store2<bf16>(e, r + 8, c, acc[mt][nt][2], acc[mt][nt][3]);
      }
    }
}

cudaError_t gemm_f32(const float* A, int lda, const float* W, int M, int N, int K, const Epi& e, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  CK_LAUNCH(launch_k(gemm_simt_kernel, dim3(grid), dim3(256), 0, st, A, lda, W, M, N, K, e));
  return cudaGetLastError();
}

cudaError_t gemm_bf16_mma(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  dim3 grid((N + MM_BN - 1) / MM_BN, (M + MM_BM - 1) / MM_BM);
  CK_LAUNCH(launch_k(gemm_mma_kernel, dim3(grid), dim3(256), MM_SMEM, st, A, lda, W, M, N, K, e));
  return cudaGetLastError();
}

cudaError_t gemm_init_attributes() {
  return cudaFuncSetAttribute(gemm_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, MM_SMEM);
}

}  // namespace sf
