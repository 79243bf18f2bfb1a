// Helpers of the tcgen05 attention kernels: the MN-major operand descriptor,
// the 128-byte swizzle of hand-written operand tiles, the exp2
// approximation.
#pragma once
#include <stdint.h>

namespace sf {

// Shared-memory descriptor of an MN-major operand with 128-byte swizzle:
// rows of 64 bf16 along N (one swizzle atom wide), consecutive K rows 128
// bytes apart, 8-row groups 1024 bytes apart (stride byte offset).
__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
  d |= (uint64_t)(8192 >> 4) << 16;          // leading byte offset: next atom along N (not reached, N = 64)
  d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset: next 8 rows along K
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// 2^x with the hardware approximation (ex2.approx.ftz.f32: relative error
// ~2^-22, far inside the bf16 rounding of P; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


// Byte offset of element (row, col) (col in bf16 units, < 64) of a K-major
// tile with 128-byte rows and the 128-byte swizzle (16-byte chunk index
// XOR row % 8), as TMA writes it and tcgen05 reads it.
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

}  // namespace sf
