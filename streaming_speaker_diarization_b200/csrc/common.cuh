// Shared device-side definitions of the B200 Sortformer engine.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace sf {

typedef __nv_bfloat16 bf16;

// Device error word bits (engine-owned int, OR-ed by kernels, read by the host
// at synchronisation points).  Kernels never trap: they record and return.
enum : int {
  ERR_BOUNDS = 1,    // an index check failed; the access was skipped
  ERR_TIMEOUT = 2,   // a bounded wait (mbarrier / flag) gave up
  ERR_SHAPE = 4,     // a kernel met a size it does not support
};

constexpr int MAX_SEQ = 512;   // sequences / streams per call
constexpr int ATT_TILE = 64;   // query rows per attention CTA

// Packed-sequence table in device memory: sequence s occupies rows
// [off[s], off[s+1]) of the token matrix; its 64-row attention query tiles
// are global tiles [tile_off[s], tile_off[s+1]), its 128-row tiles
// [tile2_off[s], tile2_off[s+1]).
struct SeqTable {
  int n_seq;
  int total;
  int off[MAX_SEQ + 1];
  int tile_off[MAX_SEQ + 1];
  int tile2_off[MAX_SEQ + 1];
};

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + __expf(-z)); }
__device__ __forceinline__ float swishf_(float z) { return z * sigmoidf_(z); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sequence containing packed row r (binary search over off[0..n_seq]).
__device__ __forceinline__ int seq_of_row(const SeqTable* __restrict__ st, int r) {
  int lo = 0, hi = st->n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (st->off[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int seq_of_tile2(const SeqTable* __restrict__ st, int g) {
  int lo = 0, hi = st->n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (st->tile2_off[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int seq_of_tile(const SeqTable* __restrict__ st, int g) {
  int lo = 0, hi = st->n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (st->tile_off[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void set_err(int* err, int bit) {
  if (err) atomicOr(err, bit);
}

// Programmatic dependent launch (when enabled): every kernel waits for its
// predecessor's memory before its first global access.  The GEMMs let their
// successor launch once their last MMA is issued, so the successor's launch
// and set-up overlap the epilogue; other kernels release it when they exit.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
#define SF_PDL_ENTRY() sf::pdl_wait()

#define CK_LAUNCH(x)                  \
  do {                                \
    cudaError_t _le = (x);            \
    if (_le != cudaSuccess) return _le; \
  } while (0)

// Launch mode of the calling engine (set at each API entry, per host
// thread): 0 = plain stream order, 1 = programmatic dependent launch.
extern thread_local int g_launch_pdl;

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_launch_pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace sf
