// Failure-detection self-test: the bounded device wait of the tcgen05
// kernels, run on an mbarrier that nothing ever arrives on.  The wait gives
// up after its clock budget (~2 s), the kernel records ERR_TIMEOUT in the
// engine's error word and returns, so the host sees SF_ETIMEOUT from
// sf_check and the CUDA context stays usable.  No fault, trap or unbounded
// loop is involved: the wait ends by the clock.
#include "common.cuh"
#include "layers.h"
#include "tcgen05.cuh"

namespace sf {

__global__ void __launch_bounds__(32) selftest_wait_kernel(int* __restrict__ err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);   // phase 0 completes only after one arrival, which never comes
  if (!mbar_wait(&bar, 0, &abort_flag)) atomicOr(err, ERR_TIMEOUT);
}

cudaError_t launch_selftest_wait(int* err, cudaStream_t st) {
  CK_LAUNCH(launch_k(selftest_wait_kernel, dim3(1), dim3(32), 0, st, err));
  return cudaGetLastError();
}

}  // namespace sf
