// k_selftest.cu -- self-test of the library's failure detection.
//
// Every wait inside a kernel of the library is bounded: a wait that runs out
// records a timeout in the sticky device error word and the kernel unwinds
// instead of hanging. This file holds a kernel that takes that path on
// purpose, with a short limit, so that a test can check it without faulting
// or hanging the GPU. It is not part of the method.
#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

// One CTA of four warps. Thread 0 initialises an mbarrier that expects one
// arrival. With arrive != 0 thread 0 arrives first, so the phase completes
// and every warp's wait must succeed; with arrive == 0 nothing arrives, and
// every warp's bounded wait (mbar_wait_warp, the wait of the TMA and
// tensor-core pipelines) must give up after limit_ns, record the timeout and
// let the warp leave together. result[w] = 1 when warp w's wait succeeded.
__global__ void __launch_bounds__(128, 1)
    selftest_mbar(unsigned* err, unsigned long long limit_ns, int arrive, int* result) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (arrive != 0 && threadIdx.x == 0) mbar_arrive(&bar);
  const bool ok = mbar_wait_warp(&bar, 0, err, limit_ns);
  if ((threadIdx.x & 31) == 0) result[threadIdx.x >> 5] = ok ? 1 : 0;
}

}  // namespace

cudaError_t launch_selftest_mbar(unsigned* err, unsigned long long limit_ns, int arrive,
                                 int* result, cudaStream_t st) {
  selftest_mbar<<<1, 128, 0, st>>>(err, limit_ns, arrive, result);
  return cudaGetLastError();
}

}  // namespace tg
