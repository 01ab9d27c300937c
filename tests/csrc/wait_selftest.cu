// GPU self-test of the bounded-wait error path the kernels use (sm100.cuh):
// a wait on an mbarrier phase that never completes must give up after its
// limit and report GDN_ERR_DEVICE_TIMEOUT through the status word, without a
// trap, a fault or a hang; the context stays usable afterwards.
//   mode 0: thread 0 waits (bounded) on a barrier nobody arrives on
//   mode 1: thread 0 arrives first, then waits: must succeed at once
//   mode 2: a 128-thread role: the leader's bounded wait gives up, it writes
//           the verdict, the role meets at a named barrier and every thread
//           leaves (the agreement pattern of the prefill kernel's roles)
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/gdn.h"
#include "sm100.cuh"

using namespace gdn::sm100;

__global__ void wait_selftest_kernel(int mode, unsigned long long limit_ns, int* status,
                                     unsigned long long* elapsed, int* left) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int verdict;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
    verdict = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (mode == 1) mbar_arrive(b);
    const unsigned long long t0 = globaltimer_ns();
    const bool ok = mbar_wait_bounded(b, 0, limit_ns);
    *elapsed = globaltimer_ns() - t0;
    verdict = ok ? 0 : 1;
    if (!ok) atomicExch(status, GDN_ERR_DEVICE_TIMEOUT);
  }
  if (mode == 2) {
    named_bar(1, 128);
    if (verdict != 0) {  // every thread of the role sees the same verdict and leaves
      atomicAdd(left, 1);
      return;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) atomicAdd(left, 1);
}

extern "C" int wait_selftest(int mode, unsigned long long limit_ns, int* status,
                             unsigned long long* elapsed, int* left, void* stream) {
  wait_selftest_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(mode, limit_ns, status,
                                                                          elapsed, left);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}
