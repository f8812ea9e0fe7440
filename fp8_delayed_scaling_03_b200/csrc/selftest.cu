// selftest.cu -- the bounded waits every kernel relies on, exercised on
// purpose (fp8_wait_selftest).  One CTA: warp 0 waits on a global flag with
// the flag protocol of the stream-K fixup, warp 1 on an mbarrier of its own
// shared memory with the protocol of the GEMM pipelines, each with the
// caller's time limit.  A flag that nothing sets and the mbarrier (which
// nothing ever arrives on) make the waits run out: each records
// FP8_ERR_DEVICE_TIMEOUT in the device status word and returns, and the kernel
// ends normally, so the context stays usable.  No wait here can outlast its
// limit.
#include "device.cuh"
#include "internal.h"
#include "launch.h"

namespace fp8lin {
namespace {

__global__ void __launch_bounds__(64) wait_selftest_kernel(const uint32_t* flag, int* status, int* results,
                                                           uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    const bool ok = flag_wait_warp(flag, status, nullptr, limit_ns);
    if ((threadIdx.x & 31) == 0) results[0] = ok ? 1 : 0;
  } else if ((threadIdx.x & 31) == 0) {
    results[1] = mbar_wait(&bar, 0, status, nullptr, limit_ns) ? 1 : 0;
  }
}

}  // namespace

cudaError_t launch_wait_selftest(const uint32_t* flag, int* status, int* results, uint64_t limit_ns,
                                 cudaStream_t s) {
  return launch_pdl(wait_selftest_kernel, dim3(1), dim3(64), 0, s, flag, status, results, limit_ns);
}

}  // namespace fp8lin
