// Self-test of the device-timeout path that every tensor-core kernel shares.
//
// One thread block allocates tensor memory, waits on an mbarrier that nothing
// ever completes, and so runs the bounded wait (tc::mbar_wait) to its limit:
// after kWaitLimitNs (2 s) of %globaltimer time the first thread to get there
// raises the block's abort flag, the others give up when they see it, the
// block frees its tensor memory and records a device timeout in the status
// word, which is what a forward kernel does when one of its waits runs out.
// Nothing here can hang: every wait ends by the clock, and the kernel uses no
// trap, no assert and no invalid address.
#include "common.cuh"
#include "launch.h"
#include "tc_common.cuh"

namespace kata {
namespace {

using namespace tc;

constexpr int kSelftestThreads = 64;      // warp 1 owns the tensor-memory allocation
constexpr uint32_t kSelftestCols = 32;    // the smallest allocation

__global__ void __launch_bounds__(kSelftestThreads, 1) wait_timeout_selftest_kernel(unsigned *status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);          // one arrival would complete the phase; none comes
    abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kSelftestCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;
  volatile int *abort = &abort_flag;
  const bool completed = mbar_wait(&bar, 0, abort);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kSelftestCols);
  if (threadIdx.x == 0 && (*abort || !completed)) flag_status(status, kStatusDeviceTimeout);
}

}  // namespace

cudaError_t selftest_wait_timeout(unsigned *status, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, kSelftestThreads, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace kata
