// Self-test of the bounded waits (failure detection without a GPU fault).
// One block with the role layout of the tensor-core kernels: warp 0 holds a
// tensor-memory allocation, warp 1 waits on an mbarrier that nothing ever
// arrives at (a phase that never completes), warps 2-3 wait on a second such
// barrier with the production limit.  Warp 1's wait gives up after `limit_ns`,
// records ST_TIMEOUT in the device status word and raises the block's abort
// flag; warps 2-3 see the flag and return; warp 0 frees its tensor memory and
// the kernel ends.  No copies are in flight at any point.
#include "internal.h"
#include "tc_common.cuh"

namespace svg {
namespace {

__global__ void __launch_bounds__(128, 1) k_selftest_wait(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    tc::mbar_init(bars + 0, 1);
    tc::mbar_init(bars + 1, 1);
    abort_word = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&tmem_slot, 32);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) {
    tc::mbar_wait_warp(bars + 0, 0, abort_flag, status, limit_ns);   // nothing arrives: times out
  } else if (warp >= 2) {
    tc::mbar_wait_warp(bars + 1, 0, abort_flag, status);             // ends on the abort flag
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_slot, 32);
  }
}

}  // namespace

cudaError_t selftest_wait_run(uint64_t limit_ns, cudaStream_t st) {
  k_selftest_wait<<<1, 128, 0, st>>>(limit_ns, status_word());
  note_launch();
  return cudaGetLastError();
}

}  // namespace svg
