// Self-test of the bounded-wait protocol every pipelined kernel of the library
// follows, on one CTA: a wait that gives up records QLORA_ERR_TIMEOUT in the
// status word and sets the CTA's abort flag, the other warps leave their own
// waits on that flag, the copies the CTA still has in flight are waited for
// (again bounded), and the tensor memory the CTA holds is freed before it
// returns.  Here the wait is on an mbarrier that nothing completes, with a
// caller-chosen limit, so the protocol runs to its end on every launch.
#pragma once

#include "nf4_device.cuh"
#include "sm100_ptx.cuh"

namespace qlora {

constexpr int kSelftestThreads = 128;
constexpr uint32_t kSelftestCopyBytes = 256;

__global__ void __launch_bounds__(kSelftestThreads, 1)
    bounded_wait_selftest_kernel(const uint8_t *src, uint32_t *status, uint64_t limit_ns) {
  __shared__ __align__(128) uint8_t buf[kSelftestCopyBytes];
  __shared__ uint64_t never, copied;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&never, 1);
    ptx::mbar_init(&copied, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) ptx::tmem_alloc(&tmem_slot, 32);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  if (threadIdx.x == 0) {  // a copy in flight while the wait runs out
    ptx::mbar_arrive_expect_tx(&copied, kSelftestCopyBytes);
    ptx::bulk_g2s(buf, src, kSelftestCopyBytes, &copied);
  }
  // every warp waits; the first lane to give up records the timeout and tells
  // the others through the abort flag
  if (!ptx::mbar_wait_for(&never, 0, &abort_flag, limit_ns) && (threadIdx.x & 31) == 0) {
    raise_status(status, QLORA_ERR_TIMEOUT);
    *reinterpret_cast<volatile int *>(&abort_flag) = 1;
  }
  // drain: the copy completes before the CTA leaves (bounded by the normal limit)
  if (threadIdx.x == 0 && !ptx::mbar_wait(&copied, 0, nullptr)) raise_status(status, QLORA_ERR_CUDA);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 32);
    ptx::tmem_relinquish();
  }
}

}  // namespace qlora
