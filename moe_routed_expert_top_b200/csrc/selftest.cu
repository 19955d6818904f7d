// selftest.cu - moe_selftest_bounded_wait: runs the pipeline wait every kernel
// of this library uses (mbar_wait, mbar_wait_until in ptx.cuh) on mbarriers
// that nothing ever arrives on, so that a caller can check on its own GPU that
// a stalled pipeline ends with MOE_DEV_TIMEOUT in the status word instead of a
// hung kernel, and that the teardown that follows (abort flag seen by the
// CTA's other waiting thread, a drain against a shared deadline, tensor memory
// freed) completes.
//
// The kernel issues no copy and no MMA, so nothing is in flight when its waits
// give up; its tensor memory is allocated and freed exactly as the GEMMs do it.
#include <cuda_runtime.h>

#include <cstdint>

#include "moe.h"
#include "ptx.cuh"

namespace moe {
namespace {

// One CTA of 64 threads. Thread 0 waits on `lonely` with the caller's limit and
// raises the CTA's abort flag when it gives up; thread 32 waits on `other` with
// a limit ten times longer and must return as soon as it sees that flag; then
// thread 0 drains `lonely` against a deadline `limit_ns` ahead. Warp 1 holds 32
// columns of tensor memory throughout and frees them at the end.
// result[0..5] = {thread 0 returned true, its wait in ns, thread 32 returned
// true, its wait in ns, the drain returned true, the drain in ns}.
__global__ void __launch_bounds__(64, 1)
    bounded_wait_kernel(uint64_t limit_ns, int32_t* status, int64_t* result) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  const uint32_t lonely = smem_u32(&bars[0]);
  const uint32_t other = smem_u32(&bars[1]);
  if (threadIdx.x == 0) {
    mbar_init(lonely, 1);
    mbar_init(other, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  if (threadIdx.x >= 32) tmem_alloc(smem_u32(&tmem_slot), 32);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    const bool ok = mbar_wait(lonely, 0, &abort_flag, status, limit_ns);
    const uint64_t t1 = globaltimer_ns();
    // teardown drain as the GEMMs do it after an abort: bounded by one deadline
    const bool drained = mbar_wait_until(lonely, 0, t1 + limit_ns);
    const uint64_t t2 = globaltimer_ns();
    result[0] = ok ? 1 : 0;
    result[1] = static_cast<int64_t>(t1 - t0);
    result[4] = drained ? 1 : 0;
    result[5] = static_cast<int64_t>(t2 - t1);
  } else if (threadIdx.x == 32) {
    const uint64_t t0 = globaltimer_ns();
    const bool ok = mbar_wait(other, 0, &abort_flag, status, 10 * limit_ns);
    result[2] = ok ? 1 : 0;
    result[3] = static_cast<int64_t>(globaltimer_ns() - t0);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x >= 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_selftest_bounded_wait(int64_t limit_ns, int32_t* dev_status,
                                                int64_t* dev_result, moe_stream_t stream) {
  if (dev_status == nullptr || dev_result == nullptr) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dev_result) & 7u) != 0) return MOE_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 1000000000) return MOE_ERR_INVALID_ARG;
  moe::bounded_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ns), dev_status, dev_result);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
