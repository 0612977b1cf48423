// Self-test of the failure path every kernel of the library relies on: a
// bounded mbarrier wait that expires records a bit in the per-device error
// word and returns, leaving the context usable. One thread waits on a
// barrier that nothing arrives on; no fault, trap or unbounded wait is
// involved.
#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

__global__ void __launch_bounds__(32) selftest_wait_kernel(unsigned* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
    // phase 0 never completes: the wait must give up after limit_ns
    if (!mbar_wait_for(smem_u32(&bar), 0, &abort_flag, limit_ns)) atomicOr(err, ERR_WAIT_SELFTEST);
  }
}

int launch_selftest_wait(unsigned* err, uint64_t limit_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
