// Self-test of the library's failure detection: a bounded mbarrier wait that
// must run out.  Every wait in the tensor-core kernels goes through
// sm100::mbar_wait, which gives up after a limit and lets the kernel set the
// device error word and wind down instead of hanging.  This kernel waits,
// with a caller-given limit, on a shared-memory mbarrier that no thread ever
// arrives at, so the wait runs out by construction.  It issues no TMA copy
// and no MMA and holds no tensor memory, so nothing is in flight when the
// wait gives up and the CTA exits cleanly.
#include "sm100.cuh"

namespace dsa {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(unsigned long long limit_ns,
                                                          unsigned* err) {
  __shared__ __align__(8) unsigned long long bar_storage;
  const uint32_t bar = sm100::smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    sm100::mbar_init(bar, 1);
    sm100::fence_mbar_init();
  }
  __syncwarp();
  // phase 0 of a fresh barrier completes only after one arrival; none comes
  const bool done = sm100::mbar_wait(bar, 0u, limit_ns);
  if (!done && threadIdx.x == 0) flag_error(err, kErrTimeout);
}

}  // namespace

cudaError_t launch_wait_timeout(unsigned long long limit_ns, unsigned* err, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace dsa
