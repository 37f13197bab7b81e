// Self-tests.
//
// 1. The library's failure detection: a bounded mbarrier wait that
// must run out.  Every wait in the tensor-core kernels goes through
// sm100::mbar_wait, which gives up after a limit and lets the kernel set the
// device error word and wind down instead of hanging.  This kernel waits,
// with a caller-given limit, on a shared-memory mbarrier that no thread ever
// arrives at, so the wait runs out by construction.  It issues no TMA copy
// and no MMA and holds no tensor memory, so nothing is in flight when the
// wait gives up and the CTA exits cleanly.
//
// 2. The FMA-pipe exponential of the attention softmax (exp2_poly_x2, off by
// default, selected per head dimension at build time): evaluates the same
// device function on an array, so a test can hold it to its error bound.
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

// y[i] = 2^x[i] by exp2_poly_x2, two elements per call (the last one
// paired with itself when n is odd).
__global__ void __launch_bounds__(256) exp2_poly_kernel(const float* __restrict__ x,
                                                        float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = i + 1 < n ? x[i + 1] : a;
  float ya, yb;
  unpack_f32x2(exp2_poly_x2(pack_f32x2(a, b)), ya, yb);
  y[i] = ya;
  if (i + 1 < n) y[i + 1] = yb;
}

}  // namespace

cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t s) {
  const int pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout(unsigned long long limit_ns, unsigned* err, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace dsa
