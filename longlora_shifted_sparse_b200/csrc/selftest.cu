// Self-test of the device-side failure path: one CTA waits on an mbarrier that nothing
// ever arrives on. The bounded wait (the same code every tcgen05 kernel uses) must give up
// after `limit_ns`, record the timeout in the status word and return, leaving the CUDA
// context usable. No trap, no fault, no unbounded spin.
#include "common.cuh"
#include "fastmath.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace s2 {
namespace {

using namespace sm100;

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(unsigned* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ AbortState abort_state;
  if (threadIdx.x == 0) {
    abort_state_init(abort_state, status, limit_ns, 0);
    mbar_init(smem_addr(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  const Abort ab{smem_addr(&abort_state)};
  mbar_wait(smem_addr(&bar), 0, ab);  // nothing arrives: expires by design
}

// Even elements of each pair through the packed two-value form, the rest through the scalar
// one, so that a single comparison covers both.
__global__ void exp2_poly_kernel(const float* x, float* y, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    if ((i & 1) == 0 && i + 1 < n) {
      float a, b;
      f2unpack(exp2_poly2(f2pack(x[i], x[i + 1])), a, b);
      y[i] = a;
    } else {
      y[i] = exp2_poly(x[i]);
    }
  }
}

}  // namespace

cudaError_t launch_exp2_poly_selftest(const float* x, float* y, int n, cudaStream_t st) {
  exp2_poly_kernel<<<(n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024, 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(unsigned* status, uint64_t limit_ns, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  wait_timeout_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace s2
