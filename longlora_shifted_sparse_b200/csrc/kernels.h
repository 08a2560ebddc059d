// Host-side launchers of the library's kernels (internal; not part of the C ABI).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace s2 {

// RoPE + PI stage: q, k -> rotated head-major copies and the (cos, sin) table.
cudaError_t launch_rope_table(const Params& p, cudaStream_t st);
cudaError_t launch_rope_pi(const Params& p, bool bf16, cudaStream_t st);

// CUDA-core kernels (any valid shape).
cudaError_t launch_simt_fwd(const Params& p, bool bf16, cudaStream_t st);
cudaError_t launch_bwd_rowsum(const Params& p, bool bf16, cudaStream_t st);
cudaError_t launch_simt_dq(const Params& p, bool bf16, cudaStream_t st);
cudaError_t launch_simt_dkdv(const Params& p, bool bf16, cudaStream_t st);

// Failure-path self-test: a bounded wait that must expire and set *status.
cudaError_t launch_wait_timeout_selftest(unsigned* status, uint64_t limit_ns, cudaStream_t st);

// Elementwise y = 2^x with the FMA-pipe polynomial the softmax uses (for testing it).
cudaError_t launch_exp2_poly_selftest(const float* x, float* y, int n, cudaStream_t st);

}  // namespace s2
