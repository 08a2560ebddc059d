// Host launchers of the tcgen05 (tensor-core) kernels. Preconditions (checked by the
// caller): bf16 tensors, d == 128, G % 256 == 0 (so G/2 is a whole number of 128-row
// tiles), N % G == 0.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace s2 {

cudaError_t launch_tc_fwd(const Params& p, cudaStream_t st);
cudaError_t launch_tc_bwd_dkdv(const Params& p, cudaStream_t st);
cudaError_t launch_tc_bwd_dq(const Params& p, cudaStream_t st);

}  // namespace s2
