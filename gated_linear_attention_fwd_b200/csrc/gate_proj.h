// gate_proj.h -- launcher declarations of the gate projection kernels (internal
// to libdig.so).
#pragma once
#include <cstddef>

#include <cuda_runtime.h>

namespace dig {

// Dynamic shared memory of the forward (backward = false) or backward kernel.
size_t gate_proj_smem_bytes(int D, int R, int dk, bool backward);
// z = (x W1) W2 + b, u = x W1 (u optional).
cudaError_t launch_gate_proj_fwd(const void* x, const float* W1, const float* W2, const float* b, float* z, float* u,
                                 long long rows, int D, int R, int dk, int tin, cudaStream_t s);
// Zeroes dW1, dW2 (and db) on the stream, then dx, dW1, dW2, db from d log alpha.
cudaError_t launch_gate_proj_bwd(const void* x, const float* W1, const float* W2, const float* u, const float* z,
                                 const float* dla, float inv_tau, void* dx, float* dW1, float* dW2, float* db,
                                 long long rows, int D, int R, int dk, int tin, int tout, cudaStream_t s);

}  // namespace dig
