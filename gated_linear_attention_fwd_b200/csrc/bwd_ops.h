// bwd_ops.h -- launcher declarations of the epilogue and SREM conv backward
// kernels (internal to libdig.so).
#pragma once
#include <cuda_runtime.h>

namespace dig {

// Conv backward: zeroes dw / dbias on the stream (when given), then dx, dw, dbias.
cudaError_t launch_srem_bwd(const void* x, const float* w, const void* dy, void* dx, float* dw, float* dbias, int B,
                            int Hg, int Wg, int C, int mode, int tin, int tout, cudaStream_t s);
// Epilogue backward: zeroes d_gamma on the stream (when given), then d_o, d_r, d_gamma.
cudaError_t launch_epilogue_bwd(const void* o, const void* r, const float* gamma, float eps, const void* dy,
                                void* d_o, void* d_r, float* d_gamma, long long rows, int dv, int tin, int tout,
                                cudaStream_t s);

}  // namespace dig
