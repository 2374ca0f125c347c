// Internal interface of the tcgen05 LM-head kernels (not part of the ABI).
#pragma once

#include <cuda_runtime.h>

namespace mtpv {

// Whether the tensor-memory kernels take M activation rows (9..64) of
// length Kd (a multiple of 64) with these 16-byte aligned pointers.
bool lm_head_tc_ok(int M, int Kd, const void *x, const void *w);

// y[M, N] = x[M, Kd] . W[N, Kd]^T (bf16 x and W, fp32 y [M, N]) in one pass
// over W.  err: a device word; a bounded wait that gave up ORs a nonzero
// code into it (the outputs of that launch are then not valid).
cudaError_t launch_lm_head_bf16_tc(const void *x, int M, int Kd, int N, const void *w, float *y,
                                   unsigned int *err, cudaStream_t s);

}  // namespace mtpv
