// Internal interface of the small-M projection kernels (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace mtpv {

// Rows of activations of length Kd that one launch can stage (as fp32) in shared memory.
size_t lm_head_max_smem_rows(int Kd);

// y[M, N] = x[M, Kd] . Wd[N, Kd]^T; fmt is an mtpv_wfmt.  Arguments are
// validated by the caller.
cudaError_t launch_lm_head(const void *x, int M, int Kd, int N, const void *w, const void *scales,
                           int fmt, float *y, cudaStream_t s);

}  // namespace mtpv
