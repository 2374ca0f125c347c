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

// The int4 group-64 head on the same path: M in 9..64, Kd a multiple of 512
// (at most 16384), x, wq and scales 16-byte aligned.
bool lm_head_tc_int4_ok(int M, int Kd, const void *x, const void *wq, const void *scales);

// Scratch of launch_lm_head_int4_tc: the error word, the activations'
// power-of-two factors and their fp16 copy.
size_t lm_head_int4_tc_scratch_bytes(int M, int Kd);

// y[M, N] = x . deq(wq, scales)^T in one pass over the nibbles (a staging
// launch, then the tensor-memory kernel); scratch's first word is the error
// word, as for the bf16 kernel.
cudaError_t launch_lm_head_int4_tc(const void *x, int M, int Kd, int N, const void *wq, const void *scales,
                                   float *y, void *scratch, cudaStream_t s);

}  // namespace mtpv
