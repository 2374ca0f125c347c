// Internal interface of the small-M projection kernels (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace mtpv {

// Rows of 4 Kd bytes that fit in 227 KB of shared memory: at least 1 for every
// supported Kd (<= 58112); the int4 path takes passes of min(8, this) rows.
size_t lm_head_max_smem_rows(int Kd);

// Device scratch of launch_lm_head for this shape (256-byte aligned; 0 when
// the shape needs none): rows past 8 of the bf16 head run on the tensor-
// memory kernel, whose first word is its error word (nonzero after the call:
// a bounded device wait gave up and y is not valid).
size_t lm_head_scratch_bytes(int M, int Kd, int fmt);

// y[M, N] = x[M, Kd] . Wd[N, Kd]^T; fmt is an mtpv_wfmt.  Arguments are
// validated by the caller; scratch holds lm_head_scratch_bytes(M, Kd, fmt).
cudaError_t launch_lm_head(const void *x, int M, int Kd, int N, const void *w, const void *scales,
                           int fmt, float *y, void *scratch, cudaStream_t s);

// Both heads of a verify step in one launch: yt[Mt, N] = xt . W^T (bf16 head)
// and yd[Md, N] = xd . deq(Wq, S)^T (int4 group-64 head), same Kd and N.
// lm_heads_pair_ok tells whether the fused kernel takes these shapes and
// pointers; otherwise the heads run as two launch_lm_head calls.  `work` is
// kHeadsPairWorkBytes of device scratch (the fused kernel's work counter,
// cleared on the stream before the kernel).
constexpr size_t kHeadsPairWorkBytes = 256;
bool lm_heads_pair_ok(int Mt, int Md, int Kd, const void *scales);
cudaError_t launch_lm_heads_pair(const void *xt, int Mt, const void *w, float *yt, const void *xd,
                                 int Md, const void *wq, const void *scales, float *yd, int Kd,
                                 int N, void *work, cudaStream_t s);

// Int4 group-64 projection y[M, N] = x . deq(wq, scales)^T for decoder
// layers and the batched int4 head (any N; M rows in passes of up to 32, one
// launch per pass, the weights read once per pass).  With silu_mul, N is a
// gate half and an up half and y[M, N/2] = silu(gate) * up.  ws holds
// int4_proj_workspace_bytes(M, Kd, N, silu_mul) bytes: the error word, one
// ticket counter per SM (each call returns them to zero: zero the workspace
// once before its first use, or pass reset_tickets to clear them on the
// stream first) and the partial sums of tiles split between SMs.  x, wq and
// scales 16-byte aligned.
size_t int4_proj_workspace_bytes(int M, int Kd, int N, bool gate_up);
cudaError_t launch_int4_proj(const void *x, int M, int Kd, int N, const void *wq, const void *scales,
                             float *y, int ldy, bool silu_mul, void *ws, bool reset_tickets, cudaStream_t s);

}  // namespace mtpv
