// Internal interface of the sampler kernels (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mtpv {

// Warp statistics of one row, written by the row's cluster.
struct RowStats {
    double Z;     // sum over the row of exp((l - m)/T)
    double Zk;    // mass of the kept (top-p) tokens
    float m;      // max logit
    float lmin;   // min logit
    float lstar;  // cut logit: token j is kept iff l_j > lstar, or l_j == lstar and j <= idxstar
    int idxstar;
    int argmax;   // lowest index among equal maxima
    int status;   // MTPV_ROW_OK or MTPV_ROW_NONFINITE
};

struct SamplerParams {
    const float *tl;        // verify: target logits [B, K+1, V]; sample: logits [R, V]
    const float *dl;        // verify: draft logits [B, K, V]
    const int32_t *drafts;  // verify: [B, K]
    const float *u_acc;     // verify: [B, K]
    const float *u_samp;    // verify: [B, K+1]; sample: [R]
    int B, K, V;
    float T, top_p;
    int verify;
    int32_t *out_tokens;  // verify: [B, K+1]; sample: [R]
    int32_t *out_acc;     // verify: [B]
    int32_t *row_status;  // verify: [B]; sample: [R]; may be null
    RowStats *stats;      // [rows]
    unsigned int *counters;  // verify: [B], zero on entry
    double *ecache;       // [rows][V]: exp((l_j - m)/T) of every row (T > 0), or null
};

size_t sampler_smem_bytes();
int sampler_cluster_size();
cudaError_t launch_sampler(const SamplerParams &p, int rows, cudaStream_t stream);

}  // namespace mtpv
