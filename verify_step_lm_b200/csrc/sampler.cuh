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

// Result of one draft position (verify): the token drawn there as if the
// first rejection were at that position, whether its draft token was
// accepted, and its status.
struct PosRecord {
    int x, accept, status, pad;
};

// One workspace slot per logits row.  The statistics kernel writes the row's
// RowStats; in verify mode the draw kernel then replaces the slot of target
// row i with position i's PosRecord (no one reads that row's statistics
// afterwards).
union RowSlot {
    RowStats st;
    PosRecord rec;
};

// A verify call's per-position inputs carried by value in the launch
// parameters, so that a call whose inputs start in host memory needs no copy
// for them: at most kInlinePositions positions (B (K + 1)).
constexpr int kInlinePositions = 64;
struct SamplerInline {
    int32_t drafts[kInlinePositions];  // [B, K]
    float u_acc[kInlinePositions];     // [B, K]
    float u_samp[kInlinePositions];    // [B, K+1]
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
    RowSlot *slots;       // [rows]
    unsigned int *counters;  // verify: [B]; zeroed by the statistics kernel
    double *ecache;       // [rows][V]: exp((l_j - m)/T) of kept tokens, 0 elsewhere (T > 0), or null
    int wait_polls;       // polls of a bounded device-side wait before it gives up (set by launch_sampler)
    int inline_inputs = 0;  // verify: drafts / u_acc / u_samp are read from inl instead
    SamplerInline inl;
};

// Process-wide bound of the sampler's device-side waits, in polls (< 0: the
// default); see mtpv_set_wait_polls.
void set_wait_polls(int polls);

// Launches the statistics kernel over `rows` logits rows, then the draw
// kernel (one cluster per draft position in verify mode, per row otherwise).
cudaError_t launch_sampler(const SamplerParams &p, int rows, cudaStream_t stream);

}  // namespace mtpv
