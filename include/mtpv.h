/*
 * mtpv.h -- C ABI of libmtpv, the speculative-decoding verify step on NVIDIA
 * B200 (sm_100a).
 *
 * The verify step is the part of self-speculative (multi-token-prediction)
 * decoding that runs after the model's own MTP head has drafted K tokens:
 *   1. a small-M projection of the hidden states through the LM head: K+1
 *      target rows through the bf16 head and K draft rows through a
 *      group-64 int4 copy of the same head (hazakura.dev MTPLX notes,
 *      "4-layer architecture", Layer 0: small-matrix (M=3..6) shader and the
 *      draft-only 4-bit LM head that keeps the target's own precision);
 *   2. Leviathan-Chen rejection sampling with residual correction and a bonus
 *      token (devtrends.cc MTPLX overview, "no second model" section;
 *      hazakura.dev notes, Layer 2: draft -> parallel verify -> ratio
 *      acceptance -> residual correction -> bonus token), with temperature
 *      and top-p applied so that the output distribution equals plain
 *      sampling at those settings (devtrends.cc overview: temperature=0.6,
 *      top_p=0.95).
 *
 * Conventions shared by every call
 *   - All tensors are dense, row-major and owned by the caller.  Device
 *     pointers must be 16-byte aligned unless stated otherwise.
 *   - The library never allocates device memory and never synchronises the
 *     stream (except mtpv_verify_step_host, which is synchronous by design).
 *     Scratch memory is the caller's workspace; its size comes from the
 *     matching *_workspace_bytes query.  A workspace may be reused by later
 *     calls on the same stream but not by calls that overlap in time.
 *   - Every compute call is asynchronous on `stream` (NULL = legacy default
 *     stream).  Argument errors are returned synchronously and nothing is
 *     launched.  A launch failure returns MTPV_ERR_CUDA.
 *   - Errors in the DATA (a draft id outside [0, V), a non-finite logit) are
 *     reported per sequence in row_status; they never fault the GPU.
 *   - The caller supplies every uniform random number (fp32 in [0, 1)); the
 *     library holds no random-number generator.
 *   - The calling thread's current CUDA context must be the one that owns
 *     the pointers (the primary context of the device, as PyTorch sets it).
 */
#ifndef MTPV_H_
#define MTPV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MTPV_API __attribute__((visibility("default")))
#else
#define MTPV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *mtpv_stream;

typedef enum {
    MTPV_OK = 0,
    MTPV_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or parameter   */
    MTPV_ERR_UNSUPPORTED = 2, /* valid request this build does not handle    */
    MTPV_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required  */
    MTPV_ERR_CUDA = 4,        /* a CUDA call or kernel launch failed         */
    MTPV_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up          */
} mtpv_status;

/* Weight storage formats of mtpv_lm_head_smallm. */
typedef enum {
    MTPV_W_BF16 = 0,     /* w: bf16 [N, Kd]; scales unused (NULL)             */
    MTPV_W_INT4_G64 = 1  /* w: uint8 [N, Kd/2], scales: bf16 [N, Kd/64]       */
} mtpv_wfmt;

/* Per-sequence data status written to row_status. */
#define MTPV_ROW_OK 0
#define MTPV_ROW_BAD_DRAFT 1    /* a draft token id outside [0, V)          */
#define MTPV_ROW_NONFINITE 2    /* a NaN or +-inf logit in one of its rows  */
#define MTPV_ROW_TIMEOUT 3      /* a bounded device-side wait gave up: the  */
                                /* sequence's outputs are not valid         */

/* Library version: major*10000 + minor*100 + patch. */
MTPV_API int mtpv_version(void);

/* Static, human-readable name of a status code (never NULL). */
MTPV_API const char *mtpv_status_string(mtpv_status st);

/* ------------------------------------------------------------------------
 * mtpv_set_wait_polls -- bound of the sampler's device-side waits.
 *
 * The sampler kernels bring slices of logits and weights into shared memory
 * with bulk copies and wait on an mbarrier for them.  Every such wait polls
 * at most `polls` times (process-wide, taken at each launch); when the bound
 * runs out the sequence (or sampled row) is reported as MTPV_ROW_TIMEOUT
 * with out_accepted = -1 and tokens -1, and the kernel waits once more, with
 * the default bound, for the copy it issued before it reads on or exits.
 * polls < 0 restores the default (2^20 polls); 0 makes every first wait give
 * up at once, which exercises the timeout path deterministically (tests).
 * Not synchronised with launches in flight on other host threads.
 * ---------------------------------------------------------------------- */
MTPV_API void mtpv_set_wait_polls(int polls);

/* ------------------------------------------------------------------------
 * mtpv_lm_head_smallm -- small-M weight-streaming projection.
 *
 * Passage: hazakura.dev MTPLX notes, Layer 0 (a matmul specialised for M=3..6
 * rows; a 4-bit LM head used for drafting while the target keeps its own
 * precision); gist.science BaseRT explainer, methodology (decode GEMV per
 * quantisation format with dequantisation inside the inner loop).
 *
 *   y[m][n] = sum_k x[m][k] * Wd[n][k],  0 <= m < M, 0 <= n < N   (fp32 out)
 *
 *   x       device, bf16 [M, Kd] row-major (activations / hidden states).
 *   M       rows, 1 <= M <= 64.
 *           M <= 8: mma.sync on the tensor cores (fp32 accumulation), rows
 *           staged in shared memory.  MTPV_W_INT4_G64 dequantises exactly to
 *           fp16 (activations scaled per row by a power of two) with one
 *           fresh accumulator per 64-weight group: through per-warp
 *           shared-memory rings when Kd is a multiple of 512, the scales
 *           are 16-byte aligned and (M + 1)(2 Kd + 16) + Kd/2 <= 75776
 *           bytes, else with direct register loads (the same bits).
 *           9 <= M <= 64, MTPV_W_BF16: one pass over the weights on
 *           tcgen05 (fifth-generation tensor cores, fp32 accumulators in
 *           tensor memory, weights streamed by TMA; rows padded to a
 *           multiple of 16), for any Kd.
 *           9 <= M <= 32, MTPV_W_INT4_G64, x, w and scales 16-byte aligned:
 *           one pass over the weights streamed by TMA through shared
 *           memory into mma.sync (the nibble n becomes the bf16 value n - 8
 *           exactly; the computation of mtpv_int4_proj, two to four n-tiles
 *           of 8 rows per pass).
 *           33 <= M <= 64, MTPV_W_INT4_G64: one pass on tcgen05 when Kd is a
 *           multiple of 512 and at most 8192 and x, w and scales are 16-byte
 *           aligned (the nibbles are dequantised to exact fp16 (n - 8) s f,
 *           f a per-row power of two, and the activations staged once as
 *           fp16 times a per-row power of two).  Other int4 shapes go in
 *           passes of min(8, floor(232448 / (4 Kd))) rows, re-reading the
 *           weights once per pass.
 *   Kd      reduction length, a positive multiple of 64, at most 58112.
 *   N       output columns (vocabulary rows of the head), N >= 1.
 *   w       device weights, layout per fmt:
 *             MTPV_W_BF16:     bf16 [N, Kd] (nn.Linear out x in layout);
 *                              Wd = w.
 *             MTPV_W_INT4_G64: uint8 [N, Kd/2]; weight k of row n is the low
 *                              nibble of byte k/2 when k is even, the high
 *                              nibble when k is odd; the nibble stores q+8
 *                              for q in [-8, 7];
 *                              Wd[n][k] = scales[n][k/64] * (nibble - 8).
 *   scales  device bf16 [N, Kd/64] for MTPV_W_INT4_G64 (2-byte aligned);
 *           ignored for MTPV_W_BF16.
 *   y       device fp32 [M, N] row-major, fully overwritten (4-byte aligned).
 *   ws, ws_bytes  workspace of mtpv_lm_head_workspace_bytes() bytes, 256-byte
 *           aligned (may be NULL when the query returns 0, as it does for
 *           M <= 8).  For M > 8 its first 32-bit word is an error word,
 *           cleared by the call: nonzero once the call has run means a
 *           bounded device-side wait gave up and y is not valid (the kernel
 *           never hangs).  The rest holds, per path, the streamed kernel's
 *           ticket counters (cleared by the call) and partial sums, or the
 *           tcgen05 int4 kernel's staged activations.
 * Accumulation is fp32.  Errors: MTPV_ERR_INVALID_ARG for NULL pointers,
 * M/Kd/N out of range or misaligned x/w; MTPV_ERR_WORKSPACE when ws_bytes is
 * below mtpv_lm_head_workspace_bytes().
 * ---------------------------------------------------------------------- */
MTPV_API size_t mtpv_lm_head_workspace_bytes(int M, int Kd, int N, mtpv_wfmt fmt);
MTPV_API mtpv_status mtpv_lm_head_smallm(const void *x, int M, int Kd, int N, const void *w,
                                const void *scales, mtpv_wfmt fmt, float *y, void *ws,
                                size_t ws_bytes, mtpv_stream stream);

/* ------------------------------------------------------------------------
 * mtpv_lm_head_pair -- the two projections of a verify step in one call:
 *
 *   yt[Mt, N] = xt[Mt, Kd] . W^T            (bf16 head, as MTPV_W_BF16)
 *   yd[Md, N] = xd[Md, Kd] . deq(wq, s)^T   (int4 group-64 head, as
 *                                            MTPV_W_INT4_G64)
 *
 * Passage: hazakura.dev MTPLX notes, Layer 0 (the target head at full
 * precision, the draft through a 4-bit copy) and its cached-graph item (one
 * fixed launch sequence per step).  Arguments as in mtpv_lm_head_smallm, the
 * same Kd and N for both heads.  When 1 <= Mt <= 8, 1 <= Md <= 8, Kd is a
 * multiple of 512, the scales are 16-byte aligned and the staging fits in
 * shared memory (2 Mt (Kd + 32) + (Md + 1)(2 Kd + 16) + Kd/2 + 39168 <=
 * 232192 bytes; Mt = 8, Md = 8 at Kd = 5120 does), both heads run in ONE
 * persistent kernel: 3 of every CTA's 16 warps first stream the int4 head
 * through their shared-memory rings (bound by dequantisation, not by HBM) and
 * then join the other 13 on the bf16 head, whose 16-row tiles every warp
 * takes one at a time from a counter in `ws`, so the bf16 stream keeps HBM
 * busy to the end.  Otherwise the call makes the two mtpv_lm_head_smallm
 * launches.
 * Either way the values are those mtpv_lm_head_smallm gives (same
 * arithmetic, bit for bit).
 * ws, ws_bytes: at least mtpv_lm_head_pair_workspace_bytes() bytes (256,
 * plus each head's mtpv_lm_head_workspace_bytes() when the heads run as two
 * launches), 256-byte aligned; need not be initialised (the call clears its
 * counter on `stream`).  Errors: as mtpv_lm_head_smallm, and
 * MTPV_ERR_WORKSPACE.
 * ---------------------------------------------------------------------- */
MTPV_API size_t mtpv_lm_head_pair_workspace_bytes(int Mt, int Md, int Kd, int N);
MTPV_API mtpv_status mtpv_lm_head_pair(const void *xt, int Mt, const void *w, float *yt,
                                       const void *xd, int Md, const void *wq,
                                       const void *scales, float *yd, int Kd, int N, void *ws,
                                       size_t ws_bytes, mtpv_stream stream);

/* ------------------------------------------------------------------------
 * mtpv_int4_proj / mtpv_int4_gate_up -- small-M decoder-layer projections
 * with int4 group-64 weights (the verify pass's other matmuls: attention
 * qkv and o, MLP gate/up and down).
 *
 * Passage: hazakura.dev MTPLX notes, Layer 0 (matmuls specialised for
 * M = 3..6 rows); gist.science BaseRT explainer, methodology (per-format
 * decode GEMV with dequantisation in the inner loop; fused op chains).
 *
 *   mtpv_int4_proj:     y[M, N] = x[M, Kd] . deq(wq, scales)^T
 *   mtpv_int4_gate_up:  h[M, F] = silu(x . G^T) * (x . U^T), where rows
 *                       0..F-1 of the [2F, Kd] head are G (gate) and rows
 *                       F..2F-1 are U (up); silu(g) = g / (1 + e^-g).
 *
 *   x       device bf16 [M, Kd] (16-byte aligned), 1 <= M <= 64.
 *   wq      device uint8 [N, Kd/2] (N = 2F for gate_up), MTPV_W_INT4_G64
 *           nibble order; scales device bf16 [N, Kd/64]; both 16-byte
 *           aligned.
 *   Kd      a positive multiple of 64, at most 2^20.  One launch per pass:
 *           M <= 8 in one pass of one MMA n-tile; more rows in passes of up
 *           to 32 (two to four n-tiles of 8 rows, a second kernel with the
 *           same arithmetic); the weights are read once per pass.
 *   y, h    device fp32 [M, N] / [M, F], fully overwritten.
 * Arithmetic: bf16 mma.sync of exactly dequantised weights (the nibble n
 * becomes the bf16 value n - 8) against the bf16 activations as given, a
 * fresh fp32 accumulator per 64-weight group multiplied by its scale.  The
 * weights stream through shared memory (TMA) in stages of 128 rows x 8
 * groups, and the list of stages is cut into one equal run per SM, so a
 * 128-row output tile may be split between neighbouring SMs; each of them
 * stores its partial sums in the workspace and the last to finish (a ticket
 * counter) adds them in SM order and writes the tile.  The summation order
 * depends only on the shapes and the GPU's SM count: results are
 * deterministic on a given GPU.
 * ws, ws_bytes: at least the matching *_workspace_bytes() bytes, 256-byte
 * aligned, zero-filled before the first call that uses it; every call
 * returns its ticket counters to zero, so one zeroing serves all later calls
 * on the same stream (calls that share a workspace must not run
 * concurrently).  The first 4 bytes are an error word: a bounded wait that
 * gave up ORs a nonzero code into it and that launch's outputs are not
 * valid; it stays set until the caller clears it.  Errors:
 * MTPV_ERR_INVALID_ARG, MTPV_ERR_WORKSPACE, MTPV_ERR_CUDA.
 * Launch: a pass of up to 8 rows is a programmatic dependent launch (it may
 * start while the kernel before it on the stream finishes, so that
 * back-to-back projections overlap one's start with the other's tail).  It
 * reads x, ws and y only after that kernel has completed, but it may read
 * wq and scales earlier: a preceding kernel that allows its dependents to
 * launch early (griddepcontrol.launch_dependents) must not write them.
 * ---------------------------------------------------------------------- */
MTPV_API size_t mtpv_int4_proj_workspace_bytes(int M, int Kd, int N);
MTPV_API mtpv_status mtpv_int4_proj(const void *x, int M, int Kd, int N, const void *wq,
                                    const void *scales, float *y, void *ws, size_t ws_bytes,
                                    mtpv_stream stream);
MTPV_API size_t mtpv_int4_gate_up_workspace_bytes(int M, int Kd, int F);
MTPV_API mtpv_status mtpv_int4_gate_up(const void *x, int M, int Kd, int F, const void *wq,
                                       const void *scales, float *h, void *ws, size_t ws_bytes,
                                       mtpv_stream stream);

/* ------------------------------------------------------------------------
 * mtpv_verify -- Leviathan-Chen verification of B independent sequences.
 *
 * Passages: devtrends.cc MTPLX overview and devtrends.ru page (exact rejection
 * sampling of Leviathan and Chen with residual correction; temperature 0.6 /
 * top_p 0.95 reproduce non-speculative sampling); hazakura.dev notes,
 * Layer 2 (ratio acceptance, residual correction, bonus token) and results
 * section (distribution identical, max_diff = 0.0; not greedy-only).
 *
 * Every row l (target or draft) is warped the same way:
 *   T > 0:  p_j = exp((l_j - max l)/T) / sum_i exp((l_i - max l)/T); tokens
 *           are ranked by (logit desc, index asc); rank r is kept iff the mass
 *           of the ranks before it is < top_p (top_p >= 1 keeps every token
 *           with p > 0); p'_j = p_j / (kept mass) for kept tokens, else 0.
 *   T == 0: p' is one-hot at the argmax (lowest index among equal maxima).
 * For sequence b with drafts d_0..d_{K-1} (p'_i from target row i, q'_i from
 * draft row i):
 *   accept d_i iff u_accept[b][i] < p'_i(d_i) / q'_i(d_i)
 *   (+inf when q'_i(d_i) == 0 < p'_i(d_i), 0 when both are 0); n = number of
 *   drafts accepted before the first rejection (K if none);
 *   n < K:  x ~ normalise(max(0, p'_n - q'_n))  (p'_n if that is all zero);
 *   n == K: x ~ p'_K (the bonus token);
 *   the draw is the inverse CDF in vocabulary order with u = u_sample[b][n]:
 *   x = min{k : sum_{j<=k} w_j > u * sum_j w_j}.
 *   Outputs: out_tokens[b] = d_0..d_{n-1}, x, then -1 up to K+1 entries;
 *   out_accepted[b] = n.
 *
 *   target_logits  device fp32 [B, K+1, V] (4-byte aligned)
 *   draft_logits   device fp32 [B, K, V]
 *   draft_tokens   device int32 [B, K]
 *   u_accept       device fp32 [B, K], values in [0, 1)
 *   u_sample       device fp32 [B, K+1], values in [0, 1)
 *   B >= 1, 1 <= K <= 16, 1 <= V <= 2^24 (B*(2K+1) <= 65535)
 *   temperature    >= 0 and finite; top_p in (0, 1] (values above 1 mean 1).
 *   out_tokens     device int32 [B, K+1];  out_accepted device int32 [B]
 *   row_status     device int32 [B] or NULL; MTPV_ROW_* per sequence.  A
 *                  sequence with a data error, or whose device-side wait ran
 *                  out of its bound (MTPV_ROW_TIMEOUT, mtpv_set_wait_polls),
 *                  gets out_accepted = -1 and out_tokens all -1.
 *   ws, ws_bytes   workspace of at least mtpv_verify_workspace_bytes(B, K, V)
 *                  bytes, 256-byte aligned.  It need not be initialised: the
 *                  call's first kernel clears what it needs.
 * Arithmetic: exp, sums, ratios and CDFs in fp64 on fp32 logits, every sum
 * in a fixed order (no floating-point atomics), so a call's outputs are the
 * same bits in every run.
 * Launch: two kernels, each launched as a programmatic dependent of the work
 * before it on `stream` (it may be scheduled while that work drains and
 * waits for its completion before reading its results).
 * ---------------------------------------------------------------------- */
MTPV_API size_t mtpv_verify_workspace_bytes(int B, int K, int V);
MTPV_API mtpv_status mtpv_verify(const float *target_logits, const float *draft_logits,
                        const int32_t *draft_tokens, const float *u_accept,
                        const float *u_sample, int B, int K, int V, float temperature,
                        float top_p, int32_t *out_tokens, int32_t *out_accepted,
                        int32_t *row_status, void *ws, size_t ws_bytes, mtpv_stream stream);

/* ------------------------------------------------------------------------
 * mtpv_verify_noalloc -- mtpv_verify without a caller-supplied workspace.
 * (The pages have no counterpart to this call; it is a convenience of this
 * library.)
 *
 * Some callers cannot hand us device scratch memory: a decode loop that must
 * never allocate once it runs (an allocation can synchronise the device and
 * stall the loop), a plug-in whose host framework owns all device memory and
 * forbids private cudaMalloc calls, or a hook that runs while a stream is
 * being captured, where an allocation would break the capture.  This entry
 * point takes exactly the inputs and outputs of mtpv_verify, with the same
 * meaning, layout and results, and allocates nothing: the kernel's scratch
 * (B ticket counters and one 40-byte statistics record per row) lives in a
 * fixed 64 KiB array compiled into the library, which every GPU that loads the
 * library keeps until the process exits.
 *
 *   Limit: round_up(4*B, 256) + round_up(40*B*(2K+1), 256) <= 65536 bytes
 *   (for K = 3, up to B = 230 sequences); larger requests return
 *   MTPV_ERR_UNSUPPORTED and launch nothing.  Other argument errors return
 *   MTPV_ERR_INVALID_ARG as in mtpv_verify.
 *   First call on a device: it looks up the array's device address once
 *   (cudaGetSymbolAddress, which may load the library's GPU code) and keeps
 *   it for the life of the process; make that first call before any stream
 *   capture, and do not call it again on a device after cudaDeviceReset (the
 *   kept address would then be stale).
 *   With no room for mtpv_verify's cached token weights, the draw recomputes
 *   each weight from the logits (one more fp64 exp per token it reads); the
 *   results are the same bits.
 *   Every call shares the one array and leaves its contents behind; each call
 *   clears the counters it needs in its first kernel.  Calls whose GPU work can
 *   overlap in time (different streams without ordering) race on the array
 *   and give wrong results: order them on one stream.
 *   It calls no cudaMalloc, cudaFree or allocating library routine.
 * ---------------------------------------------------------------------- */
MTPV_API mtpv_status mtpv_verify_noalloc(const float *target_logits, const float *draft_logits,
                                         const int32_t *draft_tokens, const float *u_accept,
                                         const float *u_sample, int B, int K, int V,
                                         float temperature, float top_p, int32_t *out_tokens,
                                         int32_t *out_accepted, int32_t *row_status,
                                         mtpv_stream stream);

/* ------------------------------------------------------------------------
 * mtpv_sample -- one draw from the warped distribution of each of R rows
 * (temperature + top-p exactly as in mtpv_verify, inverse CDF with u[r]).
 * This is the draft phase's own sampling step (hazakura.dev notes, Layer 2
 * "Draft"), used to draw draft tokens from q'.
 *
 *   logits     device fp32 [R, V];  u device fp32 [R] in [0, 1)
 *   out        device int32 [R] (-1 for a row with a non-finite logit or a
 *              timed-out device wait)
 *   row_status device int32 [R] or NULL (MTPV_ROW_OK / MTPV_ROW_NONFINITE /
 *              MTPV_ROW_TIMEOUT)
 *   1 <= R <= 65535, 1 <= V <= 2^24; ws as returned by the query.
 * ---------------------------------------------------------------------- */
MTPV_API size_t mtpv_sample_workspace_bytes(int R, int V);
MTPV_API mtpv_status mtpv_sample(const float *logits, int R, int V, float temperature, float top_p,
                        const float *u, int32_t *out, int32_t *row_status, void *ws,
                        size_t ws_bytes, mtpv_stream stream);

/* ------------------------------------------------------------------------
 * mtpv_draft_loop -- the draft phase that precedes a verify step: K draft
 * tokens per sequence, one position after the other.
 *
 * Passage: hazakura.dev MTPLX notes, Layer 2 "Draft" (the MTP head proposes
 * K tokens, each drawn from the draft distribution through the 4-bit LM
 * head) and Layer 0 (the draft head's 4-bit copy of the LM head).  The MTP
 * head's own transformer layers are outside this library: the caller passes
 * the draft hidden state of every position.
 *
 * For position i = 0..K-1, in order:
 *   draft_logits[b][i] = h_draft[b][i] . deq(w_draft, s_draft)^T
 *   out_drafts[b][i]   = one draw from q'_i (temperature + top-p exactly as
 *                        mtpv_verify; inverse CDF with u_draft[b][i])
 *
 *   w_draft, s_draft  int4 group-64 head, as MTPV_W_INT4_G64 [V, h]
 *   h_draft           device bf16 [B, K, h] (16-byte aligned)
 *   u_draft           device fp32 [B, K] in [0, 1)
 *   out_drafts        device int32 [B, K] (-1 for a row with a non-finite logit)
 *   draft_logits      device fp32 [B, K, V], or NULL (kept in the workspace)
 *   1 <= B <= 64, 1 <= K <= 16, V and h as mtpv_verify_step.
 *   ws of at least mtpv_draft_loop_workspace_bytes(B, K, V, h) bytes.
 * One int4-head launch and the two sampler launches per position (with
 * B > 1, small copies gather position i's rows); asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
MTPV_API size_t mtpv_draft_loop_workspace_bytes(int B, int K, int V, int h);
MTPV_API mtpv_status mtpv_draft_loop(const void *w_draft, const void *s_draft, const void *h_draft,
                                     const float *u_draft, int B, int K, int V, int h,
                                     float temperature, float top_p, int32_t *out_drafts,
                                     float *draft_logits, void *ws, size_t ws_bytes,
                                     mtpv_stream stream);

/* ------------------------------------------------------------------------
 * mtpv_verify_step -- the whole verify step for B sequences in one call:
 * target logits of the B*(K+1) target rows through the bf16 head, draft
 * logits of the B*K draft rows through the int4 group-64 head, then
 * mtpv_verify.  (Passages: those of mtpv_lm_head_smallm and mtpv_verify; the
 * devtrends.cc overview's single forward pass that verifies the whole draft.)
 *
 *   w_target        device bf16 [V, h]
 *   w_draft, s_draft device uint8 [V, h/2] and bf16 [V, h/64] (int4 g64)
 *   h_target        device bf16 [B*(K+1), h]: row b*(K+1)+i is position i of
 *                   sequence b
 *   h_draft         device bf16 [B*K, h]: row b*K+i is draft position i
 *   draft_tokens, u_accept, u_sample, temperature, top_p, out_*: as in
 *                   mtpv_verify.
 *   target_logits, draft_logits  device fp32 [B, K+1, V] / [B, K, V] outputs,
 *                   or NULL to keep them inside the workspace.
 *   h a positive multiple of 64; B*(K+1) <= 64; other limits as above.
 *   ws of at least mtpv_verify_step_workspace_bytes(B, K, V, h) bytes.
 * ---------------------------------------------------------------------- */
MTPV_API size_t mtpv_verify_step_workspace_bytes(int B, int K, int V, int h);
MTPV_API mtpv_status mtpv_verify_step(const void *w_target, const void *w_draft, const void *s_draft,
                             const void *h_target, const void *h_draft,
                             const int32_t *draft_tokens, const float *u_accept,
                             const float *u_sample, int B, int K, int V, int h,
                             float temperature, float top_p, int32_t *out_tokens,
                             int32_t *out_accepted, int32_t *row_status, float *target_logits,
                             float *draft_logits, void *ws, size_t ws_bytes, mtpv_stream stream);

/* ------------------------------------------------------------------------
 * mtpv_verify_step_host -- mtpv_verify_step with the per-step inputs and
 * outputs in HOST memory; the call returns after the stream has drained.
 * Weights and ws stay on the device.
 *   h_target, h_draft  copied host->device on `stream` (page-locked buffers
 *                   give asynchronous copies; pageable ones work, slower).
 *   draft_tokens, u_accept, u_sample  read by the host during the call and
 *                   passed to the sampler by value in its launch parameters
 *                   (no copy of their own; B*(K+1) <= 64 always holds here).
 *   out_tokens, out_accepted, row_status (row_status may be NULL)  written
 *                   by the sampler kernel itself when every one of them is
 *                   page-locked host memory mapped into the device's address
 *                   space (cudaPointerGetAttributes reports a device
 *                   pointer for it); otherwise written to ws and copied
 *                   device->host on `stream`.
 * ws of at least mtpv_verify_step_host_workspace_bytes(B, K, V, h) bytes.
 * ---------------------------------------------------------------------- */
MTPV_API size_t mtpv_verify_step_host_workspace_bytes(int B, int K, int V, int h);
MTPV_API mtpv_status mtpv_verify_step_host(const void *w_target, const void *w_draft, const void *s_draft,
                                  const void *h_target_host, const void *h_draft_host,
                                  const int32_t *draft_tokens_host, const float *u_accept_host,
                                  const float *u_sample_host, int B, int K, int V, int h,
                                  float temperature, float top_p, int32_t *out_tokens_host,
                                  int32_t *out_accepted_host, int32_t *row_status_host, void *ws,
                                  size_t ws_bytes, mtpv_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* MTPV_H_ */
