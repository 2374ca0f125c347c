// extern "C" entry points of libmtpv: argument checks, workspace layout and
// kernel launches.  Semantics and citations are in include/mtpv.h.
#include <cstring>
#include <math.h>
#include <stdint.h>

#include "args.cuh"
#include "common.cuh"
#include "lm_head.cuh"
#include "sampler.cuh"

namespace {

using mtpv::kMaxRows;
using mtpv::kMaxV;
using mtpv::sampling_params_ok;
using mtpv::verify_shape_ok;

constexpr size_t kAlign = 256;

size_t up(size_t n) { return (n + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

mtpv_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MTPV_OK;
    cudaGetLastError();  // clear a sticky launch error so later calls can proceed
    return MTPV_ERR_CUDA;
}

// --- workspace layouts -----------------------------------------------------
// verify: ticket counters, per-row statistics slots, then the per-row
// weights (exp((l - m)/T) of kept tokens, 0 elsewhere; fp64) that the draw
// kernel reads instead of recomputing.
struct VerifyWs {
    size_t counters, stats, ecache, total;
};
VerifyWs verify_layout(int B, int K, int V) {
    const size_t rows = (size_t)B * (2 * K + 1);
    VerifyWs l;
    l.counters = 0;
    l.stats = up(sizeof(unsigned int) * (size_t)B);
    l.ecache = l.stats + up(sizeof(mtpv::RowSlot) * rows);
    l.total = l.ecache + up(sizeof(double) * rows * (size_t)V);
    return l;
}

// Both heads' scratch: the fused kernel's work counter, then each head's own
// scratch when the two run as separate launches.
struct HeadsWs {
    size_t work, t, d, total;
};
HeadsWs heads_layout(int Mt, int Md, int Kd) {
    HeadsWs l;
    l.work = 0;
    l.t = up(mtpv::kHeadsPairWorkBytes);
    l.d = l.t + up(mtpv::lm_head_scratch_bytes(Mt, Kd, MTPV_W_BF16));
    l.total = l.d + up(mtpv::lm_head_scratch_bytes(Md, Kd, MTPV_W_INT4_G64));
    return l;
}

struct StepWs {
    size_t heads, tl, dl, verify, total;
};
StepWs step_layout(int B, int K, int V, int h) {
    StepWs l;
    l.heads = 0;  // both heads' scratch
    l.tl = l.heads + heads_layout(B * (K + 1), B * K, h).total;
    l.dl = l.tl + up(sizeof(float) * (size_t)B * (K + 1) * V);
    l.verify = l.dl + up(sizeof(float) * (size_t)B * K * V);
    l.total = l.verify + verify_layout(B, K, V).total;
    return l;
}

struct HostWs {
    size_t step, ht, hd, drafts, ua, us, tok, acc, rs, total;
};
HostWs host_layout(int B, int K, int V, int h) {
    HostWs l;
    l.step = 0;
    l.ht = step_layout(B, K, V, h).total;
    l.hd = l.ht + up((size_t)B * (K + 1) * h * 2);
    l.drafts = l.hd + up((size_t)B * K * h * 2);
    l.ua = l.drafts + up(sizeof(int32_t) * (size_t)B * K);
    l.us = l.ua + up(sizeof(float) * (size_t)B * K);
    l.tok = l.us + up(sizeof(float) * (size_t)B * (K + 1));
    l.acc = l.tok + up(sizeof(int32_t) * (size_t)B * (K + 1));
    l.rs = l.acc + up(sizeof(int32_t) * (size_t)B);
    l.total = l.rs + up(sizeof(int32_t) * (size_t)B);
    return l;
}

// draft loop: per position, the B hidden rows, their logits, uniforms and
// tokens (B > 1 only: gathered from / scattered to the [B, K] layouts), then
// the sampler's workspace.
struct DraftWs {
    size_t x, y, u, tok, samp, head, total;
};
size_t sample_ws_bytes(int R, int V) {
    return up(sizeof(mtpv::RowSlot) * (size_t)R) + up(sizeof(double) * (size_t)R * V);
}
DraftWs draft_layout(int B, int V, int h) {
    DraftWs l;
    l.x = 0;
    l.y = l.x + up((size_t)B * h * 2);
    l.u = l.y + up(sizeof(float) * (size_t)B * V);
    l.tok = l.u + up(sizeof(float) * (size_t)B);
    l.samp = l.tok + up(sizeof(int32_t) * (size_t)B);
    l.head = l.samp + sample_ws_bytes(B, V);
    l.total = l.head + up(mtpv::lm_head_scratch_bytes(B, h, MTPV_W_INT4_G64));
    return l;
}

bool lm_head_shape_ok(int M, int Kd, int N) {
    return M >= 1 && M <= 64 && Kd >= 64 && Kd % 64 == 0 && N >= 1 &&
           mtpv::lm_head_max_smem_rows(Kd) >= 1;
}

char *at(void *ws, size_t off) { return static_cast<char *>(ws) + off; }

// Both heads: one fused launch when the kernel takes the shapes, else two.
// ws holds heads_layout(Mt, Md, Kd).total bytes.
cudaError_t launch_heads(const void *xt, int Mt, const void *w, float *yt, const void *xd, int Md,
                         const void *wq, const void *scales, float *yd, int Kd, int N, void *ws,
                         cudaStream_t s) {
    const HeadsWs l = heads_layout(Mt, Md, Kd);
    if (mtpv::lm_heads_pair_ok(Mt, Md, Kd, scales))
        return mtpv::launch_lm_heads_pair(xt, Mt, w, yt, xd, Md, wq, scales, yd, Kd, N, at(ws, l.work), s);
    cudaError_t e = mtpv::launch_lm_head(xt, Mt, Kd, N, w, nullptr, MTPV_W_BF16, yt, at(ws, l.t), s);
    if (e != cudaSuccess) return e;
    return mtpv::launch_lm_head(xd, Md, Kd, N, wq, scales, MTPV_W_INT4_G64, yd, at(ws, l.d), s);
}

// inl (optional): the per-position inputs by value, in place of drafts / ua / us.
mtpv_status launch_verify(const float *tl, const float *dl, const int32_t *drafts, const float *ua,
                          const float *us, int B, int K, int V, float T, float top_p,
                          int32_t *out_tokens, int32_t *out_acc, int32_t *row_status, void *ws,
                          cudaStream_t s, const mtpv::SamplerInline *inl = nullptr) {
    const VerifyWs l = verify_layout(B, K, V);
    unsigned int *counters = reinterpret_cast<unsigned int *>(at(ws, l.counters));
    mtpv::SamplerParams p;
    p.tl = tl;
    p.dl = dl;
    p.drafts = drafts;
    p.u_acc = ua;
    p.u_samp = us;
    p.B = B;
    p.K = K;
    p.V = V;
    p.T = T;
    p.top_p = top_p;
    p.verify = 1;
    p.out_tokens = out_tokens;
    p.out_acc = out_acc;
    p.row_status = row_status;
    p.slots = reinterpret_cast<mtpv::RowSlot *>(at(ws, l.stats));
    p.counters = counters;
    p.ecache = reinterpret_cast<double *>(at(ws, l.ecache));
    if (inl) {
        p.inline_inputs = 1;
        p.inl = *inl;
    }
    return cuda_status(mtpv::launch_sampler(p, B * (2 * K + 1), s));
}

}  // namespace

extern "C" {

int mtpv_version(void) { return 100; }

void mtpv_set_wait_polls(int polls) { mtpv::set_wait_polls(polls); }

const char *mtpv_status_string(mtpv_status st) {
    switch (st) {
        case MTPV_OK: return "ok";
        case MTPV_ERR_INVALID_ARG: return "invalid argument";
        case MTPV_ERR_UNSUPPORTED: return "unsupported";
        case MTPV_ERR_WORKSPACE: return "workspace missing or too small";
        case MTPV_ERR_CUDA: return "CUDA error";
        case MTPV_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

size_t mtpv_lm_head_workspace_bytes(int M, int Kd, int N, mtpv_wfmt fmt) {
    if (!lm_head_shape_ok(M, Kd, N) || (fmt != MTPV_W_BF16 && fmt != MTPV_W_INT4_G64)) return 0;
    return mtpv::lm_head_scratch_bytes(M, Kd, (int)fmt);
}

mtpv_status mtpv_lm_head_smallm(const void *x, int M, int Kd, int N, const void *w,
                                const void *scales, mtpv_wfmt fmt, float *y, void *ws,
                                size_t ws_bytes, mtpv_stream stream) {
    if (!x || !w || !y || !lm_head_shape_ok(M, Kd, N)) return MTPV_ERR_INVALID_ARG;
    if (fmt != MTPV_W_BF16 && fmt != MTPV_W_INT4_G64) return MTPV_ERR_INVALID_ARG;
    if (fmt == MTPV_W_INT4_G64 && (!scales || !aligned(scales, 2))) return MTPV_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 4)) return MTPV_ERR_INVALID_ARG;
    const size_t need = mtpv::lm_head_scratch_bytes(M, Kd, (int)fmt);
    if (need && (!ws || !aligned(ws, kAlign) || ws_bytes < need)) return MTPV_ERR_WORKSPACE;
    return cuda_status(mtpv::launch_lm_head(x, M, Kd, N, w, scales, (int)fmt, y, ws, (cudaStream_t)stream));
}

size_t mtpv_lm_head_pair_workspace_bytes(int Mt, int Md, int Kd, int N) {
    if (!lm_head_shape_ok(Mt, Kd, N) || !lm_head_shape_ok(Md, Kd, N)) return 0;
    return heads_layout(Mt, Md, Kd).total;
}

mtpv_status mtpv_lm_head_pair(const void *xt, int Mt, const void *w, float *yt, const void *xd,
                              int Md, const void *wq, const void *scales, float *yd, int Kd, int N,
                              void *ws, size_t ws_bytes, mtpv_stream stream) {
    if (!xt || !w || !yt || !xd || !wq || !scales || !yd) return MTPV_ERR_INVALID_ARG;
    if (!lm_head_shape_ok(Mt, Kd, N) || !lm_head_shape_ok(Md, Kd, N)) return MTPV_ERR_INVALID_ARG;
    if (!aligned(xt, 16) || !aligned(w, 16) || !aligned(yt, 4) || !aligned(xd, 16) ||
        !aligned(wq, 16) || !aligned(scales, 2) || !aligned(yd, 4))
        return MTPV_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, kAlign) || ws_bytes < heads_layout(Mt, Md, Kd).total) return MTPV_ERR_WORKSPACE;
    return cuda_status(launch_heads(xt, Mt, w, yt, xd, Md, wq, scales, yd, Kd, N, ws, (cudaStream_t)stream));
}

static size_t int4_proj_ws(int M, int Kd, int N, bool gate_up) {
    if (M < 1 || M > 64 || Kd < 64 || Kd % 64 || Kd > (1 << 20) || N < 1 || N > (1 << 28)) return 0;
    if (gate_up && N % 2) return 0;
    return mtpv::int4_proj_workspace_bytes(M, Kd, N, gate_up);
}

size_t mtpv_int4_proj_workspace_bytes(int M, int Kd, int N) { return int4_proj_ws(M, Kd, N, false); }

static mtpv_status int4_proj_common(const void *x, int M, int Kd, int N, const void *wq,
                                    const void *scales, float *y, int ldy, bool silu_mul, void *ws,
                                    size_t ws_bytes, mtpv_stream stream) {
    if (!x || !wq || !scales || !y) return MTPV_ERR_INVALID_ARG;
    const size_t need = int4_proj_ws(M, Kd, N, silu_mul);
    if (need == 0) return MTPV_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(wq, 16) || !aligned(scales, 16) || !aligned(y, 4))
        return MTPV_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, kAlign) || ws_bytes < need) return MTPV_ERR_WORKSPACE;
    return cuda_status(
        mtpv::launch_int4_proj(x, M, Kd, N, wq, scales, y, ldy, silu_mul, ws, false, (cudaStream_t)stream));
}

mtpv_status mtpv_int4_proj(const void *x, int M, int Kd, int N, const void *wq, const void *scales,
                           float *y, void *ws, size_t ws_bytes, mtpv_stream stream) {
    return int4_proj_common(x, M, Kd, N, wq, scales, y, N, false, ws, ws_bytes, stream);
}

size_t mtpv_int4_gate_up_workspace_bytes(int M, int Kd, int F) {
    if (F < 1 || F > (1 << 27)) return 0;
    return int4_proj_ws(M, Kd, 2 * F, true);
}

mtpv_status mtpv_int4_gate_up(const void *x, int M, int Kd, int F, const void *wq,
                              const void *scales, float *h, void *ws, size_t ws_bytes,
                              mtpv_stream stream) {
    if (F < 1 || F > (1 << 27)) return MTPV_ERR_INVALID_ARG;
    return int4_proj_common(x, M, Kd, 2 * F, wq, scales, h, F, true, ws, ws_bytes, stream);
}

size_t mtpv_verify_workspace_bytes(int B, int K, int V) {
    if (!verify_shape_ok(B, K, V)) return 0;
    return verify_layout(B, K, V).total;
}

mtpv_status mtpv_verify(const float *target_logits, const float *draft_logits,
                        const int32_t *draft_tokens, const float *u_accept, const float *u_sample,
                        int B, int K, int V, float temperature, float top_p, int32_t *out_tokens,
                        int32_t *out_accepted, int32_t *row_status, void *ws, size_t ws_bytes,
                        mtpv_stream stream) {
    if (!target_logits || !draft_logits || !draft_tokens || !u_accept || !u_sample || !out_tokens ||
        !out_accepted)
        return MTPV_ERR_INVALID_ARG;
    if (!verify_shape_ok(B, K, V) || !sampling_params_ok(temperature, top_p))
        return MTPV_ERR_INVALID_ARG;
    if (!aligned(target_logits, 4) || !aligned(draft_logits, 4)) return MTPV_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, kAlign) || ws_bytes < verify_layout(B, K, V).total) return MTPV_ERR_WORKSPACE;
    return launch_verify(target_logits, draft_logits, draft_tokens, u_accept, u_sample, B, K, V,
                         temperature, top_p, out_tokens, out_accepted, row_status, ws,
                         (cudaStream_t)stream);
}

size_t mtpv_sample_workspace_bytes(int R, int V) {
    if (R < 1 || R > kMaxRows || V < 1 || V > kMaxV) return 0;
    return up(sizeof(mtpv::RowSlot) * (size_t)R) + up(sizeof(double) * (size_t)R * V);
}

mtpv_status mtpv_sample(const float *logits, int R, int V, float temperature, float top_p,
                        const float *u, int32_t *out, int32_t *row_status, void *ws,
                        size_t ws_bytes, mtpv_stream stream) {
    if (!logits || !u || !out) return MTPV_ERR_INVALID_ARG;
    if (R < 1 || R > kMaxRows || V < 1 || V > kMaxV || !sampling_params_ok(temperature, top_p))
        return MTPV_ERR_INVALID_ARG;
    if (!aligned(logits, 4)) return MTPV_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, kAlign) || ws_bytes < mtpv_sample_workspace_bytes(R, V))
        return MTPV_ERR_WORKSPACE;
    mtpv::SamplerParams p = {};
    p.tl = logits;
    p.dl = nullptr;
    p.u_samp = u;
    p.B = R;
    p.K = 0;
    p.V = V;
    p.T = temperature;
    p.top_p = top_p;
    p.verify = 0;
    p.out_tokens = out;
    p.row_status = row_status;
    p.slots = reinterpret_cast<mtpv::RowSlot *>(ws);
    p.counters = nullptr;
    p.ecache = reinterpret_cast<double *>(at(ws, up(sizeof(mtpv::RowSlot) * (size_t)R)));
    return cuda_status(mtpv::launch_sampler(p, R, (cudaStream_t)stream));
}

size_t mtpv_draft_loop_workspace_bytes(int B, int K, int V, int h) {
    if (!verify_shape_ok(B, K, V) || B > 64 || h < 64 || h % 64 || !lm_head_shape_ok(B, h, V)) return 0;
    return draft_layout(B, V, h).total;
}

mtpv_status mtpv_draft_loop(const void *w_draft, const void *s_draft, const void *h_draft,
                            const float *u_draft, int B, int K, int V, int h, float temperature,
                            float top_p, int32_t *out_drafts, float *draft_logits, void *ws,
                            size_t ws_bytes, mtpv_stream stream) {
    if (!w_draft || !s_draft || !h_draft || !u_draft || !out_drafts) return MTPV_ERR_INVALID_ARG;
    if (mtpv_draft_loop_workspace_bytes(B, K, V, h) == 0 || !sampling_params_ok(temperature, top_p))
        return MTPV_ERR_INVALID_ARG;
    if (!aligned(w_draft, 16) || !aligned(s_draft, 2) || !aligned(h_draft, 16) ||
        (draft_logits && !aligned(draft_logits, 4)))
        return MTPV_ERR_INVALID_ARG;
    const DraftWs l = draft_layout(B, V, h);
    if (!ws || !aligned(ws, kAlign) || ws_bytes < l.total) return MTPV_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const char *hd = static_cast<const char *>(h_draft);
    for (int i = 0; i < K; ++i) {
        // position i: rows b*K + i of the [B, K, ...] inputs
        const void *x = hd + (size_t)i * h * 2;
        const float *u = u_draft + i;
        float *y = draft_logits ? draft_logits + (size_t)i * V : reinterpret_cast<float *>(at(ws, l.y));
        int32_t *tok = out_drafts + i;
        cudaError_t e = cudaSuccess;
        if (B > 1) {
            x = at(ws, l.x);
            u = reinterpret_cast<const float *>(at(ws, l.u));
            y = reinterpret_cast<float *>(at(ws, l.y));
            tok = reinterpret_cast<int32_t *>(at(ws, l.tok));
            e = cudaMemcpy2DAsync(at(ws, l.x), (size_t)h * 2, hd + (size_t)i * h * 2, (size_t)K * h * 2,
                                  (size_t)h * 2, B, cudaMemcpyDeviceToDevice, s);
            if (e == cudaSuccess)
                e = cudaMemcpy2DAsync(at(ws, l.u), sizeof(float), u_draft + i, (size_t)K * sizeof(float),
                                      sizeof(float), B, cudaMemcpyDeviceToDevice, s);
            if (e != cudaSuccess) return cuda_status(e);
        }
        e = mtpv::launch_lm_head(x, B, h, V, w_draft, s_draft, MTPV_W_INT4_G64, y, at(ws, l.head), s);
        if (e != cudaSuccess) return cuda_status(e);
        mtpv::SamplerParams p = {};
        p.tl = y;
        p.u_samp = u;
        p.B = B;
        p.V = V;
        p.T = temperature;
        p.top_p = top_p;
        p.verify = 0;
        p.out_tokens = tok;
        p.slots = reinterpret_cast<mtpv::RowSlot *>(at(ws, l.samp));
        p.ecache = reinterpret_cast<double *>(at(ws, l.samp + up(sizeof(mtpv::RowSlot) * (size_t)B)));
        e = mtpv::launch_sampler(p, B, s);
        if (e != cudaSuccess) return cuda_status(e);
        if (B > 1) {
            e = cudaMemcpy2DAsync(out_drafts + i, (size_t)K * sizeof(int32_t), tok, sizeof(int32_t),
                                  sizeof(int32_t), B, cudaMemcpyDeviceToDevice, s);
            if (e == cudaSuccess && draft_logits)
                e = cudaMemcpy2DAsync(draft_logits + (size_t)i * V, (size_t)K * V * sizeof(float), y,
                                      (size_t)V * sizeof(float), (size_t)V * sizeof(float), B,
                                      cudaMemcpyDeviceToDevice, s);
            if (e != cudaSuccess) return cuda_status(e);
        }
    }
    return MTPV_OK;
}

size_t mtpv_verify_step_workspace_bytes(int B, int K, int V, int h) {
    if (!verify_shape_ok(B, K, V) || B * (K + 1) > 64 || h < 64 || h % 64) return 0;
    return step_layout(B, K, V, h).total;
}

}  // extern "C"

namespace {

// Arguments of a verify step other than the per-position inputs and outputs.
mtpv_status step_check(const void *w_target, const void *w_draft, const void *s_draft,
                       const void *h_target, const void *h_draft, int B, int K, int V, int h,
                       float temperature, float top_p, const float *target_logits,
                       const float *draft_logits, const void *ws, size_t ws_bytes) {
    if (!w_target || !w_draft || !s_draft || !h_target || !h_draft) return MTPV_ERR_INVALID_ARG;
    if (!verify_shape_ok(B, K, V) || B * (K + 1) > 64 || !lm_head_shape_ok(B * (K + 1), h, V) ||
        !sampling_params_ok(temperature, top_p))
        return MTPV_ERR_INVALID_ARG;
    if (!aligned(w_target, 16) || !aligned(w_draft, 16) || !aligned(s_draft, 2) ||
        !aligned(h_target, 16) || !aligned(h_draft, 16))
        return MTPV_ERR_INVALID_ARG;
    if ((target_logits && !aligned(target_logits, 4)) || (draft_logits && !aligned(draft_logits, 4)))
        return MTPV_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, kAlign) || ws_bytes < step_layout(B, K, V, h).total) return MTPV_ERR_WORKSPACE;
    return MTPV_OK;
}

// Both heads, then the sampler (arguments checked by step_check).
mtpv_status step_launch(const void *w_target, const void *w_draft, const void *s_draft,
                        const void *h_target, const void *h_draft, const int32_t *draft_tokens,
                        const float *u_accept, const float *u_sample, const mtpv::SamplerInline *inl,
                        int B, int K, int V, int h, float temperature, float top_p,
                        int32_t *out_tokens, int32_t *out_accepted, int32_t *row_status,
                        float *target_logits, float *draft_logits, void *ws, cudaStream_t s) {
    const StepWs l = step_layout(B, K, V, h);
    float *tl = target_logits ? target_logits : reinterpret_cast<float *>(at(ws, l.tl));
    float *dl = draft_logits ? draft_logits : reinterpret_cast<float *>(at(ws, l.dl));
    const cudaError_t e = launch_heads(h_target, B * (K + 1), w_target, tl, h_draft, B * K, w_draft,
                                       s_draft, dl, h, V, at(ws, l.heads), s);
    if (e != cudaSuccess) return cuda_status(e);
    return launch_verify(tl, dl, draft_tokens, u_accept, u_sample, B, K, V, temperature, top_p,
                         out_tokens, out_accepted, row_status, at(ws, l.verify), s, inl);
}

// The device address of a page-locked host buffer mapped into this device's
// address space, else null (pageable memory, or no mapping).
void *mapped_device_alias(void *host) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

}  // namespace

extern "C" {

mtpv_status mtpv_verify_step(const void *w_target, const void *w_draft, const void *s_draft,
                             const void *h_target, const void *h_draft,
                             const int32_t *draft_tokens, const float *u_accept,
                             const float *u_sample, int B, int K, int V, int h, float temperature,
                             float top_p, int32_t *out_tokens, int32_t *out_accepted,
                             int32_t *row_status, float *target_logits, float *draft_logits,
                             void *ws, size_t ws_bytes, mtpv_stream stream) {
    if (!draft_tokens || !u_accept || !u_sample || !out_tokens || !out_accepted) return MTPV_ERR_INVALID_ARG;
    const mtpv_status st = step_check(w_target, w_draft, s_draft, h_target, h_draft, B, K, V, h, temperature,
                                      top_p, target_logits, draft_logits, ws, ws_bytes);
    if (st != MTPV_OK) return st;
    return step_launch(w_target, w_draft, s_draft, h_target, h_draft, draft_tokens, u_accept, u_sample, nullptr,
                       B, K, V, h, temperature, top_p, out_tokens, out_accepted, row_status, target_logits,
                       draft_logits, ws, (cudaStream_t)stream);
}

size_t mtpv_verify_step_host_workspace_bytes(int B, int K, int V, int h) {
    if (mtpv_verify_step_workspace_bytes(B, K, V, h) == 0) return 0;
    return host_layout(B, K, V, h).total;
}

mtpv_status mtpv_verify_step_host(const void *w_target, const void *w_draft, const void *s_draft,
                                  const void *h_target_host, const void *h_draft_host,
                                  const int32_t *draft_tokens_host, const float *u_accept_host,
                                  const float *u_sample_host, int B, int K, int V, int h,
                                  float temperature, float top_p, int32_t *out_tokens_host,
                                  int32_t *out_accepted_host, int32_t *row_status_host, void *ws,
                                  size_t ws_bytes, mtpv_stream stream) {
    if (!h_target_host || !h_draft_host || !draft_tokens_host || !u_accept_host || !u_sample_host ||
        !out_tokens_host || !out_accepted_host)
        return MTPV_ERR_INVALID_ARG;
    if (mtpv_verify_step_workspace_bytes(B, K, V, h) == 0) return MTPV_ERR_INVALID_ARG;
    const HostWs l = host_layout(B, K, V, h);
    if (!ws || !aligned(ws, kAlign) || ws_bytes < l.total) return MTPV_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t nt = (size_t)B * (K + 1), nd = (size_t)B * K;
    const mtpv_status chk = step_check(w_target, w_draft, s_draft, at(ws, l.ht), at(ws, l.hd), B, K, V, h,
                                       temperature, top_p, nullptr, nullptr, at(ws, l.step), l.ht);
    if (chk != MTPV_OK) return chk;
    // The hidden states are copied in; drafts and uniforms (a few bytes per
    // position) travel by value in the sampler's launch parameters instead.
    cudaError_t e = cudaMemcpyAsync(at(ws, l.ht), h_target_host, nt * h * 2, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(at(ws, l.hd), h_draft_host, nd * h * 2, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_status(e);
    // (mtpv_verify_step's limit B (K + 1) <= 64, checked by step_check, fits the block)
    static_assert(mtpv::kInlinePositions >= 64, "per-position inputs of a verify step by value");
    mtpv::SamplerInline inl;
    std::memcpy(inl.drafts, draft_tokens_host, nd * sizeof(int32_t));
    std::memcpy(inl.u_acc, u_accept_host, nd * sizeof(float));
    std::memcpy(inl.u_samp, u_sample_host, nt * sizeof(float));
    // Outputs: written by the kernel straight into the host buffers when all
    // of them are page-locked and mapped into the device's address space,
    // else into the workspace and copied back.
    int32_t *tok = static_cast<int32_t *>(mapped_device_alias(out_tokens_host));
    int32_t *acc = static_cast<int32_t *>(mapped_device_alias(out_accepted_host));
    int32_t *rs = row_status_host ? static_cast<int32_t *>(mapped_device_alias(row_status_host)) : nullptr;
    const bool direct = tok && acc && (!row_status_host || rs);
    if (!direct) {
        tok = reinterpret_cast<int32_t *>(at(ws, l.tok));
        acc = reinterpret_cast<int32_t *>(at(ws, l.acc));
        rs = reinterpret_cast<int32_t *>(at(ws, l.rs));
    }
    const mtpv_status st = step_launch(w_target, w_draft, s_draft, at(ws, l.ht), at(ws, l.hd), nullptr, nullptr,
                                       nullptr, &inl, B, K, V, h, temperature, top_p, tok, acc, rs, nullptr,
                                       nullptr, at(ws, l.step), s);
    if (st != MTPV_OK) return st;
    if (!direct) {
        e = cudaMemcpyAsync(out_tokens_host, tok, nt * sizeof(int32_t), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(out_accepted_host, acc, (size_t)B * sizeof(int32_t), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess && row_status_host)
            e = cudaMemcpyAsync(row_status_host, rs, (size_t)B * sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return cuda_status(e);
}

}  // extern "C"
