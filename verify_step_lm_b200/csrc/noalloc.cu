// mtpv_verify_noalloc: mtpv_verify for callers that cannot allocate device
// memory.  The scratch the sampler kernel needs (per-sequence ticket counters
// and per-row softmax / top-p statistics) lives in a fixed array compiled into
// this library instead of in a caller-supplied workspace.  Semantics, limits
// and caveats are documented with the declaration in include/mtpv.h.
#include <mutex>

#include "args.cuh"
#include "common.cuh"
#include "sampler.cuh"

namespace {

constexpr size_t kScratchBytes = 64 * 1024;  // per device, held until process exit
constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;
static_assert(sizeof(mtpv::RowSlot) == 40, "the documented limit counts 40 bytes per row");

// The library's own scratch.  In host code this name is only a stand-in for
// the device object; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_verify_scratch[kScratchBytes];

void *g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

size_t round_up(size_t n) { return (n + kAlign - 1) / kAlign * kAlign; }

// Device address of g_verify_scratch on the calling thread's current device,
// looked up once per device (the first call may load this library's module).
cudaError_t scratch_on_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_verify_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" mtpv_status mtpv_verify_noalloc(const float *target_logits, const float *draft_logits,
                                           const int32_t *draft_tokens, const float *u_accept,
                                           const float *u_sample, int B, int K, int V,
                                           float temperature, float top_p, int32_t *out_tokens,
                                           int32_t *out_accepted, int32_t *row_status,
                                           mtpv_stream stream) {
    if (!target_logits || !draft_logits || !draft_tokens || !u_accept || !u_sample || !out_tokens ||
        !out_accepted)
        return MTPV_ERR_INVALID_ARG;
    if (!mtpv::verify_shape_ok(B, K, V) || !mtpv::sampling_params_ok(temperature, top_p))
        return MTPV_ERR_INVALID_ARG;
    if (((uintptr_t)target_logits & 3) || ((uintptr_t)draft_logits & 3)) return MTPV_ERR_INVALID_ARG;

    // scratch layout: B ticket counters, then one statistics record per row
    const size_t rows = (size_t)B * (2 * K + 1);
    const size_t stats_off = round_up(sizeof(unsigned int) * (size_t)B);
    const size_t need = stats_off + round_up(sizeof(mtpv::RowSlot) * rows);
    if (need > kScratchBytes) return MTPV_ERR_UNSUPPORTED;  // beyond the fixed scratch

    void *scratch = nullptr;
    cudaError_t e = scratch_on_current_device(&scratch);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MTPV_ERR_CUDA;
    }
    cudaStream_t s = (cudaStream_t)stream;
    unsigned int *counters = static_cast<unsigned int *>(scratch);
    // the statistics kernel clears the counters; the slots are written before use
    mtpv::SamplerParams p = {};
    p.tl = target_logits;
    p.dl = draft_logits;
    p.drafts = draft_tokens;
    p.u_acc = u_accept;
    p.u_samp = u_sample;
    p.B = B;
    p.K = K;
    p.V = V;
    p.T = temperature;
    p.top_p = top_p;
    p.verify = 1;
    p.out_tokens = out_tokens;
    p.out_acc = out_accepted;
    p.row_status = row_status;
    p.slots = reinterpret_cast<mtpv::RowSlot *>(static_cast<unsigned char *>(scratch) + stats_off);
    p.counters = counters;
    e = mtpv::launch_sampler(p, (int)rows, s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MTPV_ERR_CUDA;
    }
    return MTPV_OK;
}
