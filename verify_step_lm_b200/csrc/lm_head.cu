// Small-M weight-streaming projection y[M, N] = x[M, Kd] . Wd[N, Kd]^T.
//
// The pages' verify pass ends in a matmul with only M = 3..6 activation rows
// (hazakura.dev MTPLX notes, Layer 0: a shader rewritten for small matrices)
// and drafts through a 4-bit copy of the LM head (same section); decode GEMVs
// dequantise inside the inner loop, one kernel per storage format
// (gist.science BaseRT explainer, methodology: specialisation).
//
// At M <= 8 every weight is used M times: the kernel is an HBM stream.  Design
// for sm_100a:
//   - the M activation rows are staged once per CTA in shared memory (bf16);
//   - each warp owns RW consecutive weight rows at a time and sweeps the whole
//     reduction length with 16-byte non-allocating loads (U chunks per lane
//     in flight per row), so every byte of the head is read exactly once;
//   - fp32 accumulation in registers, one warp-shuffle reduction per row;
//   - int4 rows are dequantised in registers: each nibble n becomes the fp32
//     value (n - 8) through the exponent trick 0x4B000000 | n = 2^23 + n
//     (exact), the group scale multiplies the 32-weight partial sum once;
//   - a persistent grid of (SMs x resident CTAs) walks the row groups.
#include <algorithm>

#include "common.cuh"
#include "lm_head.cuh"

namespace mtpv {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

template <int M>
__device__ __forceinline__ void load_x8(const uint4 *xs, int nch, int c, float (&xf)[M][8]) {
#pragma unroll
    for (int m = 0; m < M; ++m) {
        const uint4 v = xs[m * nch + c];
        xf[m][0] = bf16_lo(v.x); xf[m][1] = bf16_hi(v.x);
        xf[m][2] = bf16_lo(v.y); xf[m][3] = bf16_hi(v.y);
        xf[m][4] = bf16_lo(v.z); xf[m][5] = bf16_hi(v.z);
        xf[m][6] = bf16_lo(v.w); xf[m][7] = bf16_hi(v.w);
    }
}

// ---------------------------------------------------------------------------
// bf16 weights: 16-byte chunk = 8 weights
// ---------------------------------------------------------------------------
template <int M, int RW, int U>
__global__ void __launch_bounds__(kGemvThreads) lm_head_bf16_kernel(
    const uint16_t *__restrict__ x, int Kd, int N, const uint16_t *__restrict__ W,
    float *__restrict__ y, int ldy) {
    extern __shared__ uint4 xs[];  // [M][Kd/8]
    const int nch = Kd >> 3;
    const uint4 *xg = reinterpret_cast<const uint4 *>(x);
    for (int i = threadIdx.x; i < M * nch; i += kGemvThreads) xs[i] = xg[i];
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int groups = (N + RW - 1) / RW;
    for (int g = blockIdx.x * kGemvWarps + warp; g < groups; g += gridDim.x * kGemvWarps) {
        const int r0 = g * RW;
        const uint4 *wr[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r)
            wr[r] = reinterpret_cast<const uint4 *>(W + (size_t)min(r0 + r, N - 1) * Kd);
        float acc[RW][M];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < M; ++m) acc[r][m] = 0.0f;

        for (int c0 = lane; c0 < nch; c0 += 32 * U) {
            uint4 wv[U][RW];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 32 * u;
#pragma unroll
                for (int r = 0; r < RW; ++r)
                    wv[u][r] = (c < nch) ? ld_stream16(wr[r] + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 32 * u;
                if (c < nch) {
                    float xf[M][8];
                    load_x8<M>(xs, nch, c, xf);
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        const uint4 w = wv[u][r];
                        const float wf[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                                             bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
#pragma unroll
                        for (int m = 0; m < M; ++m) {
                            float a = acc[r][m];
#pragma unroll
                            for (int i = 0; i < 8; ++i) a = fmaf(xf[m][i], wf[i], a);
                            acc[r][m] = a;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const float v = warp_sum(acc[r][m]);
                if (lane == 0 && r0 + r < N) y[(size_t)m * ldy + r0 + r] = v;
            }
    }
}

// ---------------------------------------------------------------------------
// int4 group-64 weights: 16-byte chunk = 32 weights = half a group
// ---------------------------------------------------------------------------
__device__ __forceinline__ float nib_minus8(uint32_t word, int i) {
    // 2^23 + n exactly, minus (2^23 + 8)
    return __uint_as_float(0x4B000000u | ((word >> (4 * i)) & 0xFu)) - 8388616.0f;
}

template <int M, int RW, int U>
__global__ void __launch_bounds__(kGemvThreads) lm_head_int4_kernel(
    const uint16_t *__restrict__ x, int Kd, int N, const uint8_t *__restrict__ Wq,
    const uint16_t *__restrict__ S, float *__restrict__ y, int ldy) {
    extern __shared__ uint4 xs[];  // [M][Kd/8] bf16
    const int nx = Kd >> 3;
    const uint4 *xg = reinterpret_cast<const uint4 *>(x);
    for (int i = threadIdx.x; i < M * nx; i += kGemvThreads) xs[i] = xg[i];
    __syncthreads();

    const int nch = Kd >> 5;   // 16-byte chunks per row
    const int ng = Kd >> 6;    // scales per row
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int groups = (N + RW - 1) / RW;
    for (int g = blockIdx.x * kGemvWarps + warp; g < groups; g += gridDim.x * kGemvWarps) {
        const int r0 = g * RW;
        const uint4 *wr[RW];
        const uint16_t *sr[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int rr = min(r0 + r, N - 1);
            wr[r] = reinterpret_cast<const uint4 *>(Wq + (size_t)rr * (Kd >> 1));
            sr[r] = S + (size_t)rr * ng;
        }
        float acc[RW][M];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < M; ++m) acc[r][m] = 0.0f;

        for (int c0 = lane; c0 < nch; c0 += 32 * U) {
            uint4 wv[U][RW];
            float sc[U][RW];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 32 * u;
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    wv[u][r] = (c < nch) ? ld_stream16(wr[r] + c) : make_uint4(0, 0, 0, 0);
                    sc[u][r] = (c < nch) ? __uint_as_float((uint32_t)__ldg(sr[r] + (c >> 1)) << 16) : 0.0f;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 32 * u;
                if (c < nch) {
                    float part[RW][M];
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int m = 0; m < M; ++m) part[r][m] = 0.0f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {  // 4 words of 8 weights
                        float xf[M][8];
                        load_x8<M>(xs, nx, c * 4 + q, xf);
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            const uint32_t word = q == 0 ? wv[u][r].x : q == 1 ? wv[u][r].y : q == 2 ? wv[u][r].z : wv[u][r].w;
                            float wf[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) wf[i] = nib_minus8(word, i);
#pragma unroll
                            for (int m = 0; m < M; ++m) {
                                float a = part[r][m];
#pragma unroll
                                for (int i = 0; i < 8; ++i) a = fmaf(xf[m][i], wf[i], a);
                                part[r][m] = a;
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int m = 0; m < M; ++m) acc[r][m] = fmaf(sc[u][r], part[r][m], acc[r][m]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const float v = warp_sum(acc[r][m]);
                if (lane == 0 && r0 + r < N) y[(size_t)m * ldy + r0 + r] = v;
            }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <typename Kern>
static int resident_ctas(Kern k, size_t smem) {
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kGemvThreads, smem) != cudaSuccess) {
        cudaGetLastError();
        occ = 1;
    }
    return std::max(1, occ);
}

template <int M>
static cudaError_t launch_bf16(const uint16_t *x, int Kd, int N, const uint16_t *W, float *y,
                               int ldy, cudaStream_t s) {
    constexpr int RW = M <= 2 ? 8 : (M <= 4 ? 4 : 2);
    constexpr int U = 2;
    auto k = lm_head_bf16_kernel<M, RW, U>;
    const size_t smem = (size_t)M * Kd * 2;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int groups = (N + RW - 1) / RW;
    const int need = (groups + kGemvWarps - 1) / kGemvWarps;
    const int grid = std::min(need, kSMs * resident_ctas(k, smem));
    k<<<grid, kGemvThreads, smem, s>>>(x, Kd, N, W, y, ldy);
    return cudaGetLastError();
}

template <int M>
static cudaError_t launch_int4(const uint16_t *x, int Kd, int N, const uint8_t *Wq,
                               const uint16_t *S, float *y, int ldy, cudaStream_t s) {
    constexpr int RW = M <= 2 ? 8 : (M <= 4 ? 4 : 2);
    constexpr int U = 1;
    auto k = lm_head_int4_kernel<M, RW, U>;
    const size_t smem = (size_t)M * Kd * 2;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int groups = (N + RW - 1) / RW;
    const int need = (groups + kGemvWarps - 1) / kGemvWarps;
    const int grid = std::min(need, kSMs * resident_ctas(k, smem));
    k<<<grid, kGemvThreads, smem, s>>>(x, Kd, N, Wq, S, y, ldy);
    return cudaGetLastError();
}

size_t lm_head_max_smem_rows(int Kd) {
    // rows of x that fit in 227 KB of shared memory
    return (size_t)(227 * 1024) / ((size_t)Kd * 2);
}

cudaError_t launch_lm_head(const void *x, int M, int Kd, int N, const void *w, const void *scales,
                           int fmt, float *y, cudaStream_t s) {
    const uint16_t *xb = static_cast<const uint16_t *>(x);
    const int step = (int)std::min<size_t>(8, lm_head_max_smem_rows(Kd));
    if (step < 1) return cudaErrorInvalidValue;
    for (int m0 = 0; m0 < M; m0 += step) {
        const int mm = std::min(step, M - m0);
        const uint16_t *xm = xb + (size_t)m0 * Kd;
        float *ym = y + (size_t)m0 * N;
        cudaError_t e = cudaSuccess;
        if (fmt == MTPV_W_BF16) {
            const uint16_t *W = static_cast<const uint16_t *>(w);
            switch (mm) {
                case 1: e = launch_bf16<1>(xm, Kd, N, W, ym, N, s); break;
                case 2: e = launch_bf16<2>(xm, Kd, N, W, ym, N, s); break;
                case 3: e = launch_bf16<3>(xm, Kd, N, W, ym, N, s); break;
                case 4: e = launch_bf16<4>(xm, Kd, N, W, ym, N, s); break;
                case 5: e = launch_bf16<5>(xm, Kd, N, W, ym, N, s); break;
                case 6: e = launch_bf16<6>(xm, Kd, N, W, ym, N, s); break;
                case 7: e = launch_bf16<7>(xm, Kd, N, W, ym, N, s); break;
                default: e = launch_bf16<8>(xm, Kd, N, W, ym, N, s); break;
            }
        } else {
            const uint8_t *Wq = static_cast<const uint8_t *>(w);
            const uint16_t *S = static_cast<const uint16_t *>(scales);
            switch (mm) {
                case 1: e = launch_int4<1>(xm, Kd, N, Wq, S, ym, N, s); break;
                case 2: e = launch_int4<2>(xm, Kd, N, Wq, S, ym, N, s); break;
                case 3: e = launch_int4<3>(xm, Kd, N, Wq, S, ym, N, s); break;
                case 4: e = launch_int4<4>(xm, Kd, N, Wq, S, ym, N, s); break;
                case 5: e = launch_int4<5>(xm, Kd, N, Wq, S, ym, N, s); break;
                case 6: e = launch_int4<6>(xm, Kd, N, Wq, S, ym, N, s); break;
                case 7: e = launch_int4<7>(xm, Kd, N, Wq, S, ym, N, s); break;
                default: e = launch_int4<8>(xm, Kd, N, Wq, S, ym, N, s); break;
            }
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mtpv
