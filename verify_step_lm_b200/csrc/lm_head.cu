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

// In-place nibble dequantisation.  Nibble i of a 32-bit word sits at bits
// 4i..4i+3; OR-ing it (unshifted, for i <= 4) into the mantissa of 2^23 gives
// the float 2^23 + n*16^i exactly, and subtracting 2^23 + 8*16^i leaves
// (n - 8)*16^i exactly.  Nibbles 5..7 are taken from the word shifted right by
// 12 (positions 2..4).  The activations are stored pre-multiplied by 16^-p,
// so every product equals (n - 8) * x exactly, as in the plain definition.
__device__ __forceinline__ float nib_at(uint32_t w, uint32_t mask, float offset) {
    return __fsub_rn(__uint_as_float(0x4B000000u | (w & mask)), offset);
}

// Shared-memory layouts of fp32 activations, XOR-swizzled so that a warp's
// 128-bit loads (one chunk per lane, consecutive chunks in consecutive lanes)
// spread over all 32 banks.
//   int4 kernels: a chunk is 32 weights = 8 float4; float4 j of chunk c is
//   stored at position j ^ (c & 7).
//   bf16 kernel:  a chunk is 8 weights = 2 float4; float4 j of chunk c is
//   stored at position j ^ ((c >> 2) & 1).
__device__ __forceinline__ int swz32(int k) {
    const int c = k >> 5, j = (k >> 2) & 7;
    return (c << 5) | ((j ^ (c & 7)) << 2) | (k & 3);
}
__device__ __forceinline__ int swz8(int k) {
    const int c = k >> 3, j = (k >> 2) & 1;
    return (c << 3) | ((j ^ ((c >> 2) & 1)) << 2) | (k & 3);
}

// Activations for the int4 kernel: fp32, weight k of each group of 8 scaled by
// 16^-p with p = k%8 for k%8 <= 4, k%8 - 3 otherwise (see nib_at).
__device__ __forceinline__ float int4_x_scale(int k) {
    const int i = k & 7;
    const int p = i <= 4 ? i : i - 3;
    return __uint_as_float((uint32_t)(127 - 4 * p) << 23);  // 2^(-4p)
}

// Eight dequantised weights (n - 8) * 16^p of one 32-bit word.
__device__ __forceinline__ void int4_word_dequant(uint32_t w, float (&f)[8]) {
    const uint32_t w2 = w >> 12;
    f[0] = nib_at(w, 0xFu, 8388616.0f);
    f[1] = nib_at(w, 0xF0u, 8388736.0f);
    f[2] = nib_at(w, 0xF00u, 8390656.0f);
    f[3] = nib_at(w, 0xF000u, 8421376.0f);
    f[4] = nib_at(w, 0xF0000u, 8912896.0f);
    f[5] = nib_at(w2, 0xF00u, 8390656.0f);
    f[6] = nib_at(w2, 0xF000u, 8421376.0f);
    f[7] = nib_at(w2, 0xF0000u, 8912896.0f);
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int q) {
    return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

template <int M, int RW, int U>
__global__ void __launch_bounds__(kGemvThreads) lm_head_int4_v2_kernel(
    const uint16_t *__restrict__ x, int Kd, int N, const uint8_t *__restrict__ Wq,
    const uint16_t *__restrict__ S, float *__restrict__ y, int ldy) {
    extern __shared__ float xsf[];  // [M][Kd] fp32, pre-scaled
    for (int i = threadIdx.x; i < M * Kd; i += kGemvThreads) {
        const int m = i / Kd, k = i - m * Kd;
        xsf[m * Kd + swz32(k)] = __uint_as_float((uint32_t)x[i] << 16) * int4_x_scale(k);
    }
    __syncthreads();

    const int nch = Kd >> 5;   // 16-byte chunks (32 weights) per row
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
                    for (int q = 0; q < 4; ++q) {
                        float4 xa[M], xb[M];
#pragma unroll
                        for (int m = 0; m < M; ++m) {
                            xa[m] = *reinterpret_cast<const float4 *>(xsf + m * Kd + c * 32 + (((2 * q) ^ (c & 7)) << 2));
                            xb[m] = *reinterpret_cast<const float4 *>(xsf + m * Kd + c * 32 + (((2 * q + 1) ^ (c & 7)) << 2));
                        }
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            float f[8];
                            int4_word_dequant(word_of(wv[u][r], q), f);
#pragma unroll
                            for (int m = 0; m < M; ++m) {
                                float t = part[r][m];
                                t = fmaf(f[0], xa[m].x, t); t = fmaf(f[1], xa[m].y, t);
                                t = fmaf(f[2], xa[m].z, t); t = fmaf(f[3], xa[m].w, t);
                                t = fmaf(f[4], xb[m].x, t); t = fmaf(f[5], xb[m].y, t);
                                t = fmaf(f[6], xb[m].z, t); t = fmaf(f[7], xb[m].w, t);
                                part[r][m] = t;
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

// Paired fp32 arithmetic of sm_100 (two lanes of work per instruction).
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(*reinterpret_cast<unsigned long long *>(&d))
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)));
    return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(*reinterpret_cast<unsigned long long *>(&d))
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)),
          "l"(*reinterpret_cast<unsigned long long *>(&c)));
    return d;
}

// As lm_head_int4_v2_kernel with the dequantising subtractions and the FMAs
// issued as f32x2 pairs; each (row, activation) keeps an even and an odd
// partial sum.
template <int M, int RW, int U>
__global__ void __launch_bounds__(kGemvThreads) lm_head_int4_v3_kernel(
    const uint16_t *__restrict__ x, int Kd, int N, const uint8_t *__restrict__ Wq,
    const uint16_t *__restrict__ S, float *__restrict__ y, int ldy) {
    extern __shared__ float xsf[];  // [M][Kd] fp32, pre-scaled
    for (int i = threadIdx.x; i < M * Kd; i += kGemvThreads) {
        const int m = i / Kd, k = i - m * Kd;
        xsf[m * Kd + swz32(k)] = __uint_as_float((uint32_t)x[i] << 16) * int4_x_scale(k);
    }
    __syncthreads();

    const int nch = Kd >> 5;
    const int ng = Kd >> 6;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int groups = (N + RW - 1) / RW;
    const float2 off01 = make_float2(8388616.0f, 8388736.0f);
    const float2 off23 = make_float2(8390656.0f, 8421376.0f);
    const float2 off45 = make_float2(8912896.0f, 8390656.0f);
    const float2 off67 = make_float2(8421376.0f, 8912896.0f);
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
                    float2 part[RW][M];
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int m = 0; m < M; ++m) part[r][m] = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float4 xa[M], xb[M];
#pragma unroll
                        for (int m = 0; m < M; ++m) {
                            xa[m] = *reinterpret_cast<const float4 *>(xsf + m * Kd + c * 32 + (((2 * q) ^ (c & 7)) << 2));
                            xb[m] = *reinterpret_cast<const float4 *>(xsf + m * Kd + c * 32 + (((2 * q + 1) ^ (c & 7)) << 2));
                        }
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            const uint32_t w = word_of(wv[u][r], q);
                            const uint32_t w2 = w >> 12;
                            const float2 f01 = sub2(make_float2(__uint_as_float(0x4B000000u | (w & 0xFu)),
                                                                __uint_as_float(0x4B000000u | (w & 0xF0u))), off01);
                            const float2 f23 = sub2(make_float2(__uint_as_float(0x4B000000u | (w & 0xF00u)),
                                                                __uint_as_float(0x4B000000u | (w & 0xF000u))), off23);
                            const float2 f45 = sub2(make_float2(__uint_as_float(0x4B000000u | (w & 0xF0000u)),
                                                                __uint_as_float(0x4B000000u | (w2 & 0xF00u))), off45);
                            const float2 f67 = sub2(make_float2(__uint_as_float(0x4B000000u | (w2 & 0xF000u)),
                                                                __uint_as_float(0x4B000000u | (w2 & 0xF0000u))), off67);
#pragma unroll
                            for (int m = 0; m < M; ++m) {
                                float2 t = part[r][m];
                                t = fma2(f01, make_float2(xa[m].x, xa[m].y), t);
                                t = fma2(f23, make_float2(xa[m].z, xa[m].w), t);
                                t = fma2(f45, make_float2(xb[m].x, xb[m].y), t);
                                t = fma2(f67, make_float2(xb[m].z, xb[m].w), t);
                                part[r][m] = t;
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int m = 0; m < M; ++m)
                            acc[r][m] = fmaf(sc[u][r], part[r][m].x + part[r][m].y, acc[r][m]);
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

// bf16 weights with the activations staged as fp32 (no per-use widening).
template <int M, int RW, int U>
__global__ void __launch_bounds__(kGemvThreads) lm_head_bf16_xf32_kernel(
    const uint16_t *__restrict__ x, int Kd, int N, const uint16_t *__restrict__ W,
    float *__restrict__ y, int ldy) {
    extern __shared__ float xsf[];  // [M][Kd]
    for (int i = threadIdx.x; i < M * Kd; i += kGemvThreads) {
        const int m = i / Kd, k = i - m * Kd;
        xsf[m * Kd + swz8(k)] = __uint_as_float((uint32_t)x[i] << 16);
    }
    __syncthreads();
    const int nch = Kd >> 3;
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
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        const int sw = (c >> 2) & 1;
                        const float4 a = *reinterpret_cast<const float4 *>(xsf + m * Kd + c * 8 + (sw << 2));
                        const float4 b = *reinterpret_cast<const float4 *>(xsf + m * Kd + c * 8 + ((sw ^ 1) << 2));
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            const uint4 w = wv[u][r];
                            float t = acc[r][m];
                            t = fmaf(a.x, bf16_lo(w.x), t); t = fmaf(a.y, bf16_hi(w.x), t);
                            t = fmaf(a.z, bf16_lo(w.y), t); t = fmaf(a.w, bf16_hi(w.y), t);
                            t = fmaf(b.x, bf16_lo(w.z), t); t = fmaf(b.y, bf16_hi(w.z), t);
                            t = fmaf(b.z, bf16_lo(w.w), t); t = fmaf(b.w, bf16_hi(w.w), t);
                            acc[r][m] = t;
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
// int4 group-64 weights on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate).  At M <= 8 the CUDA-core form above is bound by its
// dequantisation and FMA issue (ncu: ALU and FMA pipes both busy, DRAM far
// from peak), so the draft head uses this form: the weights are the A
// operand (16 vocabulary rows x 16 k), the activations the B operand (k x 8
// activation rows).  Dequantisation writes the A registers directly: one
// LOP3 per two weights, ((w >> 4j) & 0x000F000F) | 0x43004300 is the bf16
// pair (128 + n_j, 128 + n_{j+4}), exact.  Each 64-weight group gets a fresh
// accumulator so its scale applies exactly; the +128 offset is removed with
// the group's activation sum: sum (n - 8) x = sum (128 + n) x - 136 sum x.
//
// Lane (g = lane/4, t = lane%4) loads 8 bytes (16 nibbles, physical k
// 16t..16t+15 of the group) of rows g and g+8 of the 16-row block.  MMA j
// (j = 0..3) of a group takes, for logical k (2t, 2t+1, 2t+8, 2t+9), the
// physical k (16t + j, +4, +8, +12); the activations are stored in shared
// memory already in that order, so each lane's B fragments for the 4 MMAs of
// a group are 32 contiguous bytes.  Rows of that layout are padded to an odd
// number of 16-byte chunks, which keeps the 128-bit loads conflict-free.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t nib_pair_bf16(uint32_t w, int j) {
    return ((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u;
}

__device__ __forceinline__ uint2 ld_stream8(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v2.u32 {%0,%1}, [%2];"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p));
    return r;
}

// Position (in bf16 units, within one activation row of the staged layout) of
// activation k: group G, quad t, MMA j, slot s with k % 64 = 16t + j + 4s.
__device__ __forceinline__ int mma_x_pos(int k) {
    const int G = k >> 6, kk = k & 63;
    const int t = kk >> 4, w = kk & 15;
    const int j = w & 3, sl = w >> 2;
    return G * 64 + t * 16 + j * 4 + sl;
}

template <int RB, int U>
__global__ void __launch_bounds__(kGemvThreads) lm_head_int4_mma_kernel(
    const uint16_t *__restrict__ x, int M, int Kd, int N, const uint8_t *__restrict__ Wq,
    const uint16_t *__restrict__ S, float *__restrict__ y, int ldy) {
    extern __shared__ uint4 smem_mma[];
    const int Gt = Kd >> 6;
    const int rowc = Gt * 8 + 1;  // 16-byte chunks per staged activation row (odd)
    uint16_t *xb = reinterpret_cast<uint16_t *>(smem_mma);                   // [M][rowc * 8]
    float *xs = reinterpret_cast<float *>(smem_mma + M * rowc);              // [Gt][8]
    // stage: permuted bf16 activations of the M real rows, and group sums
    for (int i = threadIdx.x; i < M * Kd; i += kGemvThreads) {
        const int m = i / Kd, k = i - m * Kd;
        xb[m * rowc * 8 + mma_x_pos(k)] = x[i];
    }
    for (int i = threadIdx.x; i < Gt * 8; i += kGemvThreads) {
        const int G = i >> 3, m = i & 7;
        float sum = 0.0f;
        if (m < M)
            for (int k = 0; k < 64; ++k) sum += __uint_as_float((uint32_t)x[m * Kd + G * 64 + k] << 16);
        xs[i] = sum;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int rowbytes = Kd >> 1;
    const bool has_row = g < M;                // lanes g >= M feed zero activations
    const uint4 *xrow = smem_mma + (has_row ? g : 0) * rowc;
    const int nblk = (N + 15) / 16;
    const int ntask = (nblk + RB - 1) / RB;
    for (int task = blockIdx.x * kGemvWarps + warp; task < ntask; task += gridDim.x * kGemvWarps) {
        const uint8_t *wr[RB][2];
        const uint16_t *sr[RB][2];
#pragma unroll
        for (int rb = 0; rb < RB; ++rb)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = min((task * RB + rb) * 16 + g + 8 * h, N - 1);
                wr[rb][h] = Wq + (size_t)row * rowbytes + 8 * t;
                sr[rb][h] = S + (size_t)row * Gt;
            }
        float acc[RB][4];
#pragma unroll
        for (int rb = 0; rb < RB; ++rb)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[rb][e] = 0.0f;

        for (int G0 = 0; G0 < Gt; G0 += U) {
            uint2 wv[U][RB][2];
            float sc[U][RB][2];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int G = G0 + u;
                        wv[u][rb][h] = G < Gt ? ld_stream8(wr[rb][h] + G * 32) : make_uint2(0, 0);
                        sc[u][rb][h] = G < Gt ? __uint_as_float((uint32_t)__ldg(sr[rb][h] + G) << 16) : 0.0f;
                    }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int G = G0 + u;
                if (G < Gt) {
                    const uint4 z4 = make_uint4(0, 0, 0, 0);
                    const uint4 bA = has_row ? xrow[G * 8 + 2 * t] : z4;
                    const uint4 bB = has_row ? xrow[G * 8 + 2 * t + 1] : z4;
                    const uint32_t bl[4] = {bA.x, bA.z, bB.x, bB.z};  // b0b1 of MMA j
                    const uint32_t bh[4] = {bA.y, bA.w, bB.y, bB.w};  // b2b3 of MMA j
                    const float2 xsum = *reinterpret_cast<const float2 *>(xs + G * 8 + 2 * t);
#pragma unroll
                    for (int rb = 0; rb < RB; ++rb) {
                        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t a[4] = {nib_pair_bf16(wv[u][rb][0].x, j),
                                                   nib_pair_bf16(wv[u][rb][1].x, j),
                                                   nib_pair_bf16(wv[u][rb][0].y, j),
                                                   nib_pair_bf16(wv[u][rb][1].y, j)};
                            mma_bf16_16816(c, a, bl[j], bh[j]);
                        }
                        const float s0 = sc[u][rb][0], s1 = sc[u][rb][1];
                        acc[rb][0] = fmaf(s0, fmaf(-136.0f, xsum.x, c[0]), acc[rb][0]);
                        acc[rb][1] = fmaf(s0, fmaf(-136.0f, xsum.y, c[1]), acc[rb][1]);
                        acc[rb][2] = fmaf(s1, fmaf(-136.0f, xsum.x, c[2]), acc[rb][2]);
                        acc[rb][3] = fmaf(s1, fmaf(-136.0f, xsum.y, c[3]), acc[rb][3]);
                    }
                }
            }
        }
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
            const int r0 = (task * RB + rb) * 16;
            const int m0 = 2 * t, m1 = 2 * t + 1;
            const int ra = r0 + g, rbw = r0 + g + 8;
            if (m0 < M && ra < N) y[(size_t)m0 * ldy + ra] = acc[rb][0];
            if (m1 < M && ra < N) y[(size_t)m1 * ldy + ra] = acc[rb][1];
            if (m0 < M && rbw < N) y[(size_t)m0 * ldy + rbw] = acc[rb][2];
            if (m1 < M && rbw < N) y[(size_t)m1 * ldy + rbw] = acc[rb][3];
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
    constexpr int RW = M <= 4 ? 4 : 2;
    constexpr int U = 4;
    auto k = lm_head_bf16_xf32_kernel<M, RW, U>;
    const size_t smem = (size_t)M * Kd * sizeof(float);
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
    constexpr int RW = M <= 4 ? 4 : 2;
    constexpr int U = 2;
    auto k = lm_head_int4_v3_kernel<M, RW, U>;
    const size_t smem = (size_t)M * Kd * sizeof(float);
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

// Shared memory of the tensor-core int4 kernel for M (<= 8) activation rows.
static size_t int4_mma_smem(int M, int Kd) {
    const size_t Gt = (size_t)Kd / 64;
    return (size_t)M * (Gt * 8 + 1) * 16 + Gt * 8 * sizeof(float);
}

static cudaError_t launch_int4_mma(const uint16_t *x, int M, int Kd, int N, const uint8_t *Wq,
                                   const uint16_t *S, float *y, int ldy, cudaStream_t s) {
    constexpr int RB = 2, U = 4;
    auto k = lm_head_int4_mma_kernel<RB, U>;
    const size_t smem = int4_mma_smem(M, Kd);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int ntask = ((N + 15) / 16 + RB - 1) / RB;
    const int need = (ntask + kGemvWarps - 1) / kGemvWarps;
    const int grid = std::min(need, kSMs * resident_ctas(k, smem));
    k<<<grid, kGemvThreads, smem, s>>>(x, M, Kd, N, Wq, S, y, ldy);
    return cudaGetLastError();
}

size_t lm_head_max_smem_rows(int Kd) {
    // rows of fp32 activations that fit in 227 KB of shared memory
    return (size_t)(227 * 1024) / ((size_t)Kd * sizeof(float));
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
            if (int4_mma_smem(mm, Kd) <= (size_t)227 * 1024) {
                e = launch_int4_mma(xm, mm, Kd, N, Wq, S, ym, N, s);
                if (e != cudaSuccess) return e;
                continue;
            }
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
