// Small-M weight-streaming projection y[M, N] = x[M, Kd] . Wd[N, Kd]^T.
//
// The pages' verify pass ends in a matmul with only M = 3..6 activation rows
// (hazakura.dev MTPLX notes, Layer 0: a shader rewritten for small matrices)
// and drafts through a 4-bit copy of the LM head (same section); decode GEMVs
// dequantise inside the inner loop, one kernel per storage format
// (gist.science BaseRT explainer, methodology: specialisation).
//
// At M <= 8 every weight is used M times, so the work is an HBM stream and the
// kernels are built around keeping enough bytes in flight with as few
// instructions as possible; both heads run on the tensor cores (mma.sync
// m16n8k16, fp32 accumulate), the weights as the A operand straight from
// global loads, the activations as the B operand from shared memory:
//   bf16 head   one MMA stands for 64 FMAs and 16 bf16 widenings per lane,
//               which leaves the warps free to keep 8 KB of loads in flight
//               each (16-byte non-allocating loads, 16-row tiles).
//   int4 head   on CUDA cores the dequantisation plus M FMAs per weight left
//               the ALU and FMA pipes as the limit at a third of HBM
//               bandwidth, so the weights are dequantised straight into MMA A
//               registers.  Each warp streams 16-row tiles through its own
//               cp.async ring in shared memory.
// A persistent grid of (SMs x resident CTAs) walks the row blocks.
#include <algorithm>

#include <cuda_fp16.h>

#include "common.cuh"
#include "lm_head.cuh"
#include "lm_head_tc.cuh"

namespace mtpv {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

// ---------------------------------------------------------------------------
// bf16 head on the tensor cores (mma.sync m16n8k16 bf16, fp32 accumulate):
// the weights are the A operand (16 vocabulary rows x 16 k), the activation
// rows the B operand (k x 8 rows, NT n-tiles of 8 rows).  At M <= 8 the head
// is an HBM stream and the MMA is there to save issue slots: one MMA does the
// work of 64 FMAs plus 16 bf16 widenings per lane, so the warps spend their
// time keeping loads in flight.  The reduction index is permuted inside every
// 32-k step so that each lane's fragments are contiguous: lane (g, t) holds
// physical k 8t..8t+7 of the step, the first four for the step's first MMA
// and the last four for its second (logical k 2t, 2t+1, 2t+8, 2t+9 of an MMA
// are physical 8t + 0..3, or 8t + 4..7).  The A fragments are then one
// 16-byte global load per row, 64 contiguous bytes per row per warp, and the
// B fragments one 16-byte shared-memory load per n-tile; activation rows are
// staged as bf16 with a pitch of Kd + 32 elements (64 bytes of padding),
// which puts the two rows of a quarter-warp on different halves of the banks.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int kBmmaThreads = 512;
constexpr int kBmmaU = 8;  // 32-k steps in flight per lane: 8 KB of weights per warp

// Stage M activation rows (bf16 [M, Kd]) at xs with pitch Kd + 32; every
// thread of the block takes part, the caller places the barrier.
__device__ __forceinline__ void bf16_mma_stage_x(uint16_t *xs, const uint16_t *__restrict__ x, int M,
                                                 int Kd) {
    const int pitch = Kd + 32;
    for (int i = threadIdx.x; i < M * (Kd / 8); i += blockDim.x) {
        const int m = i / (Kd / 8), c = i - m * (Kd / 8);
        *reinterpret_cast<uint4 *>(xs + (size_t)m * pitch + c * 8) =
            *reinterpret_cast<const uint4 *>(x + (size_t)m * Kd + c * 8);
    }
}

// One 16-row tile (rows 16 tile .. 16 tile + 15) of y[M, N] for the calling warp.
template <int NT, int U>
__device__ __forceinline__ void bf16_mma_tile(const uint16_t *xs, int M, int Kd, int N,
                                              const uint16_t *__restrict__ W, float *__restrict__ y,
                                              int ldy, int tile) {
    const int pitch = Kd + 32;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    const int r0 = tile * 16;
    const uint4 *wa = reinterpret_cast<const uint4 *>(W + (size_t)min(r0 + g, N - 1) * Kd) + t;
    const uint4 *wb = reinterpret_cast<const uint4 *>(W + (size_t)min(r0 + g + 8, N - 1) * Kd) + t;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
    for (int k0 = 0; k0 < Kd; k0 += 32 * U) {
        uint4 va[U], vb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool in = k0 + 32 * u < Kd;
            va[u] = in ? ld_stream16(wa + (k0 + 32 * u) / 8) : z4;
            vb[u] = in ? ld_stream16(wb + (k0 + 32 * u) / 8) : z4;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = k0 + 32 * u;
            if (k < Kd) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int n = nt * 8 + g;
                    const uint4 xv = n < M ? *reinterpret_cast<const uint4 *>(xs + (size_t)n * pitch + k + 8 * t)
                                           : z4;
                    const uint32_t a0[4] = {va[u].x, vb[u].x, va[u].y, vb[u].y};
                    const uint32_t a1[4] = {va[u].z, vb[u].z, va[u].w, vb[u].w};
                    mma_bf16_16816(acc[nt], a0, xv.x, xv.y);
                    mma_bf16_16816(acc[nt], a1, xv.z, xv.w);
                }
            }
        }
    }
    const int ra = r0 + g, rb = ra + 8;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int m0 = nt * 8 + 2 * t, m1 = m0 + 1;
        if (m0 < M) {
            if (ra < N) y[(size_t)m0 * ldy + ra] = acc[nt][0];
            if (rb < N) y[(size_t)m0 * ldy + rb] = acc[nt][2];
        }
        if (m1 < M) {
            if (ra < N) y[(size_t)m1 * ldy + ra] = acc[nt][1];
            if (rb < N) y[(size_t)m1 * ldy + rb] = acc[nt][3];
        }
    }
}

// M <= 8 * NT rows: the CTA stages x, then its warps walk the 16-row tiles.
template <int NT, int U>
__global__ void __launch_bounds__(kBmmaThreads, 1) lm_head_bf16_mma_kernel(
    const uint16_t *__restrict__ x, int M, int Kd, int N, const uint16_t *__restrict__ W,
    float *__restrict__ y, int ldy) {
    extern __shared__ uint4 smem_bm[];
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem_bm);
    bf16_mma_stage_x(xs, x, M, Kd);
    __syncthreads();
    const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int ntiles = (N + 15) / 16;
    for (int tile = blockIdx.x * nwarps + warp; tile < ntiles; tile += gridDim.x * nwarps)
        bf16_mma_tile<NT, U>(xs, M, Kd, N, W, y, ldy, tile);
}

// ---------------------------------------------------------------------------
// int4 group-64 weights on the tensor cores (mma.sync m16n8k16, fp32
// accumulate).  The weights are the A operand (16 vocabulary rows x 16 k), the
// activations the B operand (k x 8 activation rows).  Lane (g = lane/4,
// t = lane%4) holds 8 bytes (16 nibbles, physical k 16t..16t+15 of a 64-weight
// group) of rows g and g+8 of a 16-row tile.  MMA j (j = 0..3) of a group
// takes, for logical k (2t, 2t+1, 2t+8, 2t+9), the physical k (16t + j, +4,
// +8, +12); the activations are staged in shared memory already in that
// order, so each lane's B fragments for the 4 MMAs of a group are 32
// contiguous bytes.  Staged rows are padded to an odd number of 16-byte
// chunks, which keeps the 128-bit loads conflict-free.  Each group gets a
// fresh accumulator so its bf16 scale applies exactly.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint2 ld_stream8(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v2.u32 {%0,%1}, [%2];"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p));
    return r;
}

// Position (in 16-bit units, within one activation row of the staged layout)
// of activation k: group G, quad t, MMA j, slot s with k % 64 = 16t + j + 4s.
__device__ __forceinline__ int mma_x_pos(int k) {
    const int G = k >> 6, kk = k & 63;
    const int t = kk >> 4, w = kk & 15;
    const int j = w & 3, sl = w >> 2;
    return G * 64 + t * 16 + j * 4 + sl;
}

// ---------------------------------------------------------------------------
// cp.async ring used by the fp16 int4 kernel: every warp owns NST
// shared-memory stages, each a 16-row x GPS-group tile of the head (and its
// scales), filled with 16-byte cp.async copies while the warp computes on an
// earlier stage.  Tile rows are XOR-swizzled in 16-byte chunks (chunk c of
// row r at c ^ (r & 7)) and tile row 2i feeds MMA row i, row 2i + 1 MMA row
// i + 8: the four rows a half-warp reads in one instruction then have four
// different swizzles, so the per-lane 8-byte fragment reads cover all 32
// banks once.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int GPS, int NST>
struct Int4Ring {
    static constexpr int kTileBytes = 16 * GPS * 32;   // 16 rows x GPS groups of 32 bytes
    static constexpr int kScaleBytes = 16 * GPS * 2;   // 16 rows x GPS bf16 scales
    static constexpr int kStageBytes = kTileBytes + kScaleBytes;
    static constexpr int kWarpBytes = NST * kStageBytes;
};

// fp16 dequantisation on the tensor cores.  A word's nibbles become fp16
// pairs with three shifts and four LOP3 (the magic-number conversion of Kim
// et al., "Who Says Elephants Can't Run", 2022, and the Marlin kernel,
// Frantar et al., 2024): with nibble n_j moved to bits 4..7 of the low half
// and n_{j+4} to bits 4..7 of the high half,
//   (v & 0x00F000F0) | 0x64006400 = (1024 + 16 n_j, 1024 + 16 n_{j+4})
// exactly.  Every activation is staged divided by 16, so a weight contributes
// (64 + n) x, and each group's offset term 72 x (1152 x / 16 per weight) is
// removed with a precomputed sum: the offset is 72 weight steps, which keeps
// the fp32 cancellation small (putting the nibble at bit 0 instead would make
// it 1032 steps).  The activations are fp16 after a per-row power-of-two
// scale that puts the row's largest |x| in [2^9, 2^10) before the division
// by 16 (undone on the output): a bf16 value carries 8 significant bits, so
// the fp16 copy is exact for every element down to 2^-23 of the row's largest
// |x|; smaller ones fall among the fp16 subnormals, off by at most 2^-30 of
// the row maximum (or flushed to zero).  Layouts as in the bf16 kernels.
__device__ __forceinline__ void mma_f16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16_16816_zc(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// the four fp16 pairs of one word (pair j = weights (j, j + 4) of the word),
// each (1024 + 16 n_j, 1024 + 16 n_{j+4})
__device__ __forceinline__ void nib_pairs_f16(uint32_t w, uint32_t (&p)[4]) {
    p[0] = ((w << 4) & 0x00F000F0u) | 0x64006400u;
    p[1] = (w & 0x00F000F0u) | 0x64006400u;
    p[2] = ((w >> 4) & 0x00F000F0u) | 0x64006400u;
    p[3] = ((w >> 8) & 0x00F000F0u) | 0x64006400u;
}

// Activation staging of the fp16 int4 kernels: per-row power-of-two
// prescale, fp16, permuted (plus, with zero_row, a row of zeros at index M),
// and the per-group offset sums.  Every thread of the block takes part; the block synchronises inside.
// Per-row pieces of the staging, shared by the block-wide staging below and
// the one-CTA-per-row staging kernel of the split-K projection.
// Largest |x| of the row as an fp32 bit pattern, per calling warp (every
// thread of the block walks the row; reduce the warps' values with max).
__device__ __forceinline__ uint32_t int4_row_absmax_warp(const uint16_t *__restrict__ xrow, int Kd) {
    const uint4 *xr = reinterpret_cast<const uint4 *>(xrow);
    uint32_t a = 0u;
    for (int c = threadIdx.x; c < (Kd >> 3); c += blockDim.x) {
        const uint4 v = xr[c];
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            a = max(a, max((w4[q] << 16) & 0x7fffffffu, ((w4[q] >> 16) << 16) & 0x7fffffffu));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
    return a;
}
// sh: the row's largest |x| times 2^-sh lies in [2^9, 2^10) (e: the largest
// exponent with 2^e <= max|x|); an all-zero row keeps sh = 0.
__device__ __forceinline__ int int4_row_shift(uint32_t amax) {
    const int sh = amax ? (int)(amax >> 23) - 127 - 9 : 0;
    return max(-100, min(100, sh));
}
// 8 activations per step (k = 8c .. 8c+7, one 16-byte load): in the layout
// of mma_x_pos, value w of the chunk goes to group position
// 16 ((c >> 1) & 3) + 4 (w & 3) + 2 (c & 1) + (w >> 2), so values w and w + 4
// are adjacent: four 32-bit stores of fp16 pairs.  Scale 2^-(sh + 4): the
// row's power-of-two factor, then / 16.
__device__ __forceinline__ void int4_row_convert(const uint16_t *__restrict__ xrow, int Kd, int sh,
                                                 uint16_t *dst_row) {
    const float f = __uint_as_float((uint32_t)(127 - (sh + 4)) << 23);
    const uint4 *xr = reinterpret_cast<const uint4 *>(xrow);
    uint32_t *dst = reinterpret_cast<uint32_t *>(dst_row);
    for (int c = threadIdx.x; c < (Kd >> 3); c += blockDim.x) {
        const uint4 v = xr[c];
        const float e[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                            bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
        const int base = (c >> 3) * 64 + ((c >> 1) & 3) * 16 + 2 * (c & 1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half2 h = __floats2half2_rn(e[j] * f, e[j + 4] * f);
            dst[(base + 4 * j) >> 1] = *reinterpret_cast<const uint32_t *>(&h);
        }
    }
}
// Offset sum of group G of a staged row: 1152 x (sum of the group's 64 staged
// activations), by a fixed shuffle tree; the calling warp's lane 0 gets it.
__device__ __forceinline__ float int4_group_offset(const uint16_t *staged_row, int G) {
    const int lane = threadIdx.x & 31;
    const uint16_t *r = staged_row + G * 64;
    float v = __half2float(__ushort_as_half(r[lane])) + __half2float(__ushort_as_half(r[lane + 32]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return 1152.0f * v;
}

__device__ __forceinline__ void int4_f16_stage_x(uint16_t *xb, float *xs, unsigned int *row_amax,
                                                 float *row_unscale, const uint16_t *__restrict__ x,
                                                 int M, int Kd, bool zero_row) {
    const int Gt = Kd >> 6;
    const int rowc = Gt * 8 + 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if (threadIdx.x < 8) row_amax[threadIdx.x] = 0u;
    __syncthreads();
    for (int m = 0; m < M; ++m) {  // row maxima: per warp, then one shared atomic per warp
        const uint32_t a = int4_row_absmax_warp(x + (size_t)m * Kd, Kd);
        if (lane == 0 && a) atomicMax(&row_amax[m], a);
    }
    if (zero_row)
        for (int i = threadIdx.x; i < rowc * 8; i += blockDim.x) xb[M * rowc * 8 + i] = 0;
    __syncthreads();
    if (threadIdx.x < 8) {
        const int sh = int4_row_shift(row_amax[threadIdx.x]);
        row_unscale[threadIdx.x] = __uint_as_float((uint32_t)(127 + sh) << 23);
        row_amax[threadIdx.x] = (uint32_t)sh;  // read back as int
    }
    __syncthreads();
    for (int m = 0; m < M; ++m)
        int4_row_convert(x + (size_t)m * Kd, Kd, (int)row_amax[m], xb + (size_t)m * rowc * 8);
    __syncthreads();
    for (int i = warp; i < Gt * 8; i += nw) {  // offset sums, one warp per (group, row)
        const int G = i >> 3, m = i & 7;
        const float v = m < M ? int4_group_offset(xb + (size_t)m * rowc * 8, G) : 0.0f;
        if (lane == 0) xs[i] = v;
    }
    __syncthreads();
}

// The 16-row tiles of warp gw of nw warps (grid-wide numbering), streamed
// through the warp's own ring at `ring`.
template <int GPS, int NST>
__device__ __forceinline__ void int4_f16_tiles(const uint4 *xstage, const float *xs,
                                               const float *row_unscale, unsigned char *ring,
                                               int M, int Kd, int N,
                                               const uint8_t *__restrict__ Wq,
                                               const uint16_t *__restrict__ S, float *__restrict__ y,
                                               int ldy, int gw, int nw) {
    using R = Int4Ring<GPS, NST>;
    static_assert(GPS % 8 == 0, "scale rows are copied in 16-byte chunks");
    const int Gt = Kd >> 6;
    const int rowc = Gt * 8 + 1;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const size_t rowbytes = (size_t)(Kd >> 1);
    const uint4 *xrow = xstage + (g < M ? g : M) * rowc + 2 * t;
    const float *xsl = xs + 2 * t;
    const int nblk = (N + 15) / 16;
    const int nst = Gt / GPS;
    const int first = gw, stride = nw;

    // per-lane copy pattern of a stage: chunk q = lane + 32 i of the 16 x (2 GPS) tile
    constexpr int kCp = GPS;  // 16-byte weight chunks per lane per stage
    int cp_row[kCp], cp_soff[kCp], cp_goff[kCp];
#pragma unroll
    for (int i = 0; i < kCp; ++i) {
        const int q = lane + 32 * i;
        const int r = q / (2 * GPS), c = q % (2 * GPS);
        cp_row[i] = r;
        cp_soff[i] = r * (GPS * 32) + ((c ^ (r & 7)) << 4);
        cp_goff[i] = c * 16;
    }
    const int sc_r = lane / (GPS / 8), sc_c = lane % (GPS / 8);

    int it_task = first, it_st = 0, it_slot = 0;  // next tile to issue
    auto issue = [&]() {
        if (it_task < nblk) {
            unsigned char *slot = ring + it_slot * R::kStageBytes;
            const uint8_t *base = Wq + (size_t)it_st * GPS * 32;
#pragma unroll
            for (int i = 0; i < kCp; ++i) {
                const int row = min(it_task * 16 + cp_row[i], N - 1);
                cp_async16(slot + cp_soff[i], base + row * rowbytes + cp_goff[i]);
            }
            if (lane < 2 * GPS) {
                const int row = min(it_task * 16 + sc_r, N - 1);
                cp_async16(slot + R::kTileBytes + sc_r * (GPS * 2) + sc_c * 16,
                           S + (size_t)row * Gt + (size_t)it_st * GPS + sc_c * 8);
            }
            if (++it_st == nst) { it_st = 0; it_task += stride; }
            if (++it_slot == NST) it_slot = 0;
        }
        cp_async_commit();
    };

#pragma unroll
    for (int k = 0; k < NST - 1; ++k) issue();
    int slot_i = 0;
    for (int task = first; task < nblk; task += stride) {
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int st = 0; st < nst; ++st) {
            issue();
            cp_async_wait<NST - 1>();
            __syncwarp();
            const unsigned char *slot = ring + slot_i * R::kStageBytes;
            if (++slot_i == NST) slot_i = 0;
            const uint16_t *ssl = reinterpret_cast<const uint16_t *>(slot + R::kTileBytes);
            // MMA row g is tile row 2g, MMA row g + 8 is tile row 2g + 1
            const unsigned char *rowg = slot + (2 * g) * (GPS * 32) + 8 * (t & 1);
            const unsigned char *rowg8 = rowg + GPS * 32;
            const uint4 *xr = xrow + st * GPS * 8;
            const float *xc = xsl + st * GPS * 8;
#pragma unroll
            for (int gq = 0; gq < GPS; ++gq) {
                const int sw = ((2 * gq + (t >> 1)) ^ ((2 * g) & 7)) << 4;
                const uint2 w0 = *reinterpret_cast<const uint2 *>(rowg + sw);
                const uint2 w1 = *reinterpret_cast<const uint2 *>(rowg8 + (sw ^ 16));
                const float s0 = __uint_as_float((uint32_t)ssl[(2 * g) * GPS + gq] << 16);
                const float s1 = __uint_as_float((uint32_t)ssl[(2 * g + 1) * GPS + gq] << 16);
                const uint4 bA = xr[gq * 8];
                const uint4 bB = xr[gq * 8 + 1];
                const float2 corr = *reinterpret_cast<const float2 *>(xc + gq * 8);
                uint32_t p0x[4], p1x[4], p0y[4], p1y[4];
                nib_pairs_f16(w0.x, p0x);
                nib_pairs_f16(w1.x, p1x);
                nib_pairs_f16(w0.y, p0y);
                nib_pairs_f16(w1.y, p1y);
                float c[4];
                {
                    const uint32_t a[4] = {p0x[0], p1x[0], p0y[0], p1y[0]};
                    mma_f16_16816_zc(c, a, bA.x, bA.y);
                }
                {
                    const uint32_t a[4] = {p0x[1], p1x[1], p0y[1], p1y[1]};
                    mma_f16_16816(c, a, bA.z, bA.w);
                }
                {
                    const uint32_t a[4] = {p0x[2], p1x[2], p0y[2], p1y[2]};
                    mma_f16_16816(c, a, bB.x, bB.y);
                }
                {
                    const uint32_t a[4] = {p0x[3], p1x[3], p0y[3], p1y[3]};
                    mma_f16_16816(c, a, bB.z, bB.w);
                }
                acc[0] = fmaf(s0, c[0] - corr.x, acc[0]);
                acc[1] = fmaf(s0, c[1] - corr.y, acc[1]);
                acc[2] = fmaf(s1, c[2] - corr.x, acc[2]);
                acc[3] = fmaf(s1, c[3] - corr.y, acc[3]);
            }
            __syncwarp();  // every lane is done with this slot before it is refilled
        }
        const int r0 = task * 16;
        const int m0 = 2 * t, m1 = 2 * t + 1;
        const int ra = r0 + 2 * g, rbw = ra + 1;  // MMA rows g, g + 8
        if (m0 < M) {
            const float us = row_unscale[m0];
            if (ra < N) y[(size_t)m0 * ldy + ra] = acc[0] * us;
            if (rbw < N) y[(size_t)m0 * ldy + rbw] = acc[2] * us;
        }
        if (m1 < M) {
            const float us = row_unscale[m1];
            if (ra < N) y[(size_t)m1 * ldy + ra] = acc[1] * us;
            if (rbw < N) y[(size_t)m1 * ldy + rbw] = acc[3] * us;
        }
    }
    cp_async_wait<0>();
}

template <int GPS, int NST, int NT>
__global__ void __launch_bounds__(NT) lm_head_int4_f16_kernel(
    const uint16_t *__restrict__ x, int M, int Kd, int N, const uint8_t *__restrict__ Wq,
    const uint16_t *__restrict__ S, float *__restrict__ y, int ldy) {
    using R = Int4Ring<GPS, NST>;
    constexpr int NW = NT / 32;
    extern __shared__ uint4 smem_mma[];
    __shared__ unsigned int row_amax[8];
    __shared__ float row_unscale[8];
    const int Gt = Kd >> 6;
    const int rowc = Gt * 8 + 1;
    uint16_t *xb = reinterpret_cast<uint16_t *>(smem_mma);                   // [M + 1][rowc * 8] fp16
    float *xs = reinterpret_cast<float *>(smem_mma + (M + 1) * rowc);        // [Gt][8] offset sums
    unsigned char *rings = reinterpret_cast<unsigned char *>(xs + Gt * 8);   // [warps][NST][stage]
    int4_f16_stage_x(xb, xs, row_amax, row_unscale, x, M, Kd, true);
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    int4_f16_tiles<GPS, NST>(smem_mma, xs, row_unscale, rings + (size_t)warp * R::kWarpBytes, M, Kd,
                             N, Wq, S, y, ldy, blockIdx.x * NW + warp, gridDim.x * NW);
}

// ---------------------------------------------------------------------------
// Direct-load form of the fp16 int4 kernel: each lane loads its nibbles
// straight into registers (8 bytes per row and group) and computes exactly as
// the ring kernel does (same MMA operands, order and epilogue), so both forms
// give the same bits.  Used where the ring does not fit.
// ---------------------------------------------------------------------------
// Groups [gbeg, gend) of the RB tiles of task `task`, scaled back by the
// rows' power-of-two factors and stored to y.
template <int RB, int UI>
__device__ __forceinline__ void int4_f16_direct_task(const uint4 *xstage, const float *xs,
                                                     const float *row_unscale, int M, int Kd, int N,
                                                     const uint8_t *__restrict__ Wq,
                                                     const uint16_t *__restrict__ S,
                                                     float *__restrict__ y, int ldy, int task,
                                                     int gbeg, int gend) {
    const int Gt = Kd >> 6;
    const int rowc = Gt * 8 + 1;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const size_t rowbytes = (size_t)(Kd >> 1);
    const bool has_row = g < M;  // lanes of MMA columns past the last row feed zeros
    const uint4 *xrow = xstage + (has_row ? g : 0) * rowc + 2 * t;
    const float *xsl = xs + 2 * t;
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
    for (int G0 = gbeg; G0 < gend; G0 += UI) {
        uint2 wv[UI][RB][2];
        float sc[UI][RB][2];
#pragma unroll
        for (int u = 0; u < UI; ++u)
#pragma unroll
            for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int G = G0 + u;
                    wv[u][rb][h] = G < gend ? ld_stream8(wr[rb][h] + G * 32) : make_uint2(0, 0);
                    sc[u][rb][h] = G < gend ? __uint_as_float((uint32_t)__ldg(sr[rb][h] + G) << 16) : 0.0f;
                }
#pragma unroll
        for (int u = 0; u < UI; ++u) {
            const int G = G0 + u;
            if (G < gend) {
                const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
                const uint4 bA = has_row ? xrow[G * 8] : z4;
                const uint4 bB = has_row ? xrow[G * 8 + 1] : z4;
                const float2 corr = *reinterpret_cast<const float2 *>(xsl + G * 8);
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    uint32_t p0x[4], p1x[4], p0y[4], p1y[4];
                    nib_pairs_f16(wv[u][rb][0].x, p0x);
                    nib_pairs_f16(wv[u][rb][1].x, p1x);
                    nib_pairs_f16(wv[u][rb][0].y, p0y);
                    nib_pairs_f16(wv[u][rb][1].y, p1y);
                    float c[4];
                    {
                        const uint32_t a[4] = {p0x[0], p1x[0], p0y[0], p1y[0]};
                        mma_f16_16816_zc(c, a, bA.x, bA.y);
                    }
                    {
                        const uint32_t a[4] = {p0x[1], p1x[1], p0y[1], p1y[1]};
                        mma_f16_16816(c, a, bA.z, bA.w);
                    }
                    {
                        const uint32_t a[4] = {p0x[2], p1x[2], p0y[2], p1y[2]};
                        mma_f16_16816(c, a, bB.x, bB.y);
                    }
                    {
                        const uint32_t a[4] = {p0x[3], p1x[3], p0y[3], p1y[3]};
                        mma_f16_16816(c, a, bB.z, bB.w);
                    }
                    const float s0 = sc[u][rb][0], s1 = sc[u][rb][1];
                    acc[rb][0] = fmaf(s0, c[0] - corr.x, acc[rb][0]);
                    acc[rb][1] = fmaf(s0, c[1] - corr.y, acc[rb][1]);
                    acc[rb][2] = fmaf(s1, c[2] - corr.x, acc[rb][2]);
                    acc[rb][3] = fmaf(s1, c[3] - corr.y, acc[rb][3]);
                }
            }
        }
    }
    const int m0 = 2 * t, m1 = 2 * t + 1;
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
        const int ra = (task * RB + rb) * 16 + g, rbw = ra + 8;
        if (m0 < M) {
            const float us = row_unscale[m0];
            if (ra < N) y[(size_t)m0 * ldy + ra] = acc[rb][0] * us;
            if (rbw < N) y[(size_t)m0 * ldy + rbw] = acc[rb][2] * us;
        }
        if (m1 < M) {
            const float us = row_unscale[m1];
            if (ra < N) y[(size_t)m1 * ldy + ra] = acc[rb][1] * us;
            if (rbw < N) y[(size_t)m1 * ldy + rbw] = acc[rb][3] * us;
        }
    }
}

// Standalone direct-load fp16 kernel: the int4 shapes the ring kernel does not
// take (its staging or ring would not fit in shared memory, Kd not a
// multiple of 512, unaligned scales).  Same arithmetic as the ring kernel.
template <int RB, int UI>
__global__ void __launch_bounds__(kGemvThreads) lm_head_int4_f16_direct_kernel(
    const uint16_t *__restrict__ x, int M, int Kd, int N, const uint8_t *__restrict__ Wq,
    const uint16_t *__restrict__ S, float *__restrict__ y, int ldy) {
    extern __shared__ uint4 smem_dir[];
    __shared__ unsigned int row_amax[8];
    __shared__ float row_unscale[8];
    const int Gt = Kd >> 6;
    const int rowc = Gt * 8 + 1;
    uint16_t *xb = reinterpret_cast<uint16_t *>(smem_dir);               // [M][rowc * 8]
    float *xs = reinterpret_cast<float *>(smem_dir + (size_t)M * rowc);  // [Gt][8]
    int4_f16_stage_x(xb, xs, row_amax, row_unscale, x, M, Kd, false);
    const int tasks = ((N + 15) / 16 + RB - 1) / RB;
    for (int task = blockIdx.x * kGemvWarps + (threadIdx.x >> 5); task < tasks; task += gridDim.x * kGemvWarps)
        int4_f16_direct_task<RB, UI>(smem_dir, xs, row_unscale, M, Kd, N, Wq, S, y, ldy, task, 0, Kd >> 6);
}

constexpr int kMixWarps = 16;      // per CTA, one CTA per SM
constexpr int kMixInt4Warps = 3;   // the last 3 warps of a CTA own int4 rings
constexpr int kMixThreads = 32 * kMixWarps;

// Both heads of a verify step in one persistent launch.  The last
// kMixInt4Warps warps of every CTA first stream their share of the int4 head
// through their cp.async rings (bound by dequantisation and copy latency, not
// by HBM), then join the other warps on the bf16 head, whose 16-row tiles all
// warps take one at a time from a global counter (`work`, zero on entry), so
// the bf16 stream keeps every SM busy to the end whatever the int4 warps'
// speed.  Each head's values are bit-identical to its own kernel's (same
// device functions, same tile shapes).
template <int GPS, int NST>
__global__ void __launch_bounds__(kMixThreads, 1) lm_heads_mixed_kernel(
    const uint16_t *__restrict__ xt, int Mt, const uint16_t *__restrict__ W, float *__restrict__ yt,
    const uint16_t *__restrict__ xd, int Md, const uint8_t *__restrict__ Wq,
    const uint16_t *__restrict__ S, float *__restrict__ yd, int Kd, int N, unsigned int *work) {
    using R = Int4Ring<GPS, NST>;
    extern __shared__ uint4 smem_mix[];
    __shared__ unsigned int row_amax[8];
    __shared__ float row_unscale[8];
    // a dependent launch (the sampler) may be scheduled onto SMs as this
    // grid's CTAs retire; it waits for the whole grid before reading y
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int Gt = Kd >> 6;
    const int rowc = Gt * 8 + 1;
    uint16_t *xst = reinterpret_cast<uint16_t *>(smem_mix);                   // [Mt][Kd + 32] bf16
    uint4 *x4 = smem_mix + (size_t)Mt * (Kd + 32) / 8;                        // int4 staging
    uint16_t *xb = reinterpret_cast<uint16_t *>(x4);                          // [Md + 1][rowc * 8]
    float *xs = reinterpret_cast<float *>(x4 + (size_t)(Md + 1) * rowc);      // [Gt][8]
    unsigned char *rings = reinterpret_cast<unsigned char *>(xs + Gt * 8);    // [int4 warps][NST][stage]
    bf16_mma_stage_x(xst, xt, Mt, Kd);
    int4_f16_stage_x(xb, xs, row_amax, row_unscale, xd, Md, Kd, true);  // ends with a block barrier
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w4 = warp - (kMixWarps - kMixInt4Warps);
    if (w4 >= 0)
        int4_f16_tiles<GPS, NST>(x4, xs, row_unscale, rings + (size_t)w4 * R::kWarpBytes, Md, Kd, N,
                                 Wq, S, yd, N, blockIdx.x * kMixInt4Warps + w4,
                                 gridDim.x * kMixInt4Warps);
    const unsigned tiles = (unsigned)((N + 15) / 16);
    for (;;) {
        unsigned g = 0;
        if (lane == 0) g = atomicAdd(work, 1u);
        g = __shfl_sync(0xffffffffu, g, 0);
        if (g >= tiles) break;
        bf16_mma_tile<1, kBmmaU>(xst, Mt, Kd, N, W, yt, N, (int)g);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Shared memory of the tensor-core bf16 kernel for M (<= 16) rows.
static size_t bf16_mma_smem(int M, int Kd) { return (size_t)M * (Kd + 32) * 2; }

template <int NT>
static cudaError_t launch_bf16_mma(const uint16_t *x, int M, int Kd, int N, const uint16_t *W,
                                   float *y, int ldy, cudaStream_t s) {
    auto k = lm_head_bf16_mma_kernel<NT, kBmmaU>;
    const size_t smem = bf16_mma_smem(M, Kd);
    int occ = 0, sms = 0;
    cudaError_t e = kernel_setup((const void *)k, kBmmaThreads, smem, &occ, &sms);
    if (e != cudaSuccess) return e;
    const int ntiles = (N + 15) / 16;
    const int need = (ntiles + kBmmaThreads / 32 - 1) / (kBmmaThreads / 32);
    const int grid = std::min(need, sms * occ);
    k<<<grid, kBmmaThreads, smem, s>>>(x, M, Kd, N, W, y, ldy);
    return cudaGetLastError();
}

// Shared memory of the direct-load fp16 int4 kernel for M (<= 8) rows.
static size_t int4_direct_smem(int M, int Kd) {
    const size_t Gt = (size_t)Kd / 64;
    return (size_t)M * (Gt * 8 + 1) * 16 + Gt * 8 * sizeof(float);
}

// The fp16 ring kernel: 3-stage rings of 8 groups in 12 warps per CTA.
constexpr int kF16Gps = 8, kF16Nst = 3, kF16Threads = 384;
static size_t int4_f16_smem(int M, int Kd) {
    const size_t Gt = (size_t)Kd / 64;
    return (size_t)(M + 1) * (Gt * 8 + 1) * 16 + Gt * 8 * sizeof(float) +
           (size_t)(kF16Threads / 32) * Int4Ring<kF16Gps, kF16Nst>::kWarpBytes;
}
static bool int4_f16_ok(int M, int Kd, const void *S) {
    return M <= 8 && Kd % (64 * kF16Gps) == 0 && ((uintptr_t)S & 15) == 0 &&
           int4_f16_smem(M, Kd) <= (size_t)227 * 1024;
}

static cudaError_t launch_int4_f16(const uint16_t *x, int M, int Kd, int N, const uint8_t *Wq,
                                   const uint16_t *S, float *y, int ldy, cudaStream_t s) {
    auto k = lm_head_int4_f16_kernel<kF16Gps, kF16Nst, kF16Threads>;
    const size_t smem = int4_f16_smem(M, Kd);
    int occ = 0, sms = 0;
    cudaError_t e = kernel_setup((const void *)k, kF16Threads, smem, &occ, &sms);
    if (e != cudaSuccess) return e;
    const int nblk = (N + 15) / 16;
    const int need = (nblk + kF16Threads / 32 - 1) / (kF16Threads / 32);
    const int grid = std::min(need, sms * occ);
    k<<<grid, kF16Threads, smem, s>>>(x, M, Kd, N, Wq, S, y, ldy);
    return cudaGetLastError();
}

static cudaError_t launch_int4_direct(const uint16_t *x, int M, int Kd, int N, const uint8_t *Wq,
                                      const uint16_t *S, float *y, int ldy, cudaStream_t s) {
    constexpr int RB = 2, UI = 4;
    auto k = lm_head_int4_f16_direct_kernel<RB, UI>;
    const size_t smem = int4_direct_smem(M, Kd);
    int occ = 0, sms = 0;
    cudaError_t e = kernel_setup((const void *)k, kGemvThreads, smem, &occ, &sms);
    if (e != cudaSuccess) return e;
    const int ntask = ((N + 15) / 16 + RB - 1) / RB;
    const int need = (ntask + kGemvWarps - 1) / kGemvWarps;
    const int grid = std::min(need, sms * occ);
    k<<<grid, kGemvThreads, smem, s>>>(x, M, Kd, N, Wq, S, y, ldy);
    return cudaGetLastError();
}

static size_t heads_pair_smem(int Mt, int Md, int Kd) {
    const size_t Gt = (size_t)Kd / 64;
    return bf16_mma_smem(Mt, Kd) + (size_t)(Md + 1) * (Gt * 8 + 1) * 16 + Gt * 8 * sizeof(float) +
           (size_t)kMixInt4Warps * Int4Ring<kF16Gps, kF16Nst>::kWarpBytes;
}

bool lm_heads_pair_ok(int Mt, int Md, int Kd, const void *scales) {
    return Mt >= 1 && Mt <= 8 && Md >= 1 && Md <= 8 && Kd % (64 * kF16Gps) == 0 &&
           ((uintptr_t)scales & 15) == 0 && heads_pair_smem(Mt, Md, Kd) <= (size_t)227 * 1024 - 256;
}

cudaError_t launch_lm_heads_pair(const void *xt, int Mt, const void *w, float *yt, const void *xd,
                                 int Md, const void *wq, const void *scales, float *yd, int Kd,
                                 int N, void *work, cudaStream_t s) {
    if (!lm_heads_pair_ok(Mt, Md, Kd, scales) || !work) return cudaErrorInvalidValue;
    auto k = lm_heads_mixed_kernel<kF16Gps, kF16Nst>;
    const size_t smem = heads_pair_smem(Mt, Md, Kd);
    int occ = 0, sms = 0;
    cudaError_t e = kernel_setup((const void *)k, kMixThreads, smem, &occ, &sms);
    if (e != cudaSuccess) return e;
    unsigned int *wk = static_cast<unsigned int *>(work);
    e = cudaMemsetAsync(wk, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    k<<<sms * occ, kMixThreads, smem, s>>>(
        static_cast<const uint16_t *>(xt), Mt, static_cast<const uint16_t *>(w), yt,
        static_cast<const uint16_t *>(xd), Md, static_cast<const uint8_t *>(wq),
        static_cast<const uint16_t *>(scales), yd, Kd, N, wk);
    return cudaGetLastError();
}

size_t lm_head_max_smem_rows(int Kd) {
    // rows of 4 Kd bytes that fit in 227 KB of shared memory: the shape bound
    // of both heads (Kd <= 58112) and the int4 row grouping
    return (size_t)(227 * 1024) / ((size_t)Kd * sizeof(float));
}

// Which kernel takes an int4 head of M > 8 rows: the streamed mma.sync kernel
// (proj_wide.cu) for up to 32 rows, one pass over the weights; the
// tensor-memory kernel for 33..64 rows, where the streamed kernel would need
// two passes.  Measured on B200 at vocabulary 248320, hidden 5120: streamed
// 307 / 313 / 394 / 449 us at 9 / 16 / 24 / 32 rows, tensor memory ~487 us
// at each (its single MMA-issuing thread bounds it, not the row count).
static bool int4_head_streamed(int M, int Kd) { return M > 8 && M <= 32 && Kd % 64 == 0; }

size_t lm_head_scratch_bytes(int M, int Kd, int fmt) {
    if (fmt == MTPV_W_BF16 && M > 8 && lm_head_tc_ok(M, Kd, nullptr, nullptr)) return 256;
    if (fmt == MTPV_W_INT4_G64 && int4_head_streamed(M, Kd)) return int4_proj_workspace_bytes(M, Kd, 0, false);
    if (fmt == MTPV_W_INT4_G64 && M > 8 && lm_head_tc_int4_ok(M, Kd, nullptr, nullptr, nullptr))
        return lm_head_int4_tc_scratch_bytes(M, Kd);
    return 0;
}

cudaError_t launch_lm_head(const void *x, int M, int Kd, int N, const void *w, const void *scales,
                           int fmt, float *y, void *scratch, cudaStream_t s) {
    const uint16_t *xb = static_cast<const uint16_t *>(x);
    if (fmt == MTPV_W_BF16 && M > 8 && lm_head_tc_ok(M, Kd, x, w)) {
        // every weight read once, all rows per tile, on the tensor-memory kernel
        unsigned int *err = static_cast<unsigned int *>(scratch);
        if (!err) return cudaErrorInvalidValue;
        cudaError_t e = cudaMemsetAsync(err, 0, sizeof(unsigned int), s);
        if (e != cudaSuccess) return e;
        return launch_lm_head_bf16_tc(x, M, Kd, N, w, y, err, s);
    }
    if (fmt == MTPV_W_BF16) {
        // the tensor-core kernel: 16 rows per pass when more than 8 rows come
        // and 16 staged rows fit, else passes of up to 8 rows
        const uint16_t *W = static_cast<const uint16_t *>(w);
        const size_t fit = (size_t)227 * 1024 / bf16_mma_smem(1, Kd);
        if (fit < 1) return cudaErrorInvalidValue;
        const int step = (M > 8 && fit >= 16) ? 16 : (int)std::min<size_t>(8, fit);
        for (int m0 = 0; m0 < M; m0 += step) {
            const int mm = std::min(step, M - m0);
            const cudaError_t e =
                mm > 8 ? launch_bf16_mma<2>(xb + (size_t)m0 * Kd, mm, Kd, N, W, y + (size_t)m0 * N, N, s)
                       : launch_bf16_mma<1>(xb + (size_t)m0 * Kd, mm, Kd, N, W, y + (size_t)m0 * N, N, s);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    if (int4_head_streamed(M, Kd)) {
        // one pass, streamed mma.sync; unaligned operands take the passes
        // below instead, which need no scratch (the workspace was sized for
        // this kernel, never for the tensor-memory one)
        if (!((uintptr_t)x & 15) && !((uintptr_t)w & 15) && !((uintptr_t)scales & 15))
            return launch_int4_proj(x, M, Kd, N, w, scales, y, N, false, scratch, true, s);
    } else if (M > 8 && lm_head_tc_int4_ok(M, Kd, x, w, scales)) {  // one pass, on the tensor-memory kernel
        return launch_lm_head_int4_tc(x, M, Kd, N, w, scales, y, scratch, s);
    }
    // int4 group-64: passes of up to 8 rows, each on the ring kernel when it
    // takes the shape, else on the direct-load kernel (same bits)
    const int step = (int)std::min<size_t>(8, lm_head_max_smem_rows(Kd));
    if (step < 1) return cudaErrorInvalidValue;
    const uint8_t *Wq = static_cast<const uint8_t *>(w);
    const uint16_t *S = static_cast<const uint16_t *>(scales);
    for (int m0 = 0; m0 < M; m0 += step) {
        const int mm = std::min(step, M - m0);
        const uint16_t *xm = xb + (size_t)m0 * Kd;
        float *ym = y + (size_t)m0 * N;
        cudaError_t e;
        if (int4_f16_ok(mm, Kd, S))
            e = launch_int4_f16(xm, mm, Kd, N, Wq, S, ym, N, s);
        else if (int4_direct_smem(mm, Kd) <= (size_t)227 * 1024)
            e = launch_int4_direct(xm, mm, Kd, N, Wq, S, ym, N, s);
        else
            return cudaErrorInvalidValue;  // no int4 kernel for this shape
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mtpv
