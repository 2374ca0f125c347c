// LM-head projections for more than 8 activation rows on the fifth-generation
// tensor cores (tcgen05): y[M, N] = x[M, Kd] . W[N, Kd]^T for 9 <= M <= 64.
//
// A batched verify step (several sequences, K + 1 rows each) projects tens of
// rows through the heads (hazakura.dev MTPLX notes, Layer 0: the LM head's
// matmul specialised by row count; the draft-only 4-bit copy of the head).
// At that row count the weight stream is still the bound, but per-lane MMAs
// would have to re-read the weights once per 8 or 16 rows; here every weight
// is read from HBM once, whatever M:
//   * a persistent grid walks 128-row tiles of the head; one thread of
//     warp 0 streams each tile's 64-column slices of W (and the matching
//     slice of x) into a ring of shared-memory stages with TMA
//     (cp.async.bulk.tensor, 128-byte swizzle, no multicast);
//   * one thread of warp 1 issues tcgen05.mma (A = the weight slice,
//     B = the activation slice, both K-major in shared memory) into an fp32
//     accumulator in tensor memory, two accumulators in turn so that a
//     tile's epilogue overlaps the next tile's MMAs;
//   * four epilogue warps read the accumulator with tcgen05.ld (warp w reads
//     TMEM lanes 32 (w % 4) .. + 31, i.e. 32 vocabulary rows) and store y.
// The int4 group-64 head runs the same pipeline with four more warps that
// dequantise each slice into the A stage (fp16, 128-byte swizzle) before the
// MMA reads it; its activations are fp16, prepared once per call.
// Every mbarrier wait is bounded: a wait that gives up sets the kernel's
// error word, stops the CTA's pipeline, waits (bounded) for its copies in
// flight and releases its tensor memory before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "lm_head_tc.cuh"
#include "tma.cuh"

namespace mtpv {

namespace {

constexpr int kTcStages = 8;                 // handled in pairs: one wait and one commit per 8 MMAs
constexpr int kTcPairs = kTcStages / 2;
constexpr int kTcRows = 128;                 // vocabulary rows per tile (the MMA's M)
constexpr int kTcK = 64;                     // reduction elements per stage: one 128-byte row
constexpr int kTcABytes = kTcRows * kTcK * 2;  // 16 KB per stage
constexpr int kTcMaxN = 64;                  // activation rows (the MMA's N), padded to 16
constexpr int kTcBBytesMax = kTcMaxN * kTcK * 2;
// Partial accumulators per tile: a stage's consecutive 16-element MMAs write
// different ones, so they need not wait for each other (at these small N a
// chain of MMAs into one accumulator runs at ~110 ns per MMA on B200); the
// epilogue adds the partials in a fixed order.
constexpr int kTcParts = 4;

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Shared-memory matrix descriptor of a K-major tile with 128-byte rows and the
// 128-byte swizzle (8-row groups 1024 bytes apart), tcgen05 format.
__device__ __forceinline__ uint64_t sw128_desc(const void *tile) {
    const uint64_t addr = su32(tile);
    return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// D[tmem] (+)= A[smem] . B[smem]^T, kind::f16 (bf16 or fp16 inputs, fp32 accumulate)
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on an mbarrier once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t *b) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(b))
                 : "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// Instruction descriptor of kind::f16: fp32 accumulator, A and B of the
// given type (0 fp16, 1 bf16), both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t tc_idesc(uint32_t ab_type, int n) {
    return (1u << 4) | (ab_type << 7) | (ab_type << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);
}

// Shared memory: the stages (1024-byte aligned for the swizzle), then the
// barriers and the tensor-memory address.
struct TcCtl {
    uint64_t full[kTcPairs];    // TMA bytes of a pair of stages landed (producer)
    uint64_t empty[kTcPairs];   // the MMAs that read a pair of stages completed
    uint64_t tfull[2];          // accumulator a holds a finished tile
    uint64_t tempty[2];         // accumulator a has been read out
    uint32_t tmem;
    int abort;                  // a wait gave up: every role stops
};

}  // namespace

// ---------------------------------------------------------------------------
// bf16 head
// ---------------------------------------------------------------------------
// Warp 0: TMA producer; warp 1: MMA issuer (and TMEM owner); warps 2..5: epilogue.
__global__ void __launch_bounds__(192, 1) lm_head_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmW,
                                                                   const __grid_constant__ CUtensorMap tmX,
                                                                   float *__restrict__ y, int M, int N, int Kd,
                                                                   int nb, unsigned int *err) {
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    unsigned char *base = reinterpret_cast<unsigned char *>(((uintptr_t)tc_smem + 1023) & ~(uintptr_t)1023);
    unsigned char *sa = base;                                   // [stages][16 KB]
    unsigned char *sb = sa + kTcStages * kTcABytes;             // [stages][nb * 128 B]
    const int bbytes = nb * kTcK * 2;
    TcCtl &c = *reinterpret_cast<TcCtl *>(sb + kTcStages * kTcBBytesMax);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = (N + kTcRows - 1) / kTcRows;
    const int nk = Kd / kTcK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcPairs; ++s) {
            bar_init(&c.full[s], 1);
            bar_init(&c.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            bar_init(&c.tfull[a], 1);
            bar_init(&c.tempty[a], 128);
        }
        c.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // two accumulators of kTcParts x nb fp32 columns each
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&c.tmem)),
                     "r"(2u * kTcParts * kTcMaxN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = c.tmem;

    if (warp == 0) {
        if (lane == 0) {
            int pr = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
                for (int kb = 0; kb < nk; kb += 2) {  // a pair of 64-column slices (the last may be alone)
                    if (!bar_wait(&c.empty[pr], phase ^ 1)) { atomicOr(err, 1u); c.abort = 1; }
                    if (*(volatile int *)&c.abort) break;
                    const int n2 = kb + 1 < nk ? 2 : 1;
                    bar_arrive_expect(&c.full[pr], (uint32_t)(n2 * (kTcABytes + bbytes)));
                    for (int u = 0; u < n2; ++u) {
                        tma_load_2d(sa + (2 * pr + u) * kTcABytes, &tmW, (kb + u) * kTcK, tile * kTcRows, &c.full[pr]);
                        tma_load_2d(sb + (2 * pr + u) * kTcBBytesMax, &tmX, (kb + u) * kTcK, 0, &c.full[pr]);
                    }
                    if (++pr == kTcPairs) { pr = 0; phase ^= 1; }
                }
                if (*(volatile int *)&c.abort) break;
            }
            // the copies still in flight land before the CTA may exit
            for (int s = 0; s < kTcPairs; ++s) bar_wait(&c.full[s], s < pr ? phase : phase ^ 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc_idesc(1u, nb);
            int pr = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t aphase = 0;
            for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
                if (!bar_wait(&c.tempty[acc], aphase ^ 1)) { atomicOr(err, 2u); c.abort = 1; }
                if (*(volatile int *)&c.abort) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * kTcParts * nb);
                for (int kb = 0; kb < nk; kb += 2) {
                    if (!bar_wait(&c.full[pr], phase)) { atomicOr(err, 4u); c.abort = 1; }
                    if (*(volatile int *)&c.abort) break;
                    tc_fence_after();
                    const int n2 = kb + 1 < nk ? 2 : 1;
                    for (int u = 0; u < n2; ++u) {
                        const uint64_t ad = sw128_desc(sa + (2 * pr + u) * kTcABytes);
                        const uint64_t bd = sw128_desc(sb + (2 * pr + u) * kTcBBytesMax);
                        // a slice's four 16-element steps go to four partial
                        // accumulators, so consecutive MMAs do not wait on each other
#pragma unroll
                        for (int k = 0; k < kTcK / 16; ++k)  // 16 elements = 32 bytes per MMA
                            tc_mma(d + (uint32_t)(k * nb), ad + 2 * k, bd + 2 * k, idesc, (kb + u) != 0);
                    }
                    tc_commit(&c.empty[pr]);
                    if (++pr == kTcPairs) { pr = 0; phase ^= 1; }
                }
                if (*(volatile int *)&c.abort) break;
                tc_commit(&c.tfull[acc]);
                if (++acc == 2) { acc = 0; aphase ^= 1; }
            }
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31
        const int q = warp & 3;
        int acc = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            bool ok = bar_wait(&c.tfull[acc], aphase);
            if (!ok) { atomicOr(err, 8u); c.abort = 1; }
            if (__any_sync(0xffffffffu, !ok) || *(volatile int *)&c.abort) break;
            tc_fence_after();
            const int v = tile * kTcRows + 32 * q + lane;
            const uint32_t t0 = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * kTcParts * nb);
            for (int c0 = 0; c0 < nb; c0 += 16) {
                float r[16];
                tc_ld16(t0 + (uint32_t)c0, r);
#pragma unroll
                for (int pp = 1; pp < kTcParts; ++pp) {  // the partial sums, added in order
                    float o[16];
                    tc_ld16(t0 + (uint32_t)(pp * nb + c0), o);
#pragma unroll
                    for (int j = 0; j < 16; ++j) r[j] += o[j];
                }
                if (v < N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < M) y[(size_t)(c0 + j) * N + v] = r[j];
                }
            }
            tc_fence_before();
            bar_arrive(&c.tempty[acc]);
            if (++acc == 2) { acc = 0; aphase ^= 1; }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(2u * kTcParts * kTcMaxN)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// int4 group-64 head
// ---------------------------------------------------------------------------
// The dequantised weights go from registers straight into tensor memory
// (tcgen05.st) and the MMA reads A from there, so a stage costs shared
// memory only its raw nibbles and the activation slice.  Weight k of a row
// is (n_k - 8) s_g; in fp16 that product is exact when s_g's 8 significant
// bits land in the normal range, which a per-row power of two f = 2^(11 - e)
// arranges (e: exponent of the row's largest |s|, so |(n - 8) s f| < 2^15;
// groups more than 2^25 below that largest scale lose low bits).  The
// activations are fp16 too, each row times a power of two that puts its
// largest |x| in [2^14, 2^15) (elements more than 2^38 below it flush to
// zero); both factors are undone on the fp32 output.  Inside each 8-weight
// chunk the reduction runs in the order (0, 4, 1, 5, 2, 6, 3, 7), for the
// weights and the staged activations alike, which is the order in which
// nibble pairs come out of a 32-bit word.
namespace {

// Three rings, each deep enough for its own latency: raw nibbles from HBM
// (16 stages of one 64-weight group, 4 KB), and, in pairs of groups,
// activation slices from L2 and dequantised A in tensor memory (4 pairs of
// 8 KB / 32 columns each).  The single thread that issues the MMAs is the
// pipeline's bottleneck (each tcgen05.mma at these sizes costs it about 125
// cycles), so it waits, fences and commits once per pair of groups.
constexpr int kT4Raw = 16;
constexpr int kT4Pairs = 4;
constexpr int kT4B = 2 * kT4Pairs;
constexpr int kT4RawBytes = kTcRows * 32;   // 128 rows x 64 nibbles
constexpr int kT4Threads = 480;             // warps: 0 TMA (nibbles, scales), 1 MMA, 2..5 epilogue,
                                            // 6..13 dequantise, 14 TMA (activations)
constexpr int kT4ACols = 32;                // TMEM columns of one stage's A (64 fp16 per lane)
constexpr uint32_t kT4TmemCols = 512;       // accumulators in columns [0, 256), the A ring in [256, 512)
constexpr uint32_t kT4ABase = 256;
constexpr int kT4MaxG = 128;                // groups per row (Kd <= 8192): two tiles of scales fit

struct T4Ctl {
    uint64_t rfull[kT4Raw];   // nibbles of a group landed
    uint64_t rfree[kT4Raw];   // the dequantisers (256) have read them
    uint64_t bfull[kT4Pairs];   // a pair's activation slices landed
    uint64_t aready[kT4Pairs];  // a pair's A is in tensor memory (256)
    uint64_t pfree[kT4Pairs];   // the MMAs that read a pair's A and activations completed
    uint64_t sfull[2];        // a tile's scales landed (buffer = tile parity)
    uint64_t sfree[2];        // dequantisers (256) and epilogue (128) are done with them
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// D[tmem] (+)= A[tmem] . B[smem]^T, kind::f16
__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}"
        ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Exponent e of the largest |s| of a row of G bf16 scales (the row's power of
// two is 2^(11 - e)); 11 for an all-zero row; clamped to [-100, 100].
__device__ __forceinline__ int row_scale_exp(const uint16_t *srow, int G) {
    uint32_t mx = 0u;
    for (int g = 0; g < G; ++g) mx = max(mx, (uint32_t)(srow[g] & 0x7FFFu));
    if (mx == 0u) return 11;
    const int e = (int)(mx >> 7) - 127;
    return max(-100, min(100, e));
}
__device__ __forceinline__ float pow2f(int k) { return __uint_as_float((uint32_t)(127 + k) << 23); }

// Ring position: slot and the parity of the slot's current fill.
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n) {
        if (++slot == n) { slot = 0; phase ^= 1; }
    }
};

}  // namespace

// Activation staging: row m of x (bf16) times 2^sh (largest |x| into
// [2^14, 2^15)), fp16, chunks of 8 stored in the order (0, 4, 1, 5, 2, 6, 3,
// 7); unscale[m] = 2^-sh.  One CTA per row.
__global__ void __launch_bounds__(256) int4_tc_stage_x_kernel(const uint16_t *__restrict__ x, int Kd,
                                                              uint4 *__restrict__ xp, float *__restrict__ unscale) {
    __shared__ uint32_t s_max;
    const int m = blockIdx.x;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + (size_t)m * Kd);
    if (threadIdx.x == 0) s_max = 0u;
    __syncthreads();
    uint32_t a = 0u;
    for (int c = threadIdx.x; c < Kd / 8; c += blockDim.x) {
        const uint4 v = xr[c];
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) a = max(a, max(w4[q] & 0x7FFFu, (w4[q] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0 && a) atomicMax(&s_max, a);
    __syncthreads();
    const int e = s_max ? max(-100, min(100, (int)(s_max >> 7) - 127)) : 0;  // bf16 exponent of max |x|
    const int sh = 14 - e;
    const float f = pow2f(sh);
    if (threadIdx.x == 0) unscale[m] = pow2f(-sh);
    uint4 *dst = xp + (size_t)m * (Kd / 8);
    for (int c = threadIdx.x; c < Kd / 8; c += blockDim.x) {
        const uint4 v = xr[c];
        const float e8[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                             bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half2 h = __floats2half2_rn(e8[j] * f, e8[j + 4] * f);
            o[j] = *reinterpret_cast<const uint32_t *>(&h);
        }
        dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Warp 0: TMA of nibbles and scales; warp 14: TMA of activation slices;
// warp 1: MMA issuer (and TMEM owner); warps 2..5: epilogue; warps 6..13:
// dequantisers (warp 6 + 4h + i handles k half h of the rows in TMEM lane
// quarter (6 + 4h + i) % 4).
__global__ void __launch_bounds__(kT4Threads, 1) lm_head_int4_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
    const __grid_constant__ CUtensorMap tmX, const float *__restrict__ unscale, float *__restrict__ y,
    int M, int N, int Kd, int nb, int parts, unsigned int *err) {
    extern __shared__ __align__(1024) unsigned char t4_smem[];
    unsigned char *base = reinterpret_cast<unsigned char *>(((uintptr_t)t4_smem + 1023) & ~(uintptr_t)1023);
    const int G = Kd / 64;
    const size_t sbytes = (size_t)kTcRows * G * 2;                  // a multiple of 16 (G % 8 == 0)
    unsigned char *sbst = base;                                     // [kT4B][8 KB] activation slices
    unsigned char *sraw = sbst + kT4B * kTcBBytesMax;               // [kT4Raw][4 KB] nibbles
    unsigned char *ssc = sraw + kT4Raw * kT4RawBytes;               // [2][128][G] bf16 scales
    T4Ctl &c = *reinterpret_cast<T4Ctl *>(ssc + 2 * sbytes);
    const int bbytes = nb * kTcK * 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = (N + kTcRows - 1) / kTcRows;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kT4Raw; ++i) {
            bar_init(&c.rfull[i], 1);
            bar_init(&c.rfree[i], 256);
        }
        for (int i = 0; i < kT4Pairs; ++i) {
            bar_init(&c.bfull[i], 1);
            bar_init(&c.aready[i], 256);
            bar_init(&c.pfree[i], 1);
        }
        for (int a = 0; a < 2; ++a) {
            bar_init(&c.sfull[a], 1);
            bar_init(&c.sfree[a], 384);
            bar_init(&c.tfull[a], 1);
            bar_init(&c.tempty[a], 128);
        }
        c.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&c.tmem)),
                     "r"(kT4TmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = c.tmem;
    auto stopped = [&]() { return *(volatile int *)&c.abort != 0; };
    auto give_up = [&](unsigned code) {
        atomicOr(err, code);
        c.abort = 1;
    };

    if (warp == 0) {
        if (lane == 0) {
            Ring rr;
            int it = 0;
            int sload[2] = {-1, -1};  // parity of the last scale load issued into each buffer
            for (int tile = blockIdx.x; tile < ntiles && !stopped(); tile += gridDim.x, ++it) {
                const int sb = it & 1;
                if (!bar_wait(&c.sfree[sb], ((it >> 1) & 1) ^ 1)) { give_up(16u); break; }
                sload[sb] = (it >> 1) & 1;
                bar_arrive_expect(&c.sfull[sb], (uint32_t)sbytes);
                tma_load_2d(ssc + sb * sbytes, &tmS, 0, tile * kTcRows, &c.sfull[sb]);
                for (int g = 0; g < G; ++g) {
                    if (!bar_wait(&c.rfree[rr.slot], rr.phase ^ 1)) { give_up(1u); break; }
                    if (stopped()) break;
                    bar_arrive_expect(&c.rfull[rr.slot], (uint32_t)kT4RawBytes);
                    tma_load_2d(sraw + rr.slot * kT4RawBytes, &tmQ, g * 32, tile * kTcRows, &c.rfull[rr.slot]);
                    rr.next(kT4Raw);
                }
            }
            // the copies still in flight land before the CTA may exit
            for (int i = 0; i < kT4Raw; ++i) bar_wait(&c.rfull[i], i < rr.slot ? rr.phase : rr.phase ^ 1);
            for (int b = 0; b < 2; ++b)
                if (sload[b] >= 0) bar_wait(&c.sfull[b], (uint32_t)sload[b]);
        }
    } else if (warp == 14) {
        if (lane == 0) {
            Ring rp;
            for (int tile = blockIdx.x; tile < ntiles && !stopped(); tile += gridDim.x) {
                for (int g = 0; g < G; g += 2) {
                    if (!bar_wait(&c.pfree[rp.slot], rp.phase ^ 1)) { give_up(128u); break; }
                    if (stopped()) break;
                    bar_arrive_expect(&c.bfull[rp.slot], (uint32_t)(2 * bbytes));
                    for (int u = 0; u < 2; ++u)
                        tma_load_2d(sbst + (2 * rp.slot + u) * kTcBBytesMax, &tmX, (g + u) * kTcK, 0, &c.bfull[rp.slot]);
                    rp.next(kT4Pairs);
                }
            }
            for (int i = 0; i < kT4Pairs; ++i) bar_wait(&c.bfull[i], i < rp.slot ? rp.phase : rp.phase ^ 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc_idesc(0u, nb);
            Ring rp;
            int acc = 0;
            uint32_t aphase = 0;
            for (int tile = blockIdx.x; tile < ntiles && !stopped(); tile += gridDim.x) {
                if (!bar_wait(&c.tempty[acc], aphase ^ 1)) { give_up(2u); break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * parts * nb);
                for (int g = 0; g < G; g += 2) {
                    if (!bar_wait(&c.aready[rp.slot], rp.phase) || !bar_wait(&c.bfull[rp.slot], rp.phase)) {
                        give_up(4u);
                        break;
                    }
                    if (stopped()) break;
                    tc_fence_after();
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint32_t a = tmem + kT4ABase + (uint32_t)((2 * rp.slot + u) * kT4ACols);
                        const uint64_t bd = sw128_desc(sbst + (2 * rp.slot + u) * kTcBBytesMax);
#pragma unroll
                        for (int k = 0; k < kTcK / 16; ++k)  // 16 fp16 = 8 TMEM columns / 32 bytes per MMA
                            tc_mma_ts(d + (uint32_t)((k % parts) * nb), a + 8u * k, bd + 2 * k, idesc,
                                      (g + u != 0 || k >= parts) ? 1u : 0u);
                    }
                    tc_commit(&c.pfree[rp.slot]);
                    rp.next(kT4Pairs);
                }
                if (stopped()) break;
                tc_commit(&c.tfull[acc]);
                if (++acc == 2) { acc = 0; aphase ^= 1; }
            }
        }
    } else if (warp < 6) {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31
        const int q = warp & 3, r = 32 * q + lane;
        int acc = 0, it = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int sb = it & 1;
            const bool ok = bar_wait(&c.tfull[acc], aphase) && bar_wait(&c.sfull[sb], (it >> 1) & 1);
            if (!ok) give_up(8u);
            if (__any_sync(0xffffffffu, !ok) || stopped()) break;
            tc_fence_after();
            const uint16_t *srow = reinterpret_cast<const uint16_t *>(ssc + sb * sbytes) + (size_t)r * G;
            const float rowmul = pow2f(row_scale_exp(srow, G) - 11);
            bar_arrive(&c.sfree[sb]);
            const int v = tile * kTcRows + r;
            const uint32_t t0 = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * parts * nb);
            for (int c0 = 0; c0 < nb; c0 += 16) {
                float o[16];
                tc_ld16(t0 + (uint32_t)c0, o);
                for (int pp = 1; pp < parts; ++pp) {  // the partial sums, added in order
                    float o2[16];
                    tc_ld16(t0 + (uint32_t)(pp * nb + c0), o2);
#pragma unroll
                    for (int j = 0; j < 16; ++j) o[j] += o2[j];
                }
                if (v < N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < M) y[(size_t)(c0 + j) * N + v] = o[j] * rowmul * __ldg(unscale + c0 + j);
                }
            }
            tc_fence_before();
            bar_arrive(&c.tempty[acc]);
            if (++acc == 2) { acc = 0; aphase ^= 1; }
        }
    } else {
        // dequantisers: row r of the tile, k half h of every 64-weight group,
        // two groups per step; the tensor-memory stores of one step complete
        // while the next step converts (its ready arrivals come after that)
        const int dw = warp - 6, h = dw >> 2, q = warp & 3, r = 32 * q + lane;
        const __half2 k1032 = __floats2half2_rn(1032.0f, 1032.0f);
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + kT4ABase + (uint32_t)(16 * h);
        Ring rr, rp;
        int it = 0;
        int pend = -1;  // A pair of the pending step, -1: none
        auto flush = [&]() {
            if (pend >= 0) {
                tc_wait_st();
                tc_fence_before();
                bar_arrive(&c.aready[pend]);
                pend = -1;
            }
        };
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int sb = it & 1;
            bool ok = bar_wait(&c.sfull[sb], (it >> 1) & 1);
            if (!ok) give_up(32u);
            if (__any_sync(0xffffffffu, !ok) || stopped()) break;
            const uint16_t *srow = reinterpret_cast<const uint16_t *>(ssc + sb * sbytes) + (size_t)r * G;
            const float f = pow2f(11 - row_scale_exp(srow, G));
            for (int g = 0; g < G; g += 2) {  // G is even; ring sizes are even, so slots pair up
                ok = bar_wait(&c.rfull[rr.slot], rr.phase) && bar_wait(&c.rfull[rr.slot + 1], rr.phase) &&
                     bar_wait(&c.pfree[rp.slot], rp.phase ^ 1);
                if (!ok) give_up(64u);
                if (__any_sync(0xffffffffu, !ok) || stopped()) break;
                uint4 raw[2];
                __half2 s2[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const float sv = __uint_as_float((uint32_t)srow[g + u] << 16) * f;
                    s2[u] = __floats2half2_rn(sv, sv);
                    raw[u] = *reinterpret_cast<const uint4 *>(sraw + (rr.slot + u) * kT4RawBytes + r * 32 + h * 16);
                }
                bar_arrive(&c.rfree[rr.slot]);
                bar_arrive(&c.rfree[rr.slot + 1]);
                uint32_t out[2][16];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t wd[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t pbits = ((wd[i] >> (4 * j)) & 0x000F000Fu) | 0x64006400u;  // 1024 + n
                            __half2 hv = *reinterpret_cast<const __half2 *>(&pbits);
                            hv = __hmul2(__hsub2(hv, k1032), s2[u]);  // (n - 8) s f, exact
                            out[u][4 * i + j] = *reinterpret_cast<const uint32_t *>(&hv);
                        }
                    }
                }
                flush();  // the previous step's stores are done: its groups are ready
                tc_fence_after();
                tc_st16(lane_base + (uint32_t)(2 * rp.slot * kT4ACols), out[0]);
                tc_st16(lane_base + (uint32_t)((2 * rp.slot + 1) * kT4ACols), out[1]);
                pend = rp.slot;
                rr.next(kT4Raw);
                rr.next(kT4Raw);
                rp.next(kT4Pairs);
            }
            flush();
            bar_arrive(&c.sfree[sb]);
            if (stopped()) break;
        }
        flush();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kT4TmemCols) : "memory");
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t encode_fn(PFN_cuTensorMapEncodeTiled_v12000 *fn) {
    std::call_once(g_encode_once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        cudaGetLastError();
    });
    *fn = g_encode;
    return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

size_t tc_smem_bytes() { return 1024 + (size_t)kTcStages * (kTcABytes + kTcBBytesMax) + sizeof(TcCtl); }

}  // namespace

cudaError_t map_2d(CUtensorMap *m, const void *ptr, CUtensorMapDataType type, int elem_bytes, int cols,
                   int rows, int box_cols, int box_rows, CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    cudaError_t e = encode_fn(&enc);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * (cuuint64_t)elem_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(m, type, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

size_t t4_smem_bytes(int Kd) {
    const size_t sbytes = (size_t)kTcRows * (Kd / 64) * 2;
    return 1024 + (size_t)kT4B * kTcBBytesMax + (size_t)kT4Raw * kT4RawBytes + 2 * sbytes + sizeof(T4Ctl);
}

bool lm_head_tc_int4_ok(int M, int Kd, const void *x, const void *wq, const void *scales) {
    return M >= 9 && M <= kTcMaxN && Kd % 512 == 0 && Kd / 64 <= kT4MaxG && ((uintptr_t)x & 15) == 0 &&
           ((uintptr_t)wq & 15) == 0 && ((uintptr_t)scales & 15) == 0 && t4_smem_bytes(Kd) <= 227 * 1024;
}

size_t lm_head_int4_tc_scratch_bytes(int M, int Kd) { return 512 + (((size_t)M * Kd * 2 + 255) & ~(size_t)255); }

cudaError_t launch_lm_head_int4_tc(const void *x, int M, int Kd, int N, const void *wq, const void *scales,
                                   float *y, void *scratch, cudaStream_t s) {
    if (!lm_head_tc_int4_ok(M, Kd, x, wq, scales) || !scratch) return cudaErrorInvalidValue;
    unsigned int *err = static_cast<unsigned int *>(scratch);
    float *unscale = reinterpret_cast<float *>(static_cast<char *>(scratch) + 256);
    uint4 *xp = reinterpret_cast<uint4 *>(static_cast<char *>(scratch) + 512);
    const int nb = (M + 15) / 16 * 16, G = Kd / 64;
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    int4_tc_stage_x_kernel<<<M, 256, 0, s>>>(static_cast<const uint16_t *>(x), Kd, xp, unscale);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap tmQ, tmS, tmX;
    e = map_2d(&tmQ, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Kd / 2, N, 32, kTcRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e == cudaSuccess)
        e = map_2d(&tmS, scales, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, G, N, G, kTcRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e == cudaSuccess)
        e = map_2d(&tmX, xp, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, Kd, M, kTcK, nb, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const size_t smem = t4_smem_bytes(Kd);
    int occ = 0, sms = 0;
    e = kernel_setup((const void *)lm_head_int4_tc_kernel, kT4Threads, smem, &occ, &sms);
    if (e != cudaSuccess) return e;
    const int ntiles = (N + kTcRows - 1) / kTcRows;
    // partial accumulators: as many as fit two buffers of them in 256 columns
    const int parts = std::min(4, 256 / (2 * nb));
    lm_head_int4_tc_kernel<<<std::min(ntiles, sms * occ), kT4Threads, smem, s>>>(tmQ, tmS, tmX, unscale, y, M, N,
                                                                                 Kd, nb, parts, err);
    return cudaGetLastError();
}

bool lm_head_tc_ok(int M, int Kd, const void *x, const void *w) {
    return M >= 9 && M <= kTcMaxN && Kd % kTcK == 0 && ((uintptr_t)x & 15) == 0 && ((uintptr_t)w & 15) == 0;
}

cudaError_t launch_lm_head_bf16_tc(const void *x, int M, int Kd, int N, const void *w, float *y,
                                   unsigned int *err, cudaStream_t s) {
    if (!lm_head_tc_ok(M, Kd, x, w) || !err) return cudaErrorInvalidValue;
    const int nb = (M + 15) / 16 * 16;
    CUtensorMap tmW, tmX;
    cudaError_t e = map_2d(&tmW, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Kd, N, kTcK, kTcRows,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = map_2d(&tmX, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Kd, M, kTcK, nb, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const size_t smem = tc_smem_bytes();
    int occ = 0, sms = 0;
    e = kernel_setup((const void *)lm_head_bf16_tc_kernel, 192, smem, &occ, &sms);
    if (e != cudaSuccess) return e;
    const int ntiles = (N + kTcRows - 1) / kTcRows;
    const int grid = std::min(ntiles, sms * occ);
    lm_head_bf16_tc_kernel<<<grid, 192, smem, s>>>(tmW, tmX, y, M, N, Kd, nb, err);
    return cudaGetLastError();
}

}  // namespace mtpv
