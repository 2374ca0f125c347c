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

namespace mtpv {

namespace {

constexpr int kTcStages = 6;
constexpr int kTcRows = 128;                 // vocabulary rows per tile (the MMA's M)
constexpr int kTcK = 64;                     // reduction elements per stage: one 128-byte row
constexpr int kTcABytes = kTcRows * kTcK * 2;  // 16 KB per stage
constexpr int kTcMaxN = 64;                  // activation rows (the MMA's N), padded to 16
constexpr int kTcBBytesMax = kTcMaxN * kTcK * 2;
constexpr int kTcWaitLimit = 1 << 20;        // polls of one mbarrier wait before it gives up

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t su32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void bar_init(uint64_t *b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive_expect(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
// Waits until the barrier's phase with the given parity has completed; false
// if it gave up after kTcWaitLimit polls.
__device__ __forceinline__ bool bar_wait(uint64_t *b, uint32_t parity) {
    for (int i = 0; i < kTcWaitLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(su32(b)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *b) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(su32(dst)), "l"(map), "r"(x), "r"(y), "r"(su32(b))
        : "memory");
}
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
    uint64_t full[kTcStages];   // TMA bytes of stage s landed (producer)
    uint64_t ready[kTcStages];  // int4: stage s dequantised (128 threads)
    uint64_t empty[kTcStages];  // the MMAs that read stage s completed
    uint64_t sfull;             // int4: the tile's scales landed
    uint64_t sfree;             // int4: the dequantisers are done with the tile's scales
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
        for (int s = 0; s < kTcStages; ++s) {
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
    if (warp == 1) {  // two accumulators of nb fp32 columns each
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&c.tmem)),
                     "r"(2u * kTcMaxN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = c.tmem;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
                for (int kb = 0; kb < nk; ++kb) {
                    if (!bar_wait(&c.empty[stage], phase ^ 1)) { atomicOr(err, 1u); c.abort = 1; }
                    if (*(volatile int *)&c.abort) break;
                    bar_arrive_expect(&c.full[stage], (uint32_t)(kTcABytes + bbytes));
                    tma_load_2d(sa + stage * kTcABytes, &tmW, kb * kTcK, tile * kTcRows, &c.full[stage]);
                    tma_load_2d(sb + stage * kTcBBytesMax, &tmX, kb * kTcK, 0, &c.full[stage]);
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
                if (*(volatile int *)&c.abort) break;
            }
            // the copies still in flight land before the CTA may exit
            for (int s = 0; s < kTcStages; ++s) {
                // stage s was last filled in the phase before `phase` if s >= stage
                const uint32_t ph = s < stage ? phase : phase ^ 1;
                bar_wait(&c.full[s], ph);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc_idesc(1u, nb);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t aphase = 0;
            for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
                if (!bar_wait(&c.tempty[acc], aphase ^ 1)) { atomicOr(err, 2u); c.abort = 1; }
                if (*(volatile int *)&c.abort) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * kTcMaxN);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!bar_wait(&c.full[stage], phase)) { atomicOr(err, 4u); c.abort = 1; }
                    if (*(volatile int *)&c.abort) break;
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(sa + stage * kTcABytes);
                    const uint64_t bd = sw128_desc(sb + stage * kTcBBytesMax);
#pragma unroll
                    for (int k = 0; k < kTcK / 16; ++k)  // 16 elements = 32 bytes per MMA
                        tc_mma(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
                    tc_commit(&c.empty[stage]);
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
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
            const uint32_t t0 = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * kTcMaxN);
            for (int c0 = 0; c0 < nb; c0 += 16) {
                float r[16];
                tc_ld16(t0 + (uint32_t)c0, r);
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2u * kTcMaxN)
                     : "memory");
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

// 2-D tensor map of a row-major [rows, cols] matrix of 2-byte elements, box
// of 64 columns x box_rows rows, 128-byte swizzle, zero fill out of bounds.
cudaError_t map_2d(CUtensorMap *m, const void *ptr, CUtensorMapDataType type, int cols, int rows,
                   int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    cudaError_t e = encode_fn(&enc);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTcK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(m, type, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

size_t tc_smem_bytes() { return 1024 + (size_t)kTcStages * (kTcABytes + kTcBBytesMax) + sizeof(TcCtl); }

}  // namespace

bool lm_head_tc_ok(int M, int Kd, const void *x, const void *w) {
    return M >= 9 && M <= kTcMaxN && Kd % kTcK == 0 && ((uintptr_t)x & 15) == 0 && ((uintptr_t)w & 15) == 0;
}

cudaError_t launch_lm_head_bf16_tc(const void *x, int M, int Kd, int N, const void *w, float *y,
                                   unsigned int *err, cudaStream_t s) {
    if (!lm_head_tc_ok(M, Kd, x, w) || !err) return cudaErrorInvalidValue;
    const int nb = (M + 15) / 16 * 16;
    CUtensorMap tmW, tmX;
    cudaError_t e = map_2d(&tmW, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Kd, N, kTcRows);
    if (e == cudaSuccess) e = map_2d(&tmX, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Kd, M, nb);
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
