// mbarrier and TMA (cp.async.bulk.tensor) wrappers shared by the kernels that
// stream tiles into shared memory, and the host-side tensor-map encoder.
// Every wait is bounded: it reports failure instead of spinning forever.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace mtpv {

constexpr int kBarWaitLimit = 1 << 20;  // polls of one mbarrier wait before it gives up

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
// if it gave up after kBarWaitLimit polls.
__device__ __forceinline__ bool bar_wait(uint64_t *b, uint32_t parity) {
    for (int i = 0; i < kBarWaitLimit; ++i) {
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
// One box of a 2-D tensor map into shared memory; the bytes complete a
// transaction count on the mbarrier.  x is the innermost coordinate.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *b) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(su32(dst)), "l"(map), "r"(x), "r"(y), "r"(su32(b))
        : "memory");
}

// 2-D tensor map of a row-major [rows, cols] matrix (elem_bytes per element),
// box of box_cols x box_rows, zero fill out of bounds.
cudaError_t map_2d(CUtensorMap *m, const void *ptr, CUtensorMapDataType type, int elem_bytes, int cols, int rows,
                   int box_cols, int box_rows, CUtensorMapSwizzle swizzle);

}  // namespace mtpv
