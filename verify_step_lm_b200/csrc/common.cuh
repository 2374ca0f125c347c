// Internal helpers shared by the libmtpv CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mtpv.h"

namespace mtpv {

// Launch setup of `kernel` on the current device: opts it into `smem` bytes of
// dynamic shared memory and returns how many of its CTAs of `threads` threads
// fit on one SM, and (sms) the device's SM count (148 on a B200), which sizes
// the persistent grids.  Cached per (kernel, device, threads, smem): once a
// first call has run, later launches of the same shape make no CUDA API call
// here, which also keeps them capturable into a CUDA graph.
cudaError_t kernel_setup(const void *kernel, int threads, size_t smem, int *ctas_per_sm, int *sms);

// SM count of the current device (cached per device); 0 if it cannot be read.
int current_device_sms();

// ---------------------------------------------------------------------------
// global loads
// ---------------------------------------------------------------------------
// Streamed, read-once weights: non-coherent path, no L1 allocation, ask L2 to
// fetch the surrounding 256-byte block.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// L2-coherent load (skips L1), for values written by other SMs in this launch.
__device__ __forceinline__ float ld_cg_f32(const float *p) { return __ldcg(p); }

// ---------------------------------------------------------------------------
// bf16 lanes of a 32-bit word (element 2i in the low half) widened to fp32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ---------------------------------------------------------------------------
// warp reductions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace mtpv
