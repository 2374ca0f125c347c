// Internal pieces shared by the two int4 projection kernels (proj.cu: passes
// of up to 8 activation rows; proj_wide.cu: passes of 9..32 rows): the stage
// geometry, shared-memory and copy helpers, the nibble extraction, the
// stream-K bookkeeping and the workspace layout.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "tma.cuh"

namespace mtpv {
namespace pj {

constexpr int kTileRows = 128;                // weight rows per tile
constexpr int kG = 8;                         // 64-weight groups per stage
constexpr int kWBytes = kTileRows * kG * 32;  // nibbles of a stage: 2 boxes of 128-byte rows
constexpr int kSBytes = kTileRows * 32;       // scales: two 16-byte chunks per row
constexpr int kMaxStages = 8;
constexpr int kPart = 1024;                   // floats of one n-tile of a partial tile
constexpr int kSmemCap = 227 * 1024;
constexpr int kMaxNT = 4;                     // MMA n-tiles (8 activation rows each) per pass, at most

struct Ctl {
    uint64_t full[kMaxStages];   // a stage's nibbles, activations and scales landed
    uint64_t empty[kMaxStages];  // the computing warps are done with a stage
    int abort;                   // a wait gave up: no more copies, no more compute
    int last;                    // this CTA drew the tile's last ticket
};
constexpr size_t kCtlBytes = (sizeof(Ctl) + 15) / 16 * 16;

struct Args {
    const uint16_t *s;       // scales [N, Kd/64] bf16
    float *y;                // [M, ldy]
    float *part;             // [grid][2][NT][kPart] partial tiles
    unsigned int *tickets;   // [grid], zero between calls
    unsigned int *err;
    long long T;             // stages in all (tiles x stages per tile)
    int M, Kd, N, F, ldy;    // M: rows of this pass; F: output columns (N, or N/2 for gate_up)
    int spt;                 // stages per tile
    int stages;              // ring depth
};

// shared-memory loads at 32-bit shared addresses
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float lds_bf16(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
    return __uint_as_float(v << 16);
}

// 16 bytes at base + off into shared memory, zero-filled past total bytes
// (nothing is read there).
__device__ __forceinline__ void cp_async16(void *dst, const void *base, size_t off, size_t total) {
    const uint32_t n = off >= total ? 0u : (uint32_t)min((size_t)16, total - off);
    const char *src = static_cast<const char *>(base) + (n ? off : 0);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(su32(dst)), "l"(src), "r"(n) : "memory");
}
// Arrive on the mbarrier once this thread's cp.async copies so far have landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t *b) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(su32(b)) : "memory");
}
// Waits for the barrier phase like bar_wait, but gives up early once the
// CTA's abort word (a 32-bit shared address) is set; the word is read only
// while the phase is still pending.
__device__ __forceinline__ bool bar_wait_or_abort(uint64_t *b, uint32_t parity, uint32_t abort_addr) {
    for (int i = 0; i < kBarWaitLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(su32(b)), "r"(parity)
            : "memory");
        if (done) return true;
        uint32_t ab;
        asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(ab) : "r"(abort_addr) : "memory");
        if (ab) return false;
    }
    return false;
}
// Named barrier 1 over the first `threads` threads of the CTA.
template <int threads>
__device__ __forceinline__ void named_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(threads) : "memory");
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The eight nibbles of a word as bf16 pairs (v_i, v_{i+4}), i = 0..3, with
// each nibble n in the low mantissa bits of 128.0 (explicit shr + lop3: on
// sm_100 faster than the compiler's code for the same C expression);
// Minus8 then subtracts 136 in bf16, which leaves n - 8 exactly.
template <bool Minus8>
__device__ __forceinline__ uint32_t nib_pair(uint32_t v) {
    uint32_t r;
    asm("lop3.b32 %0, %1, 0x000F000F, 0x43004300, 0xEA;" : "=r"(r) : "r"(v));  // (v & m) | c
    if (Minus8) asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(0x43084308u));
    return r;
}
template <bool Minus8>
__device__ __forceinline__ void nib_pairs(uint32_t w, uint32_t (&p)[4]) {
    uint32_t s4, s8, s12;
    asm("shr.b32 %0, %1, 4;" : "=r"(s4) : "r"(w));
    asm("shr.b32 %0, %1, 8;" : "=r"(s8) : "r"(w));
    asm("shr.b32 %0, %1, 12;" : "=r"(s12) : "r"(w));
    p[0] = nib_pair<Minus8>(w);
    p[1] = nib_pair<Minus8>(s4);
    p[2] = nib_pair<Minus8>(s8);
    p[3] = nib_pair<Minus8>(s12);
}

__device__ __forceinline__ float silu(float v) { return v / (1.0f + __expf(-v)); }

// The activation row behind MMA column c of an n-tile: (c >> 1) | ((c & 1) << 2),
// i.e. columns 0..7 take rows 0, 4, 1, 5, 2, 6, 3, 7.  Lanes g and g + 1 of a
// quarter-warp then read rows whose 128-byte-swizzle keys differ in bit 2, so
// their 16-byte activation chunks fall in disjoint bank groups (with row = c
// both rows' chunks collided, a 2-way conflict on every fragment load).
__host__ __device__ __forceinline__ int act_row(int c) { return (c >> 1) | ((c & 1) << 2); }

// The CTA whose run holds stage a (runs: [c T / grid, (c + 1) T / grid)).
__device__ __forceinline__ long long run_owner(long long a, long long T, long long grid) {
    return ((a + 1) * grid + T - 1) / T - 1;
}

inline int tiles(int N, bool gate_up) { return gate_up ? (N / 2 + 63) / 64 : (N + kTileRows - 1) / kTileRows; }

// Workspace: the error word, one ticket counter per SM (a CTA is the first
// contributor of at most one split tile, so tickets are indexed by that CTA),
// then two partial tiles of nt n-tiles per SM.
struct Ws {
    size_t tickets, part, total;
};
inline Ws layout(int nt, int sms) {
    Ws l;
    l.tickets = 256;
    l.part = l.tickets + ((size_t)sms * sizeof(unsigned int) + 255) / 256 * 256;
    l.total = l.part + (size_t)sms * 2 * nt * kPart * sizeof(float);
    return l;
}

// One pass of 9..32 rows on the wide kernel (proj_wide.cu).
cudaError_t launch_wide_pass(const CUtensorMap &tmW, const CUtensorMap &tmX, Args a, int nt, bool gate_up, int psms,
                             cudaStream_t s);

}  // namespace pj
}  // namespace mtpv
