// Int4 group-64 projections for a handful of activation rows:
//   y[M, N] = x[M, Kd] . deq(Wq, S)^T,   deq = s_g (n - 8)
//   gate_up: h[M, F] = silu(x . G^T) * (x . U^T), G and U the two halves
// (hazakura.dev MTPLX notes, Layer 0: the verify pass's matmuls run with a
// handful of rows; gist.science BaseRT explainer, methodology: per-format
// GEMV with dequantisation in the inner loop, fused op chains).  This file
// holds the kernel for passes of up to 8 rows and the launch that splits M
// into passes: up to 8 rows here, 9..32 rows per pass on the wide kernel
// (proj_wide.cu), which keeps more n-tiles in registers.
//
// The nibbles (14-95 MB per decoder matrix) are the whole cost, so the
// kernel streams them through shared memory at HBM rate:
//   * the work is a list of stages, one stage = a tile of 128 weight rows
//     (128 output columns; gate_up: 64 gate rows and the matching 64 up rows)
//     times 8 groups of 64 weights; the tile-major list is cut into one equal
//     run per CTA, so every SM streams the same number of bytes whatever N
//     and Kd are (a stream-K split of the reduction);
//   * one producer warp per CTA moves each stage into a ring in shared
//     memory: nibbles and activations by TMA (128-byte swizzle, no
//     multicast), scales by cp.async, all completing on the stage's mbarrier;
//   * sixteen consumer warps: warp w takes group w % 8 of every stage and
//     four of the eight 16-row MMA tiles (gate_up: warps 0-7 the gate rows,
//     8-15 the up rows); a nibble n becomes the bf16 value 128 + n exactly
//     (OR it into the mantissa of 128.0), the activations are used as given
//     (bf16), mma.sync m16n8k16 sums (128 + n_k) x_k over a group in fp32
//     and adding the group's -136 sum_k x_k (computed once per group by MMAs
//     whose A is -136 everywhere) leaves sum_k (n_k - 8) x_k; the group's
//     scale multiplies it into the warp's running sum;
//   * at the end of a tile (or of its run) the CTA adds its warps' sums in a
//     fixed order; a CTA that covered the whole tile writes y (gate_up:
//     silu(g) u), otherwise it stores its partial tile and takes a ticket,
//     and the CTA that draws the last ticket adds the partials in CTA order
//     (fixed for a given SM count, so results are deterministic), writes y
//     and resets the ticket.
// Every mbarrier wait is bounded; a wait that gives up ORs a code into the
// workspace's error word, the CTA stops computing (it still takes its
// tickets, so the counters stay consistent) and the producer waits, bounded,
// for its copies in flight before the CTA exits.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "lm_head.cuh"
#include "proj.cuh"

namespace mtpv {

namespace {

constexpr int kNarrowCW = 16;                      // consumer warps
constexpr int kNarrowThreads = 32 * (kNarrowCW + 1);  // + the producer warp (the last one)
constexpr int kNarrowXBox = 1024;                  // one group of up to 8 activation rows
constexpr int kNarrowXBytes = pj::kG * kNarrowXBox;
constexpr int kNarrowStage = pj::kWBytes + kNarrowXBytes + pj::kSBytes;
constexpr int kNarrowRed = kNarrowCW * 16 * 32;    // floats: each warp's 16 sums per lane
constexpr int kNarrowRows = 8;                     // activation rows per pass
constexpr int kWideRows = 8 * pj::kMaxNT;          // rows per pass of the wide kernel

}  // namespace

template <bool GU>
__global__ void __launch_bounds__(kNarrowThreads, 1)
    int4_proj_narrow_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, pj::Args a) {
    extern __shared__ __align__(1024) unsigned char pj_smem[];
    unsigned char *ring = reinterpret_cast<unsigned char *>(((uintptr_t)pj_smem + 1023) & ~(uintptr_t)1023);
    float *red = reinterpret_cast<float *>(ring + (size_t)a.stages * kNarrowStage);
    pj::Ctl &c = *reinterpret_cast<pj::Ctl *>(red + kNarrowRed);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Gt = a.Kd >> 6;
    const long long grid = gridDim.x;
    const long long s0 = (long long)blockIdx.x * a.T / grid;
    const long long s1 = (long long)(blockIdx.x + 1) * a.T / grid;
    // a dependent launch may be scheduled onto SMs as this grid's CTAs leave
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.stages; ++i) {
            bar_init(&c.full[i], 33);  // the producer's expect_tx + its 32 lanes' cp.async arrivals
            bar_init(&c.empty[i], kNarrowCW);
        }
        c.abort = 0;
        c.last = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == kNarrowCW) {
        // ---------------- producer ----------------
        const size_t sbytes = (size_t)a.N * Gt * 2;
        const bool two_chunks = ((2 * Gt) & 15) != 0;  // a row's 8 scales straddle 16-byte chunks
        const uint32_t tx = pj::kWBytes + pj::kG * a.M * 128;
        const uint32_t abort32 = su32(&c.abort);
        // stage s into ring slot `slot`: its weights (nibbles by TMA, scales by
        // cp.async into a 32-byte slot per row: the aligned 16-byte chunk(s)
        // holding groups 8 ch .. 8 ch + 7), and its activations (TMA)
        auto issue_weights = [&](long long s, int slot) {
            const int X = (int)(s / a.spt), ch = (int)(s - (long long)X * a.spt);
            unsigned char *st = ring + (size_t)slot * kNarrowStage;
            if (lane == 0) {
                bar_arrive_expect(&c.full[slot], tx);
#pragma unroll
                for (int p = 0; p < 2; ++p) {  // groups 4p .. 4p+3 of the stage: 128-byte rows
                    const int xc = (ch * pj::kG + 4 * p) * 32;
                    if (GU) {
                        tma_load_2d(st + p * 16384, &tmW, xc, X * 64, &c.full[slot]);
                        tma_load_2d(st + p * 16384 + 8192, &tmW, xc, a.F + X * 64, &c.full[slot]);
                    } else {
                        tma_load_2d(st + p * 16384, &tmW, xc, X * pj::kTileRows, &c.full[slot]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane + 32 * i;
                const long long row = GU ? (r < 64 ? (long long)X * 64 + r : (long long)a.F + X * 64 + (r - 64))
                                         : (long long)X * pj::kTileRows + r;
                const size_t off = ((size_t)row * Gt + (size_t)ch * pj::kG) * 2;
                const size_t al = off & ~(size_t)15;
                unsigned char *dst = st + pj::kWBytes + kNarrowXBytes + r * 32;
                pj::cp_async16(dst, a.s, al, sbytes);
                if (two_chunks) pj::cp_async16(dst + 16, a.s, al + 16, sbytes);
            }
            pj::cp_async_arrive(&c.full[slot]);
        };
        auto issue_acts = [&](long long s, int slot) {
            if (lane == 0) {
                const int ch = (int)(s % a.spt);
                unsigned char *st = ring + (size_t)slot * kNarrowStage;
#pragma unroll
                for (int jj = 0; jj < pj::kG; ++jj)
                    tma_load_2d(st + pj::kWBytes + jj * kNarrowXBox, &tmX, (ch * pj::kG + jj) * 64, 0, &c.full[slot]);
            }
        };
        // The ring's first stages: weights and scales before waiting for the
        // grid before this one on the stream (nothing on the stream writes
        // them), the activations once that grid has completed.
        const long long fill = std::min<long long>(a.stages, s1 - s0);
        for (long long k = 0; k < fill; ++k) issue_weights(s0 + k, (int)k);
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (long long k = 0; k < fill; ++k) issue_acts(s0 + k, (int)k);
        long long issued = fill;
        int slot = (int)(fill % a.stages);
        uint32_t phase = fill == a.stages ? 1u : 0u;
        for (long long s = s0 + fill; s < s1; ++s) {
            const bool ok = __all_sync(0xffffffffu, pj::bar_wait_or_abort(&c.empty[slot], phase ^ 1, abort32));
            if (!ok) {
                if (lane == 0) {
                    atomicOr(a.err, 1u);
                    *(volatile int *)&c.abort = 1;
                }
                break;
            }
            issue_weights(s, slot);
            issue_acts(s, slot);
            ++issued;
            if (++slot == a.stages) {
                slot = 0;
                phase ^= 1;
            }
        }
        // the copies still in flight land before the CTA may exit
        for (int i = 0; i < a.stages; ++i) {
            const long long k = issued > i ? (issued - 1 - i) / a.stages + 1 : 0;
            if (k) bar_wait(&c.full[i], (uint32_t)((k - 1) & 1));
        }
        return;
    }

    // ---------------- consumers ----------------
    // (the workspace and y are touched only after the grid before this one
    // on the stream has completed)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int g = lane >> 2, t = lane & 3;
    const int j = warp & 7, hb = warp >> 3;  // group of the stage; MMA tiles 4 hb .. 4 hb + 3
    const int xr = pj::act_row(g);  // the activation row behind this lane's MMA column
    const bool has_row = xr < a.M;
    // byte offset of group 0 of the stage inside a row's scale chunk: rows of
    // this lane are = g (mod 8) in the tile, and (F + g) for gate_up's up rows
    const int srow = (GU && hb) ? ((a.F + g) & 7) : g;
    const int soff = (((2 * Gt) & 15) * srow) & 15;
    const int c0 = 2 * (j & 3);  // the group's two 16-byte chunks in its 128-byte row
    // per-lane offsets inside a stage: nibble words of rows 16 (4 hb) + g (+ 8 + 16 tt),
    // activation chunks of row g, scales of the same rows
    const uint32_t ring32 = su32(ring);
    const uint32_t wofs0 = (uint32_t)((j >> 2) * 16384 + (16 * 4 * hb + g) * 128 + ((c0 ^ g) << 4) + 4 * t);
    const uint32_t wofs1 = (uint32_t)((j >> 2) * 16384 + (16 * 4 * hb + g) * 128 + (((c0 + 1) ^ g) << 4) + 4 * t);
    const uint32_t xofs0 = (uint32_t)(pj::kWBytes + j * kNarrowXBox + xr * 128 + ((t ^ xr) << 4));
    const uint32_t xofs1 = (uint32_t)(pj::kWBytes + j * kNarrowXBox + xr * 128 + (((4 + t) ^ xr) << 4));
    const uint32_t sofs = (uint32_t)(pj::kWBytes + kNarrowXBytes + soff + 2 * j + (16 * 4 * hb + g) * 32);
    float acc[4][4];
#pragma unroll
    for (int tt = 0; tt < 4; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[tt][e] = 0.0f;
    int slot = 0;
    uint32_t phase = 0;
    bool bad = false;
    const uint32_t abort32 = su32(&c.abort);
    int X = (int)(s0 / a.spt), ch = (int)(s0 - (long long)X * a.spt);
    for (long long s = s0; s < s1; ++s) {
        if (!bad) {
            const bool ok = __all_sync(0xffffffffu, pj::bar_wait_or_abort(&c.full[slot], phase, abort32));
            if (!ok) {
                bad = true;
                if (lane == 0) {
                    atomicOr(a.err, 2u);
                    *(volatile int *)&c.abort = 1;
                }
            }
        }
        if (!bad && ch * pj::kG + j < Gt) {
            const uint32_t st = ring32 + (uint32_t)slot * kNarrowStage;
            // activations of row act_row(g): elements 8t .. 8t+7 and 32+8t .. 32+8t+7 of the group
            uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
            if (has_row) {
                x0 = pj::lds128(st + xofs0);
                x1 = pj::lds128(st + xofs1);
            }
            // MMA i takes, for lane (g, t), the physical k pairs (8t+i, 8t+i+4)
            // and (32+8t+i, 32+8t+i+4) as its logical (2t, 2t+1) and (2t+8, 2t+9)
            const uint32_t X0[4] = {x0.x, x0.y, x0.z, x0.w}, X1[4] = {x1.x, x1.y, x1.z, x1.w};
            uint32_t b0[4], b1[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
                b0[i] = __byte_perm(X0[i >> 1], X0[2 + (i >> 1)], sel);
                b1[i] = __byte_perm(X1[i >> 1], X1[2 + (i >> 1)], sel);
            }
            // the group's offset term -136 sum_k x[m][k], the same for every
            // weight row: an MMA with A = -136 everywhere (exact in bf16)
            float off[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            {
                const uint32_t am[4] = {0xC308C308u, 0xC308C308u, 0xC308C308u, 0xC308C308u};
#pragma unroll
                for (int i = 0; i < 4; ++i) pj::mma_bf16(off, am, b0[i], b1[i]);
            }
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {  // rows ra = 16 (4 hb + tt) + g and rb = ra + 8
                uint32_t pa0[4], pa1[4], pb0[4], pb1[4];
                pj::nib_pairs<false>(pj::lds32(st + wofs0 + tt * 2048), pa0);
                pj::nib_pairs<false>(pj::lds32(st + wofs1 + tt * 2048), pa1);
                pj::nib_pairs<false>(pj::lds32(st + wofs0 + tt * 2048 + 1024), pb0);
                pj::nib_pairs<false>(pj::lds32(st + wofs1 + tt * 2048 + 1024), pb1);
                const float sa = pj::lds_bf16(st + sofs + tt * 512), sc = pj::lds_bf16(st + sofs + tt * 512 + 256);
                // sum_k (128 + n_k) x_k, then + (-136 sum_k x_k) = sum_k (n_k - 8) x_k
                float cc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t af[4] = {pa0[i], pb0[i], pa1[i], pb1[i]};
                    pj::mma_bf16(cc, af, b0[i], b1[i]);
                }
                acc[tt][0] = fmaf(sa, cc[0] + off[0], acc[tt][0]);
                acc[tt][1] = fmaf(sa, cc[1] + off[1], acc[tt][1]);
                acc[tt][2] = fmaf(sc, cc[2] + off[2], acc[tt][2]);
                acc[tt][3] = fmaf(sc, cc[3] + off[3], acc[tt][3]);
            }
        }
        __syncwarp();
        if (lane == 0) bar_arrive(&c.empty[slot]);
        if (++slot == a.stages) {
            slot = 0;
            phase ^= 1;
        }
        const int Xs = X;  // the tile of this stage
        if (++ch == a.spt) {
            ch = 0;
            ++X;
        } else if (s + 1 != s1) {
            continue;
        }

        // ---- end of this CTA's part of tile Xs ----
#pragma unroll
        for (int v = 0; v < 16; ++v) {
            red[(warp * 16 + v) * 32 + lane] = acc[v >> 2][v & 3];
            acc[v >> 2][v & 3] = 0.0f;
        }
        pj::named_sync<kNarrowCW * 32>();
        // thread q: entry (v, lane') of both row halves b = 0, 1 (warps 8b .. 8b+7)
        const int q = threadIdx.x, v = q >> 5, lq = q & 31;
        const int m = pj::act_row(2 * (lq & 3) + (v & 1));
        const int rloc = 16 * (v >> 2) + (lq >> 2) + 8 * ((v >> 1) & 1);  // row within a 64-row half
        float val[2];
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            float sum = 0.0f;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) sum += red[((b * 8 + jj) * 16 + v) * 32 + lq];
            val[b] = sum;
        }
        const long long cf = pj::run_owner((long long)Xs * a.spt, a.T, grid);
        const long long cl = pj::run_owner((long long)Xs * a.spt + a.spt - 1, a.T, grid);
        if (cf == cl) {  // the whole tile is this CTA's
            if (m < a.M) {
                if (GU) {
                    const int col = Xs * 64 + rloc;
                    if (col < a.F) a.y[(size_t)m * a.ldy + col] = pj::silu(val[0]) * val[1];
                } else {
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const int col = Xs * pj::kTileRows + 64 * b + rloc;
                        if (col < a.N) a.y[(size_t)m * a.ldy + col] = val[b];
                    }
                }
            }
            pj::named_sync<kNarrowCW * 32>();  // red is read before the next tile's sums go there
            continue;
        }
        const int pslot = (s0 / a.spt == Xs) ? 0 : 1;  // the run's first tile, or its last
        float *pp = a.part + ((size_t)blockIdx.x * 2 + pslot) * pj::kPart;
        if (m < a.M) {
            pp[q] = val[0];
            pp[512 + q] = val[1];
        }
        pj::named_sync<kNarrowCW * 32>();
        if (q == 0) {  // the barrier made the CTA's stores this thread's; the fence publishes them
            __threadfence();
            const unsigned int old = atomicAdd(&a.tickets[cf], 1u);
            const int last = (old == (unsigned int)(cl - cf)) ? 1 : 0;
            if (last) __threadfence();
            *(volatile int *)&c.last = last;
        }
        pj::named_sync<kNarrowCW * 32>();
        if (*(volatile int *)&c.last) {
            if (m < a.M) {
                float v0 = 0.0f, v1 = 0.0f;
                for (long long cc = cf; cc <= cl; ++cc) {  // contributors in CTA order
                    const int sl = ((cc * a.T / grid) / a.spt == Xs) ? 0 : 1;
                    const float *qp = a.part + ((size_t)cc * 2 + sl) * pj::kPart;
                    v0 += __ldcg(qp + q);
                    v1 += __ldcg(qp + 512 + q);
                }
                if (GU) {
                    const int col = Xs * 64 + rloc;
                    if (col < a.F) a.y[(size_t)m * a.ldy + col] = pj::silu(v0) * v1;
                } else {
                    const int col0 = Xs * pj::kTileRows + rloc;
                    if (col0 < a.N) a.y[(size_t)m * a.ldy + col0] = v0;
                    if (col0 + 64 < a.N) a.y[(size_t)m * a.ldy + col0 + 64] = v1;
                }
            }
            if (q == 0) a.tickets[cf] = 0u;  // ready for the next call
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

int narrow_stages() {
    const int n = (pj::kSmemCap - 1024 - kNarrowRed * 4 - (int)pj::kCtlBytes) / kNarrowStage;
    return std::min(n, pj::kMaxStages);
}
size_t narrow_smem(int stages) { return 1024 + (size_t)stages * kNarrowStage + kNarrowRed * 4 + pj::kCtlBytes; }

// n-tiles the widest pass of M rows needs (the narrow kernel's partials are one n-tile)
int passes_nt(int M) { return M <= kNarrowRows ? 1 : std::min(pj::kMaxNT, (std::min(M, kWideRows) + 7) / 8); }

int plan_sms() {
    const int n = current_device_sms();
    return n > 0 ? n : 148;
}

}  // namespace

size_t int4_proj_workspace_bytes(int M, int Kd, int N, bool gate_up) {
    (void)Kd;
    (void)N;
    (void)gate_up;
    return pj::layout(passes_nt(M), plan_sms()).total;
}

cudaError_t launch_int4_proj(const void *x, int M, int Kd, int N, const void *wq, const void *scales,
                             float *y, int ldy, bool silu_mul, void *ws, bool reset_tickets, cudaStream_t s) {
    if (((uintptr_t)x & 15) || ((uintptr_t)wq & 15) || ((uintptr_t)scales & 15) || Kd % 64 || M < 1)
        return cudaErrorInvalidValue;
    const int psms = plan_sms();  // the workspace holds tickets and partial tiles for this many CTAs
    const int spt = (Kd / 64 + pj::kG - 1) / pj::kG;
    const pj::Ws l = pj::layout(passes_nt(M), psms);
    char *w = static_cast<char *>(ws);
    pj::Args a;
    a.s = static_cast<const uint16_t *>(scales);
    a.part = reinterpret_cast<float *>(w + l.part);
    a.tickets = reinterpret_cast<unsigned int *>(w + l.tickets);
    a.err = reinterpret_cast<unsigned int *>(w);
    a.T = (long long)pj::tiles(N, silu_mul) * spt;
    a.Kd = Kd;
    a.N = N;
    a.F = silu_mul ? N / 2 : N;
    a.ldy = ldy;
    a.spt = spt;
    a.stages = 0;
    cudaError_t e;
    if (reset_tickets) {
        e = cudaMemsetAsync(w, 0, l.part, s);  // error word and tickets
        if (e != cudaSuccess) return e;
    }
    CUtensorMap tmW;
    e = map_2d(&tmW, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Kd / 2, N, 128, silu_mul ? 64 : pj::kTileRows,
               CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const int rows = M <= kNarrowRows ? kNarrowRows : kWideRows;
    for (int m0 = 0; m0 < M; m0 += rows) {
        const int mp = std::min(rows, M - m0);
        CUtensorMap tmX;
        e = map_2d(&tmX, static_cast<const uint16_t *>(x) + (size_t)m0 * Kd, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   Kd, mp, 64, mp, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
        a.M = mp;
        a.y = y + (size_t)m0 * ldy;
        if (mp > kNarrowRows) {
            e = pj::launch_wide_pass(tmW, tmX, a, (mp + 7) / 8, silu_mul, psms, s);
        } else {
            const int stages = narrow_stages();
            const size_t smem = narrow_smem(stages);
            const void *kernel = silu_mul ? (const void *)int4_proj_narrow_kernel<true>
                                          : (const void *)int4_proj_narrow_kernel<false>;
            int occ = 0, sms = 0;
            e = kernel_setup(kernel, kNarrowThreads, smem, &occ, &sms);
            if (e != cudaSuccess) return e;
            a.stages = stages;
            const int grid = (int)std::max(1LL, std::min<long long>(a.T, std::min(sms, psms)));
            // a programmatic dependent of the grid before it on the stream:
            // its CTAs start streaming weights as that grid's CTAs leave
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(grid, 1, 1);
            cfg.blockDim = dim3(kNarrowThreads, 1, 1);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = s;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            at[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            e = silu_mul ? cudaLaunchKernelEx(&cfg, int4_proj_narrow_kernel<true>, tmW, tmX, a)
                         : cudaLaunchKernelEx(&cfg, int4_proj_narrow_kernel<false>, tmW, tmX, a);
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mtpv
