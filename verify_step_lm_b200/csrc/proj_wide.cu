// The int4 projection for passes of 9..32 activation rows (two to four MMA
// n-tiles of 8 rows): the batched verify step's int4 draft head (24 rows at 8
// sequences x 3 drafts) and decoder projections for more than 8 rows, with
// the weights read once per pass (hazakura.dev MTPLX notes, Layer 0: the LM
// head's matmul specialised by row count; gist.science BaseRT explainer,
// methodology: dequantisation in the inner loop).
//
// Same stage stream and stream-K split as the narrow kernel (proj.cu); what
// differs is the warp layout, chosen to keep NT n-tiles of accumulators in
// 128 registers:
//   * 16 warps, no separate producer (17 warps would cap a thread at 96
//     registers: a sub-partition holding five warps has 16 K registers); the
//     last warp fills the ring ahead and refills each slot as soon as every
//     warp has released it;
//   * warp w takes two 16-row MMA tiles (rows 32 (w % 4) .. + 31; gate_up:
//     w % 4 < 2 the gate rows, else the up rows) and two of the stage's
//     groups (2 (w / 4), + 1), for every n-tile;
//   * a nibble n becomes the bf16 value n - 8 exactly (OR it into the
//     mantissa of 128.0, subtract 136 in bf16), mma.sync m16n8k16 sums a
//     group per n-tile in fp32, the group's scale multiplies it into the sum;
//   * at a tile's end the warps' sums are added in a fixed order one n-tile
//     at a time, and split tiles are finished through the tickets as in the
//     narrow kernel.
// On B200 this beats the tensor-memory int4 head at these row counts: at
// vocabulary 248320 and hidden 5120, 307 / 313 / 394 / 449 us at 9 / 16 / 24
// / 32 rows against ~487 us, because a small-N tcgen05.mma costs its issuing
// thread ~200 cycles while an mma.sync m16n8k16 costs the SM ~2.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "proj.cuh"

namespace mtpv {

namespace {

constexpr int kWideWarps = 16;
constexpr int kWideThreads = 32 * kWideWarps;
constexpr int kWideRed = kWideWarps * 8 * 32;  // floats: each warp's 8 sums per lane, one n-tile at a time

// activations of a stage: per group one box of up to 8 NT rows of 128 bytes
__host__ __device__ constexpr int wide_xbytes(int nt) { return pj::kG * nt * 1024; }
__host__ __device__ constexpr int wide_stage_bytes(int nt) { return pj::kWBytes + wide_xbytes(nt) + pj::kSBytes; }

}  // namespace

template <bool GU, int NT>
__global__ void __launch_bounds__(kWideThreads, 1)
    int4_proj_wide_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, pj::Args a) {
    constexpr int kStage = wide_stage_bytes(NT);
    constexpr int kXBytes = wide_xbytes(NT);
    extern __shared__ __align__(1024) unsigned char pj_smem[];
    unsigned char *ring = reinterpret_cast<unsigned char *>(((uintptr_t)pj_smem + 1023) & ~(uintptr_t)1023);
    float *red = reinterpret_cast<float *>(ring + (size_t)a.stages * kStage);
    pj::Ctl &c = *reinterpret_cast<pj::Ctl *>(red + kWideRed);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Gt = a.Kd >> 6;
    const long long grid = gridDim.x;
    const long long s0 = (long long)blockIdx.x * a.T / grid;
    const long long s1 = (long long)(blockIdx.x + 1) * a.T / grid;
    const uint32_t abort32 = su32(&c.abort);

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.stages; ++i) {
            bar_init(&c.full[i], 33);  // the filler's expect_tx + its 32 lanes' cp.async arrivals
            bar_init(&c.empty[i], kWideWarps);
        }
        c.abort = 0;
        c.last = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // ---------------- the ring's filling (the last warp) ----------------
    const bool filler = warp == kWideWarps - 1;
    const size_t sbytes = (size_t)a.N * Gt * 2;
    const bool two_chunks = ((2 * Gt) & 15) != 0;  // a row's 8 scales straddle 16-byte chunks
    const uint32_t tx = pj::kWBytes + pj::kG * a.M * 128;
    long long issued = 0;                          // stages issued so far (filler)
    int fX = (int)(s0 / a.spt), fch = (int)(s0 - (long long)fX * a.spt);
    bool fstop = false;
    // stage s0 + issued into its slot (whose previous use every warp has released)
    auto fill = [&]() {
        const int fslot = (int)(issued % a.stages);
        unsigned char *st = ring + (size_t)fslot * kStage;
        if (lane == 0) {
            bar_arrive_expect(&c.full[fslot], tx);
#pragma unroll
            for (int p = 0; p < 2; ++p) {  // groups 4p .. 4p+3 of the stage: 128-byte rows
                const int xc = (fch * pj::kG + 4 * p) * 32;
                if (GU) {
                    tma_load_2d(st + p * 16384, &tmW, xc, fX * 64, &c.full[fslot]);
                    tma_load_2d(st + p * 16384 + 8192, &tmW, xc, a.F + fX * 64, &c.full[fslot]);
                } else {
                    tma_load_2d(st + p * 16384, &tmW, xc, fX * pj::kTileRows, &c.full[fslot]);
                }
            }
#pragma unroll
            for (int jj = 0; jj < pj::kG; ++jj)
                tma_load_2d(st + pj::kWBytes + jj * NT * 1024, &tmX, (fch * pj::kG + jj) * 64, 0, &c.full[fslot]);
        }
        // scales of tile rows lane + 32 i: the aligned 16-byte chunk(s) holding groups 8 ch .. 8 ch + 7
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = lane + 32 * i;
            const long long row = GU ? (r < 64 ? (long long)fX * 64 + r : (long long)a.F + fX * 64 + (r - 64))
                                     : (long long)fX * pj::kTileRows + r;
            const size_t off = ((size_t)row * Gt + (size_t)fch * pj::kG) * 2;
            const size_t al = off & ~(size_t)15;
            unsigned char *dst = st + pj::kWBytes + kXBytes + r * 32;
            pj::cp_async16(dst, a.s, al, sbytes);
            if (two_chunks) pj::cp_async16(dst + 16, a.s, al + 16, sbytes);
        }
        pj::cp_async_arrive(&c.full[fslot]);
        ++issued;
        if (++fch == a.spt) {
            fch = 0;
            ++fX;
        }
    };
    if (filler)
        while (issued < a.stages && s0 + issued < s1) fill();

    // ---------------- consumers ----------------
    const int g = lane >> 2, t = lane & 3;
    const int tp = warp & 3, gp = warp >> 2;  // tiles 2 tp, 2 tp + 1 (rows 32 tp ..); groups 2 gp, 2 gp + 1
    // byte offset of group 0 of the stage inside a row's scale chunk: rows of
    // this lane are = g (mod 8) in the tile, and (F + g) for gate_up's up rows
    const int srow = (GU && tp >= 2) ? ((a.F + g) & 7) : g;
    const int soff = (((2 * Gt) & 15) * srow) & 15;
    const uint32_t ring32 = su32(ring);
    // per-lane offsets inside a stage, for each of the warp's two groups
    const int xr = pj::act_row(g);  // the activation row (within an n-tile) behind this lane's MMA column
    uint32_t wofs0[2], wofs1[2], xofs0[2], xofs1[2], sofs[2];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
        const int j = 2 * gp + jj, c0 = 2 * (j & 3);  // the group's two 16-byte chunks in its 128-byte row
        const int rowb = (j >> 2) * 16384 + (32 * tp + g) * 128;
        wofs0[jj] = (uint32_t)(rowb + ((c0 ^ g) << 4) + 4 * t);
        wofs1[jj] = (uint32_t)(rowb + (((c0 + 1) ^ g) << 4) + 4 * t);
        xofs0[jj] = (uint32_t)(pj::kWBytes + j * NT * 1024 + xr * 128 + ((t ^ xr) << 4));
        xofs1[jj] = (uint32_t)(pj::kWBytes + j * NT * 1024 + xr * 128 + (((4 + t) ^ xr) << 4));
        sofs[jj] = (uint32_t)(pj::kWBytes + kXBytes + soff + 2 * j + (32 * tp + g) * 32);
    }
    float acc[2][NT][4];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[tt][nt][e] = 0.0f;
    int slot = 0;
    uint32_t phase = 0;
    bool bad = false;
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
        if (!bad) {
            const uint32_t st = ring32 + (uint32_t)slot * kStage;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                if (ch * pj::kG + 2 * gp + jj >= Gt) continue;  // past the row's last group (warp-uniform)
                // activations: row 8 nt + act_row(g), elements 8t .. 8t+7 and 32+8t .. 32+8t+7 of
                // the group; MMA i takes, for lane (g, t), the physical k pairs
                // (8t+i, 8t+i+4) and (32+8t+i, 32+8t+i+4) as its logical (2t, 2t+1)
                // and (2t+8, 2t+9)
                uint32_t b0[NT][4], b1[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
                    if (8 * nt + xr < a.M) {
                        x0 = pj::lds128(st + xofs0[jj] + nt * 1024);
                        x1 = pj::lds128(st + xofs1[jj] + nt * 1024);
                    }
                    const uint32_t X0[4] = {x0.x, x0.y, x0.z, x0.w}, X1[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
                        b0[nt][i] = __byte_perm(X0[i >> 1], X0[2 + (i >> 1)], sel);
                        b1[nt][i] = __byte_perm(X1[i >> 1], X1[2 + (i >> 1)], sel);
                    }
                }
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {  // rows ra = 32 tp + 16 tt + g and rb = ra + 8
                    uint32_t pa0[4], pa1[4], pb0[4], pb1[4];
                    pj::nib_pairs<true>(pj::lds32(st + wofs0[jj] + tt * 2048), pa0);
                    pj::nib_pairs<true>(pj::lds32(st + wofs1[jj] + tt * 2048), pa1);
                    pj::nib_pairs<true>(pj::lds32(st + wofs0[jj] + tt * 2048 + 1024), pb0);
                    pj::nib_pairs<true>(pj::lds32(st + wofs1[jj] + tt * 2048 + 1024), pb1);
                    const float sa = pj::lds_bf16(st + sofs[jj] + tt * 512);
                    const float sc = pj::lds_bf16(st + sofs[jj] + tt * 512 + 256);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float cc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint32_t af[4] = {pa0[i], pb0[i], pa1[i], pb1[i]};
                            pj::mma_bf16(cc, af, b0[nt][i], b1[nt][i]);
                        }
                        acc[tt][nt][0] = fmaf(sa, cc[0], acc[tt][nt][0]);
                        acc[tt][nt][1] = fmaf(sa, cc[1], acc[tt][nt][1]);
                        acc[tt][nt][2] = fmaf(sc, cc[2], acc[tt][nt][2]);
                        acc[tt][nt][3] = fmaf(sc, cc[3], acc[tt][nt][3]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) bar_arrive(&c.empty[slot]);
        if (filler && !fstop && s0 + issued < s1) {
            // the slot's next stage, once every warp has released this one
            const bool ok = __all_sync(0xffffffffu, pj::bar_wait_or_abort(&c.empty[slot], phase, abort32));
            if (ok) {
                fill();
            } else {
                fstop = true;
                if (lane == 0) {
                    atomicOr(a.err, 1u);
                    *(volatile int *)&c.abort = 1;
                }
            }
        }
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
        const long long cf = pj::run_owner((long long)Xs * a.spt, a.T, grid);
        const long long cl = pj::run_owner((long long)Xs * a.spt + a.spt - 1, a.T, grid);
        const bool sole = cf == cl;  // the whole tile is this CTA's
        const int pslot = (s0 / a.spt == Xs) ? 0 : 1;  // the run's first tile, or its last
        float *pp = a.part + ((size_t)blockIdx.x * 2 + pslot) * (NT * pj::kPart);
        // thread q: entry (v, lane') of warps tp' = q / 256 (rows 32 tp' ..) and
        // tp' + 2 (rows 64 + 32 tp' ..), summed over the four group pairs
        const int q = threadIdx.x, lq = q & 31, v = (q >> 5) & 7, tq = q >> 8;
        const int rloc = 32 * tq + 16 * (v >> 2) + (lq >> 2) + 8 * ((v >> 1) & 1);  // row within a 64-row half
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int vv = 0; vv < 8; ++vv) red[(warp * 8 + vv) * 32 + lane] = acc[vv >> 2][nt][vv & 3];
            pj::named_sync<kWideThreads>();
            float val0 = 0.0f, val1 = 0.0f;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                val0 += red[((4 * gq + tq) * 8 + v) * 32 + lq];
                val1 += red[((4 * gq + tq + 2) * 8 + v) * 32 + lq];
            }
            const int m = 8 * nt + pj::act_row(2 * (lq & 3) + (v & 1));
            if (sole) {
                if (m < a.M) {
                    if (GU) {
                        const int col = Xs * 64 + rloc;
                        if (col < a.F) a.y[(size_t)m * a.ldy + col] = pj::silu(val0) * val1;
                    } else {
                        const int col = Xs * pj::kTileRows + rloc;
                        if (col < a.N) a.y[(size_t)m * a.ldy + col] = val0;
                        if (col + 64 < a.N) a.y[(size_t)m * a.ldy + col + 64] = val1;
                    }
                }
            } else {
                pp[nt * pj::kPart + q] = val0;
                pp[nt * pj::kPart + 512 + q] = val1;
            }
            pj::named_sync<kWideThreads>();  // red is read before the next n-tile's sums go there
        }
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[tt][nt][e] = 0.0f;
        if (sole) continue;
        if (q == 0) {  // the barrier made the CTA's stores this thread's; the fence publishes them
            __threadfence();
            const unsigned int old = atomicAdd(&a.tickets[cf], 1u);
            const int last = (old == (unsigned int)(cl - cf)) ? 1 : 0;
            if (last) __threadfence();
            *(volatile int *)&c.last = last;
        }
        pj::named_sync<kWideThreads>();
        if (*(volatile int *)&c.last) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int m = 8 * nt + pj::act_row(2 * (lq & 3) + (v & 1));
                if (m >= a.M) continue;
                float v0 = 0.0f, v1 = 0.0f;
                for (long long cc = cf; cc <= cl; ++cc) {  // contributors in CTA order
                    const int sl = ((cc * a.T / grid) / a.spt == Xs) ? 0 : 1;
                    const float *qp = a.part + ((size_t)cc * 2 + sl) * (NT * pj::kPart) + nt * pj::kPart;
                    v0 += __ldcg(qp + q);
                    v1 += __ldcg(qp + 512 + q);
                }
                if (GU) {
                    const int col = Xs * 64 + rloc;
                    if (col < a.F) a.y[(size_t)m * a.ldy + col] = pj::silu(v0) * v1;
                } else {
                    const int col = Xs * pj::kTileRows + rloc;
                    if (col < a.N) a.y[(size_t)m * a.ldy + col] = v0;
                    if (col + 64 < a.N) a.y[(size_t)m * a.ldy + col + 64] = v1;
                }
            }
            if (q == 0) a.tickets[cf] = 0u;  // ready for the next call
        }
    }
    if (filler) {  // the copies still in flight land before the CTA may exit
        for (int i = 0; i < a.stages; ++i) {
            const long long k = issued > i ? (issued - 1 - i) / a.stages + 1 : 0;
            if (k) bar_wait(&c.full[i], (uint32_t)((k - 1) & 1));
        }
    }
}


namespace {

int wide_stages(int nt) {
    const int n = (pj::kSmemCap - 1024 - kWideRed * 4 - (int)pj::kCtlBytes) / wide_stage_bytes(nt);
    return std::min(n, pj::kMaxStages);
}

template <bool GU, int NT>
cudaError_t launch_wide(const CUtensorMap &tmW, const CUtensorMap &tmX, pj::Args a, int psms, cudaStream_t s) {
    const int stages = wide_stages(NT);
    const size_t smem = 1024 + (size_t)stages * wide_stage_bytes(NT) + kWideRed * 4 + pj::kCtlBytes;
    int occ = 0, sms = 0;
    cudaError_t e = kernel_setup((const void *)int4_proj_wide_kernel<GU, NT>, kWideThreads, smem, &occ, &sms);
    if (e != cudaSuccess) return e;
    a.stages = stages;
    const int grid = (int)std::max(1LL, std::min<long long>(a.T, std::min(sms, psms)));
    int4_proj_wide_kernel<GU, NT><<<grid, kWideThreads, smem, s>>>(tmW, tmX, a);
    return cudaGetLastError();
}

template <bool GU>
cudaError_t launch_wide_nt(int nt, const CUtensorMap &tmW, const CUtensorMap &tmX, const pj::Args &a, int psms,
                           cudaStream_t s) {
    switch (nt) {
        case 2: return launch_wide<GU, 2>(tmW, tmX, a, psms, s);
        case 3: return launch_wide<GU, 3>(tmW, tmX, a, psms, s);
        default: return launch_wide<GU, 4>(tmW, tmX, a, psms, s);
    }
}

}  // namespace

cudaError_t pj::launch_wide_pass(const CUtensorMap &tmW, const CUtensorMap &tmX, pj::Args a, int nt, bool gate_up,
                                 int psms, cudaStream_t s) {
    return gate_up ? launch_wide_nt<true>(nt, tmW, tmX, a, psms, s) : launch_wide_nt<false>(nt, tmW, tmX, a, psms, s);
}

}  // namespace mtpv
