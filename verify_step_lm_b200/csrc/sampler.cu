// Leviathan-Chen verification and per-row sampling over the vocabulary.
//
// What is computed (devtrends.cc MTPLX overview, "no second model" section:
// exact rejection sampling of Leviathan and Chen with residual correction,
// temperature 0.6 / top_p 0.95 kept exact; hazakura.dev MTPLX notes, Layer 2:
// ratio acceptance -> residual correction -> bonus token):
//   every row l:  p_j = exp((l_j - m)/T)/Z, m = max l; top-p keeps the ranks
//                 (logit desc, index asc) whose preceding mass is < top_p;
//                 p'_j = p_j / kept mass.  T == 0: one-hot at the argmax.
//   sequence:     accept d_i while u_acc[i] < p'_i(d_i)/q'_i(d_i); at the
//                 first rejection n draw from normalise(max(0, p'_n - q'_n))
//                 (p'_n if that is all zero), else the bonus from p'_K; the
//                 draw is the inverse CDF in vocabulary order.
//
// Design for sm_100a: two kernels, each a grid of thread-block clusters of C
// CTAs (16, or 8 when a 16-CTA cluster cannot be resident); every cross-CTA
// step goes through distributed shared memory and hardware cluster barriers:
// a CTA writes its share into a slot of every CTA of the cluster before the
// barrier and reads the slots locally after it (no global flags).  Slices
// move between global and shared memory by bulk copies where aligned; their
// mbarrier waits are the only polling loops, each with a bound.  Both kernels
// are programmatic dependents of the work before them on the stream.
// Statistics kernel, one cluster per logits row; each CTA owns a contiguous
// slice of the vocabulary and keeps it in shared memory:
//   P1  the slice is read once (one bulk copy when aligned, else coalesced
//       loads); max / min / argmax / finiteness
//   P2  e_j = exp((l_j - m)/T) in fp64 for every token: Z and a 2048-bin mass
//       histogram on (m - l_j) over the row's own range
//   P3  the bin where the descending cumulative mass reaches top_p * Z; its
//       tokens are gathered into CTA 0, sorted on a (logit desc, index asc)
//       64-bit key and scanned for the exact cut token.  A crossing bin with
//       more than kCandCap tokens (massive ties, degenerate ranges) falls back
//       to an 8-pass weighted radix select on the same key.
//   out the row's statistics, and (workspace permitting) the row's weights
//       e_j of kept tokens, 0 elsewhere: p'_j = e_j / Z' with no further test.
//       When the located bin holds the cut, the other CTAs store the weights
//       masked by bin while CTA 0 computes the cut; CTA 0 then zeroes its
//       candidates past the cut.
// Draw kernel, one cluster per draft position i of a sequence (sampling: per
// row).  The acceptance test of d_i reads two weights; the cluster then draws
// position i's residual token (the bonus at i == K) with u_samp[i], as if the
// first rejection were at i, by a cluster-wide inverse CDF over the weights:
// every load is independent of the others, nothing is recomputed.  The last
// cluster of a sequence to finish (a global ticket counter; nobody waits)
// reads the K+1 position records, finds n and writes the outputs.  Drawing
// every position in parallel gives the same tokens as drawing only at n,
// since each draw uses its own uniform.
// The draw's partial sums are formed in one fixed nested order (CTA slice ->
// warp -> thread's contiguous sub-chunk -> token, every level a sequential
// chain), so the total, the prefix that picks the CTA, the warp, the thread
// and the token agree bit for bit.  All probability arithmetic is fp64 on the
// fp32 logits.
#include <cooperative_groups.h>
#include <float.h>
#include <limits.h>
#include <math.h>

#include <atomic>
#include <type_traits>
#include <mutex>

#include "common.cuh"
#include "sampler.cuh"

namespace cg = cooperative_groups;

namespace mtpv {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kCandCap = 4096;
constexpr int kCacheFloats = 9728;  // logits slice kept in shared memory (38 KB), and its exps
constexpr int kBatch = 8;           // loads in flight per thread in streaming loops
constexpr int kExpTab = 64;         // entries of the exp table (2^(j/64))
constexpr int kMaxCluster = 16;     // CTAs per cluster at most (a power of two; see cluster_size_for)

// Dynamic shared memory of the statistics kernel: a region reused phase by
// phase, then the small bookkeeping struct.
//   region: [logits slice: kCacheFloats fp32][their exps: kCacheFloats fp64]
//           (or, for a longer slice, its logits alone: kCacheFloatsLogits fp32)
//           [hist_mass: kBins fp64][cand: kCandCap u64]
//           [cand_e: kCandCap fp64]
// kCacheFloatsLogits holds a slice of vocabulary 248320 over 8 CTAs.
constexpr int kCacheFloatsLogits = 31232;
constexpr size_t kOffExp = kCacheFloats * sizeof(float);
constexpr size_t kOffHistMass = (kOffExp + kCacheFloats * sizeof(double)) > kCacheFloatsLogits * sizeof(float)
                                    ? (kOffExp + kCacheFloats * sizeof(double))
                                    : kCacheFloatsLogits * sizeof(float);
constexpr size_t kOffCand = kOffHistMass + kBins * sizeof(double);
constexpr size_t kOffCandE = kOffCand + kCandCap * sizeof(unsigned long long);
constexpr size_t kRegionBytes = kOffCandE + kCandCap * sizeof(double);
static_assert(kOffExp % 16 == 0 && kOffHistMass % 16 == 0, "region alignment");
static_assert(kOffHistMass % 16 == 0, "region alignment");
constexpr int kDrawBufDoubles = 19456;  // the draw kernel's weight buffer (152 KB: two rows' slices)
constexpr size_t kDrawBufBytes = kDrawBufDoubles * sizeof(double);

struct SamplerSmem {
    double own_mass[256];  // radix select: mass per digit
    int own_cnt[256];
    double rad_mass[256];
    int rad_cnt[256];
    double red_d[kWarps];
    float red_f[kWarps];
    float red_f2[kWarps];
    int red_i[kWarps];
    int red_i2[kWarps];
    double warp_tot[kWarps];
    double thr_excl[kThreads];
    // written by every CTA of the cluster into every CTA (slot = the writer's
    // rank) before a cluster barrier, read locally after it
    float all_max[kMaxCluster], all_min[kMaxCluster];
    int all_arg[kMaxCluster], all_bad[kMaxCluster];
    double all_Z[kMaxCluster], all_rt[kMaxCluster], all_part[kMaxCluster], all_M[kMaxCluster];
    double my_partial;
    // broadcast into every CTA of the cluster
    int bc_bin;
    double bc_A;  // radix select: the mass above the selected digit
    unsigned int cand_count;
    unsigned int local_n, local_base;
    // derived by every CTA for itself
    double draw_total, cut_Zk;
    int wstar, x_found, first_fail, cut_idx;
    int cut_pos, cut_n;  // statistics kernel, CTA 0: the cut's place among the sorted candidates, their number
    float cut_l;
    int res_acc;  // draw kernel, CTA 0: the position's acceptance
    unsigned long long bar;  // mbarrier of the bulk copies
    int wait_ok;             // thread 0's outcome of a bulk-copy wait, for the block
    double exp_tab[kExpTab];  // 2^(j/64), for exp_neg
};

constexpr size_t kStatsSmemBytes = kRegionBytes + sizeof(SamplerSmem);
constexpr size_t kDrawSmemBytes = kDrawBufBytes + sizeof(SamplerSmem);

struct Region {
    float *cache;
    double *ecache;
    double *hist_mass;
    unsigned long long *cand;
    double *cand_e;
};

// ---------------------------------------------------------------------------
// helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned int ordered_bits(float l) {
    unsigned int b = __float_as_uint(__fadd_rn(l, 0.0f));  // -0 -> +0: equal values tie
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float from_ordered_bits(unsigned int k) {
    unsigned int b = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(b);
}
// Descending key order == (logit desc, index asc).
__device__ __forceinline__ unsigned long long rank_key(float l, int j) {
    return ((unsigned long long)ordered_bits(l) << 32) |
           (unsigned long long)(0xffffffffu - (unsigned)j);
}
__device__ __forceinline__ float key_logit(unsigned long long k) {
    return from_ordered_bits((unsigned)(k >> 32));
}
__device__ __forceinline__ int key_index(unsigned long long k) {
    return (int)(0xffffffffu - (unsigned)(k & 0xffffffffu));
}

// exp(x) in fp64 for x <= 0, table-driven (P. T. P. Tang, "Table-driven
// implementation of the exponential function in IEEE floating-point
// arithmetic", ACM TOMS 15, 1989): x = (64 k' + j) ln2/64 + r with
// |r| <= ln2/128, exp(x) = 2^k' * 2^(j/64) * exp(r).  k = 64 k' + j is
// rint(64 x / ln 2); r = x - k ln2/64 with ln2/64 split into a 36-bit head
// (k times it is exact, |k| < 2^17) and the double nearest the rest;
// exp(r) - 1 from its Taylor series to degree 5 (truncation below 4e-17
// relative at |r| = ln2/128); tab[j] = 2^(j/64), built with exp2 by
// build_exp_table.  2^k' is assembled in the exponent field (two steps below
// 2^-1022).  Arguments below -745.2 give 0.
__device__ __forceinline__ void build_exp_table(double *tab) {
    if (threadIdx.x < kExpTab) tab[threadIdx.x] = exp2((double)threadIdx.x / kExpTab);
}

__device__ __forceinline__ double exp_neg(double x, const double *tab) {
    if (!(x > -745.2)) return 0.0;
    const double kInv = 0x1.71547652b82fep+6;  // 64 / ln 2
    const double kL1 = 0x1.62e42fefa0000p-7;   // ln 2 / 64, its first 36 bits
    const double kL2 = 0x1.cf79abc9e3b3ap-46;  // ln 2 / 64 - kL1
    const double kRound = 6755399441055744.0;  // 1.5 * 2^52: adding it rounds to an integer
    const double t = __fma_rn(x, kInv, kRound);
    const double kd = __dsub_rn(t, kRound);
    const int k = (int)__double2loint(t);
    double r = __fma_rn(-kd, kL1, x);
    r = __fma_rn(-kd, kL2, r);
    double q = 0.008333333333333333;    // 1/5!
    q = __fma_rn(q, r, 0.041666666666666664);  // 1/4!
    q = __fma_rn(q, r, 0.16666666666666666);   // 1/3!
    q = __fma_rn(q, r, 0.5);
    q = __fma_rn(q, r, 1.0);
    const double tj = tab[k & (kExpTab - 1)];
    const double v = __fma_rn(tj, __dmul_rn(q, r), tj);  // 2^(j/64) exp(r)
    const int e = k >> 6;                                 // floor(k / 64)
    if (e >= -1022) return v * __hiloint2double((e + 1023) << 20, 0);
    return (v * __hiloint2double((e + 1023 + 54) << 20, 0)) * 0x1p-54;
}

// e_j = exp((l_j - m) / T), with 1/T precomputed.
__device__ __forceinline__ double e_of(float l, double m, double invT, const double *tab) {
    return exp_neg(__dmul_rn(__dsub_rn((double)l, m), invT), tab);
}

// Small integers through the fp32 adder instead of the conversion unit (which
// runs at a fraction of the adder's rate): 2^23 + y rounded to an integer
// holds that integer in its low mantissa bits, exactly while 0 <= y < 2^22.
// floor_small(y) == (int)y and rint_small(y) == __float2uint_rn(y) there;
// small_float(b) == (float)b for 0 <= b < 2^22.
__device__ __forceinline__ int floor_small(float y) {
    return (int)(__float_as_uint(__fadd_rd(y, 8388608.0f)) - 0x4b000000u);
}
__device__ __forceinline__ unsigned rint_small(float y) {
    return __float_as_uint(__fadd_rn(y, 8388608.0f)) - 0x4b000000u;
}
__device__ __forceinline__ float small_float(int b) {
    return __fsub_rn(__uint_as_float(0x4b000000u + (unsigned)b), 8388608.0f);
}

// Level-1 bin of a logit: linear in (m - l) over the row's range; monotone
// (non-increasing) in l, equal logits share a bin.  (m - l) inv_w lies in
// [0, kBins (1 + 2^-22)] for every logit of a finite row.
__device__ __forceinline__ int bin_of(float l, float m, float inv_w) {
    return min(kBins - 1, max(0, floor_small(__fmul_rn(__fsub_rn(m, l), inv_w))));
}

__device__ __forceinline__ bool is_kept(const RowStats &st, float l, int j) {
    return (l > st.lstar) || (l == st.lstar && j <= st.idxstar);
}

// p'_j of one row given its statistics (logits read from global memory).
__device__ __forceinline__ double warped_prob(const RowStats &st, const float *L, int j, double T,
                                              double invT, const double *tab) {
    if (T == 0.0) return j == st.argmax ? 1.0 : 0.0;
    const float l = L[j];
    if (!is_kept(st, l, j)) return 0.0;
    return e_of(l, (double)st.m, invT, tab) / st.Zk;
}

// Fixed-tree block sum (deterministic for a given launch shape).
__device__ double block_sum_d(double v, SamplerSmem &s) {
    v = warp_sum_d(v);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) s.red_d[w] = v;
    __syncthreads();
    if (w == 0) {
        double r = lane < kWarps ? s.red_d[lane] : 0.0;
        r = warp_sum_d(r);
        if (lane == 0) s.red_d[0] = r;
    }
    __syncthreads();
    double r = s.red_d[0];
    __syncthreads();
    return r;
}

// block_sum_d of two values at once (each summed exactly as block_sum_d would).
__device__ void block_sum_d2(double &a, double &b, SamplerSmem &s) {
    a = warp_sum_d(a);
    b = warp_sum_d(b);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) {
        s.red_d[w] = a;
        s.warp_tot[w] = b;
    }
    __syncthreads();
    if (w == 0) {
        double ra = lane < kWarps ? s.red_d[lane] : 0.0;
        double rb = lane < kWarps ? s.warp_tot[lane] : 0.0;
        ra = warp_sum_d(ra);
        rb = warp_sum_d(rb);
        if (lane == 0) {
            s.red_d[0] = ra;
            s.warp_tot[0] = rb;
        }
    }
    __syncthreads();
    a = s.red_d[0];
    b = s.warp_tot[0];
    __syncthreads();
}

// Programmatic dependent launch: wait until the grids this one depends on
// have completed and their writes are visible; let dependents be scheduled.
__device__ __forceinline__ void wait_for_producer() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Bulk copies between global and shared memory (the copy engine moves a whole
// contiguous run; both addresses 16-byte aligned, the size a multiple of 16).
// Completion of loads is tracked by an mbarrier with a byte count; every wait
// is bounded (kWaitLimit polls) and reports whether the copy landed.
constexpr int kWaitLimit = 1 << 20;
__device__ __forceinline__ unsigned smem_u32(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(unsigned long long *bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect(unsigned long long *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_load(void *dst, const void *src, unsigned bytes, unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ bool mbar_wait(unsigned long long *bar, unsigned phase, int limit) {
    for (int i = 0; i < limit; ++i) {
        unsigned done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(phase)
            : "memory");
        if (done) return true;
    }
    return false;
}
// The block's wait for a bulk copy: thread 0 polls (bounded by limit; when
// that gives up, a second bound of kWaitLimit for the copy in flight) and the
// block learns the outcome at the barrier, which also orders every thread's
// reads of the copied data after thread 0 saw the copy complete.  One poller
// instead of 512 keeps the polling off the barrier the copy completes on.
__device__ __forceinline__ bool mbar_wait_block(unsigned long long *bar, unsigned phase, int limit, int *flag) {
    if (threadIdx.x == 0) {
        const bool ok = mbar_wait(bar, phase, limit);
        if (!ok) mbar_wait(bar, phase, kWaitLimit);
        *flag = ok ? 1 : 0;
    }
    __syncthreads();
    return *(volatile int *)flag != 0;
}
__device__ __forceinline__ bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }
// Warp-wide (max with its lowest index, min, or) of per-lane partials; every
// lane ends with the result.
__device__ __forceinline__ void warp_max_min_arg(float &mx, int &arg, float &mn, int &bad) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float om = __shfl_xor_sync(0xffffffffu, mx, o);
        const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
        if (om > mx || (om == mx && oa < arg)) { mx = om; arg = oa; }
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        bad |= __shfl_xor_sync(0xffffffffu, bad, o);
    }
}

// Block-wide scan of one double per thread: Kogge-Stone inside each warp, the
// warp totals chained in order by one thread, so that every thread's
// exclusive value (*excl) is bit for bit the previous thread's inclusive one
// (the return value).  Uses warp_tot and red_d; ends with a barrier.
__device__ double block_scan_d(double v, SamplerSmem &s, double *excl) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    double x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double u = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x = __dadd_rn(u, x);
    }
    const double prev = __shfl_up_sync(0xffffffffu, x, 1);
    if (lane == 31) s.warp_tot[w] = x;
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0;
        for (int i = 0; i < kWarps; ++i) {
            s.red_d[i] = a;
            a = __dadd_rn(a, s.warp_tot[i]);
        }
    }
    __syncthreads();
    const double off = s.red_d[w];
    *excl = lane > 0 ? __dadd_rn(off, prev) : off;
    const double incl = __dadd_rn(off, x);
    __syncthreads();
    return incl;
}

// Sum of vals[0..C) (one per CTA of the cluster, already in this CTA's shared
// memory), accumulated in rank order by every lane of the calling warp (a
// broadcast shuffle chain).  *excl gets the sum of the ranks before `want`.
__device__ __forceinline__ double ordered_sum(const double *vals, int C, int want, double *excl) {
    const int lane = threadIdx.x & 31;
    const double v = lane < C ? vals[lane] : 0.0;
    double acc = 0.0, ex = 0.0;
    for (int r = 0; r < C; ++r) {
        const double vr = __shfl_sync(0xffffffffu, v, r);
        if (r == want) ex = acc;
        acc = __dadd_rn(acc, vr);
    }
    if (excl) *excl = ex;
    return acc;
}

// The two halves of a cluster barrier (every thread of every CTA arrives once).
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Write v into slot `rank` of arr in every CTA of the cluster: lanes 0..C-1
// of the calling warp each store to one CTA (v uniform over the warp).
template <typename T>
__device__ __forceinline__ void publish(cg::cluster_group &cl, T *arr, int rank, int C, T v) {
    const int lane = threadIdx.x & 31;
    if (lane < C) *cl.map_shared_rank(arr + rank, lane) = v;
}

// Warp-cooperative ordered prefix over a[0..n) (n a multiple of 32): lane l
// sums a[l*q .. (l+1)*q) sequentially and the lane sums are chained in lane
// order.  Returns the total.  With search, finds the first index i whose
// inclusive prefix p_i satisfies base + p_i >= thr and returns it in *first
// (-1 if none) with *before = base + (prefix before i).  Totals and searches
// use the same additions, so a search started from a range's own base always
// ends inside the range when base + total >= thr.
__device__ double warp_prefix_search(const double *a, int n, double base, double thr, bool search,
                                     int *first, double *before) {
    const int lane = threadIdx.x & 31;
    const int q = n / 32;
    const double *my = a + lane * q;
    double lt = 0.0;
    for (int j = 0; j < q; ++j) lt = __dadd_rn(lt, my[j]);
    double acc = 0.0, start = 0.0;
    for (int r = 0; r < 32; ++r) {
        const double v = __shfl_sync(0xffffffffu, lt, r);
        if (r == lane) start = acc;
        acc = __dadd_rn(acc, v);
    }
    if (search) {
        int f = -1;
        double bef = 0.0, loc = 0.0;
        for (int j = 0; j < q; ++j) {
            const double nl = __dadd_rn(loc, my[j]);
            if (__dadd_rn(base, __dadd_rn(start, nl)) >= thr) {
                f = lane * q + j;
                bef = __dadd_rn(base, __dadd_rn(start, loc));
                break;
            }
            loc = nl;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, f >= 0);
        if (hit) {
            const int L = __ffs(hit) - 1;
            *first = __shfl_sync(0xffffffffu, f, L);
            *before = __shfl_sync(0xffffffffu, bef, L);
        } else {
            *first = -1;
            *before = __dadd_rn(base, acc);
        }
    }
    return acc;
}

// Verify rows are ordered per sequence as K+1 target rows then K draft rows;
// sample rows are the logits rows themselves.
__device__ __forceinline__ const float *row_ptr(const SamplerParams &p, int row) {
    if (!p.verify) return p.tl + (size_t)row * p.V;
    const int S = 2 * p.K + 1;
    const int b = row / S, i = row - b * S;
    if (i <= p.K) return p.tl + ((size_t)b * (p.K + 1) + i) * p.V;
    return p.dl + ((size_t)b * p.K + (i - p.K - 1)) * p.V;
}

// What a draw sums over, in units of 1/Z'_t (the inverse CDF does not depend
// on a common scale): kind 0 -> e_t[kept_t]  (= Z'_t p'_t);
// kind 1 -> max(0, e_t[kept_t] - rho e_d[kept_d]) with rho = Z'_t / Z'_d
// (= Z'_t max(0, p'_t - q'_d)).  With the statistics kernel's weights (Et,
// Ed: e of kept tokens, 0 elsewhere) a weight is two independent loads;
// without them (null) it is recomputed from the logits and the statistics.
struct DrawSrc {
    RowStats st_t, st_d;
    const float *Lt, *Ld;
    const double *Et, *Ed;
    const double *tab;  // exp table
    double rho;
    int kind;
};

__device__ __forceinline__ double draw_combine(const DrawSrc &d, double wt, double wd) {
    if (d.kind == 0) return wt;
    const double w = __dsub_rn(wt, __dmul_rn(d.rho, wd));
    return w > 0.0 ? w : 0.0;
}

__device__ __forceinline__ double draw_weight(const DrawSrc &d, int j, double invT) {
    if (d.Et) return draw_combine(d, d.Et[j], d.kind == 1 ? d.Ed[j] : 0.0);
    const float lt = d.Lt[j];
    const double wt = is_kept(d.st_t, lt, j) ? e_of(lt, (double)d.st_t.m, invT, d.tab) : 0.0;
    if (d.kind == 0) return wt;
    const float ld = d.Ld[j];
    const double wd = is_kept(d.st_d, ld, j) ? e_of(ld, (double)d.st_d.m, invT, d.tab) : 0.0;
    return draw_combine(d, wt, wd);
}

// draw_weight for the kBatch tokens j0, j0 + kThreads, ...: every load of the
// batch is issued before the arithmetic (tokens at or past v1 get 0).
__device__ __forceinline__ void draw_weights_batch(const DrawSrc &d, int v1, int j0, double invT,
                                                   double (&w)[kBatch]) {
    if (d.Et) {
        double et[kBatch], ed[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int j = j0 + q * kThreads;
            et[q] = j < v1 ? d.Et[j] : 0.0;
            ed[q] = (d.kind == 1 && j < v1) ? d.Ed[j] : 0.0;
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) w[q] = draw_combine(d, et[q], ed[q]);
        return;
    }
    float lt[kBatch], ld[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
        const int j = j0 + q * kThreads;
        lt[q] = j < v1 ? __ldg(d.Lt + j) : -INFINITY;
        ld[q] = (d.kind == 1 && j < v1) ? __ldg(d.Ld + j) : -INFINITY;
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
        const int j = j0 + q * kThreads;
        const double wt = (j < v1 && is_kept(d.st_t, lt[q], j)) ? e_of(lt[q], (double)d.st_t.m, invT, d.tab) : 0.0;
        const double wd = (d.kind == 1 && j < v1 && is_kept(d.st_d, ld[q], j))
                              ? e_of(ld[q], (double)d.st_d.m, invT, d.tab) : 0.0;
        w[q] = draw_combine(d, wt, wd);
    }
}

// ---------------------------------------------------------------------------
// Cluster-wide inverse-CDF draw over the row: x = min{k : C_k > u * total}.
// Every CTA of the cluster calls it; the CTA holding the crossing writes
// *x_out and returns kDrawWrote, the others kDrawNone; when a CTA of the
// cluster gave up waiting for a copy, every CTA returns kDrawTimeout and
// nobody writes.  With allow_fallback, a residual whose total is exactly
// zero (p' == q') is replaced by p'_t.
// Summation: each thread sums its contiguous sub-chunk sequentially (tau);
// the lanes' sums are scanned inside the warp (a fixed shuffle tree), the
// warps' totals chained in warp order, the CTAs' in rank order.  A token's
// cumulative value is Pc + (Om_w + (lp_t + loc_j)); the search picks the
// first warp, then lane, then token whose value passes the target, with the
// very sums used for the totals, so it always lands on a token of the
// crossing CTA (with a positive weight, or on its last positive one when the
// target falls in a rounding gap between two lanes).
// ---------------------------------------------------------------------------
constexpr int kDrawNone = 0;     // this CTA did not write the token
constexpr int kDrawWrote = 1;    // this CTA found the token and wrote it
constexpr int kDrawTimeout = 2;  // a CTA of the cluster gave up waiting for a copy (nobody wrote)

__device__ int cluster_draw(cg::cluster_group &cluster, SamplerSmem &s, double *wbuf, DrawSrc src,
                             bool allow_fallback, double invT, float u, int v0, int v1, int *x_out,
                             int wait_polls) {
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int n = v1 - v0;
    const int ch = (n + kThreads - 1) / kThreads;
    const int t0 = min(v1, v0 + tid * ch), t1 = min(v1, t0 + ch);
    // With the statistics kernel's weights, aligned, and room for both rows:
    // the copy engine brings the slices of e_t (and e_d) into shared memory
    // in vocabulary order; residual weights are combined where they are read
    // (e_t stays intact for the fallback to p'_n).
    const bool bulk = src.Et && n > 0 && (n & 1) == 0 && 2 * n <= kDrawBufDoubles &&
                      aligned16(src.Et + v0) && (src.kind == 0 || aligned16(src.Ed + v0));
    const double *bt = wbuf, *bd = wbuf + n;
    bool landed = true;
    if (bulk) {
        if (tid == 0) {
            mbar_init(&s.bar);
            const unsigned bytes = (unsigned)n * 8u;
            mbar_expect(&s.bar, src.kind == 1 ? 2u * bytes : bytes);
            bulk_load(wbuf, src.Et + v0, bytes, &s.bar);
            if (src.kind == 1) bulk_load(wbuf + n, src.Ed + v0, bytes, &s.bar);
        }
        landed = mbar_wait_block(&s.bar, 0, wait_polls, &s.wait_ok);
    }
    // Otherwise weights are computed once, coalesced, into shared memory;
    // thread t's sub-chunk lives at wbuf[t * P ..] with an odd stride P (no
    // bank conflicts).
    const int P = ch | 1;
    const bool buffered = !bulk && ch > 0 && (size_t)kThreads * P <= (size_t)kDrawBufDoubles;
    const double *mine = wbuf + (size_t)tid * P;
    auto wat = [&](int j) -> double {
        if (bulk) return src.kind == 1 ? draw_combine(src, bt[j - v0], bd[j - v0]) : bt[j - v0];
        return buffered ? mine[j - t0] : draw_weight(src, j, invT);
    };

    for (int attempt = 0; attempt < 2; ++attempt) {
        if (buffered) {
            __syncthreads();  // earlier users of the region are done
            for (int i0 = tid; i0 < n; i0 += kBatch * kThreads) {
                double wv[kBatch];
                draw_weights_batch(src, v1, v0 + i0, invT, wv);
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const int i = i0 + q * kThreads;
                    if (i < n) {
                        const int t = i / ch;
                        wbuf[(size_t)t * P + (i - t * ch)] = wv[q];
                    }
                }
            }
            __syncthreads();
        }
        double tau = 0.0;
        for (int j = t0; j < t1; ++j) tau = __dadd_rn(tau, wat(j));
        // inclusive scan of the lanes' sums (fixed shuffle tree); lp = the
        // lane's exclusive prefix, wtot = the warp's total
        double incl = tau;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl = __dadd_rn(incl, v);
        }
        double lp = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) lp = 0.0;
        if (lane == 31) s.warp_tot[w] = incl;
        __syncthreads();
        if (w == 0) {
            double a = 0.0;
            for (int i = 0; i < kWarps; ++i) a = __dadd_rn(a, s.warp_tot[i]);
            if (lane == 0) s.my_partial = a;
            publish(cluster, s.all_part, rank, C, a);
            publish(cluster, s.all_bad, rank, C, landed ? 0 : 1);
        }
        cluster.sync();
        double Pc = 0.0;
        const double total = ordered_sum(s.all_part, C, rank, &Pc);  // every warp, same order
        bool timed_out = false;
        for (int r = 0; r < C; ++r) timed_out |= s.all_bad[r] != 0;
        if (total == 0.0 && allow_fallback && src.kind == 1 && !timed_out) {
            src.kind = 0;  // p' == q' exactly: draw from p'_n
            cluster.sync();  // every CTA has read all_part before the next attempt rewrites it
            continue;
        }
        const double target = __dmul_rn((double)u, total);
        const double next = __dadd_rn(Pc, s.my_partial);
        if (timed_out) return kDrawTimeout;
        if (!(Pc <= target && target < next)) return kDrawNone;  // the crossing is in another CTA
        if (tid == 0) {
            double a = 0.0, om = 0.0;
            int ws = kWarps - 1;
            for (int i = 0; i < kWarps; ++i) {
                const double nx = __dadd_rn(a, s.warp_tot[i]);
                if (__dadd_rn(Pc, nx) > target) { ws = i; om = a; break; }
                a = nx;
            }
            s.wstar = ws;
            s.draw_total = om;  // prefix of the crossing warp
            s.x_found = -1;
        }
        __syncthreads();
        if (w == s.wstar) {
            const double om = s.draw_total;
            const double end = __dadd_rn(Pc, __dadd_rn(om, __dadd_rn(lp, tau)));
            const unsigned hit = __ballot_sync(0xffffffffu, end > target);
            const int L = hit ? __ffs(hit) - 1 : 31;
            if (lane == L) {
                double loc = 0.0;
                int found = -1;
                for (int j = t0; j < t1; ++j) {
                    loc = __dadd_rn(loc, wat(j));
                    if (__dadd_rn(Pc, __dadd_rn(om, __dadd_rn(lp, loc))) > target) { found = j; break; }
                }
                s.x_found = found;
            }
        }
        __syncthreads();
        if (tid == 0) {
            int x = s.x_found;
            if (x < 0)  // the target fell in a rounding gap: this CTA's last positive weight
                for (int j = v1 - 1; j >= v0; --j)
                    if (wat(j) > 0.0) { x = j; break; }
            *x_out = x;
        }
        return tid == 0 ? kDrawWrote : kDrawNone;
    }
    return kDrawNone;
}

// ---------------------------------------------------------------------------
// statistics kernel: one cluster per logits row
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) sampler_stats_kernel(const __grid_constant__ SamplerParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SamplerSmem &s = *reinterpret_cast<SamplerSmem *>(smem_raw + kRegionBytes);
    Region rg;
    rg.cache = reinterpret_cast<float *>(smem_raw);
    rg.ecache = reinterpret_cast<double *>(smem_raw + kOffExp);
    rg.hist_mass = reinterpret_cast<double *>(smem_raw + kOffHistMass);
    rg.cand = reinterpret_cast<unsigned long long *>(smem_raw + kOffCand);
    rg.cand_e = reinterpret_cast<double *>(smem_raw + kOffCandE);
    float *cache = rg.cache;
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int tid = threadIdx.x;
    const int lane = tid & 31, wid = tid >> 5;
    const int V = p.V;
    const int slice = (V + C - 1) / C;
    const int v0 = min(V, rank * slice), v1 = min(V, v0 + slice);
    const bool cached_e = (v1 - v0) <= kCacheFloats;        // logits and their exps in shared memory
    const bool cached = (v1 - v0) <= kCacheFloatsLogits;    // logits in shared memory
    const float *L = row_ptr(p, row);
    const double T = (double)p.T;
    const double invT = T > 0.0 ? 1.0 / T : 0.0;
    const bool topp_all = !(p.top_p < 1.0f);
    double *erow = p.ecache ? p.ecache + (size_t)row * V : nullptr;
    build_exp_table(s.exp_tab);  // first used after the P1 barriers
    allow_dependents();          // the draw kernel waits for this grid's completion itself
    wait_for_producer();         // the logits
    if (p.verify && row == 0 && rank == 0)  // ticket counters of the draw kernel
        for (int k = tid; k < p.B; k += kThreads) p.counters[k] = 0u;
    // A token's logit: from the slice cache when the slice fits it, else from
    // global memory.  The source is chosen once: written as a per-element
    // "cached ? cache[.] : L[.]", the compiler may issue both loads and
    // select, paying an L2 round trip per batch even when every token is in
    // shared memory.
    const float *lsrc = cached ? cache : L;
    const int loff = cached ? v0 : 0;
    auto lval = [&](int j) -> float { return lsrc[j - loff]; };

    // ---------------- P1: read the slice; max, min, argmax, finiteness ----------------
    float g_m, g_min;
    int g_arg, g_bad;
    {
        float mx = -INFINITY, mn = INFINITY;
        int arg = INT_MAX, bad = 0;
        // an aligned slice comes in with one bulk copy; otherwise batches of
        // kBatch loads are issued before any use or store, so the L2 round
        // trips overlap
        const int n = v1 - v0;
        const bool bulk = cached && n > 0 && (n & 3) == 0 && aligned16(L + v0);
        if (bulk) {
            if (tid == 0) {
                mbar_init(&s.bar);
                mbar_expect(&s.bar, (unsigned)n * 4u);
                bulk_load(cache, L + v0, (unsigned)n * 4u, &s.bar);
            }
            if (!mbar_wait_block(&s.bar, 0, p.wait_polls, &s.wait_ok)) bad = 2;  // reported as timed out
        }
        if (bulk) {
            // 16-byte shared loads of contiguous runs, each thread's tokens in
            // ascending order (the first of equal maxima is kept; the warp
            // reduction takes the lowest index)
            const unsigned cbase = smem_u32(cache);
            for (int i = tid; i < (n >> 2); i += kThreads) {
                float e[4];
                asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                             : "=f"(e[0]), "=f"(e[1]), "=f"(e[2]), "=f"(e[3])
                             : "r"(cbase + 16u * (unsigned)i));
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float l = e[k];
                    if (!isfinite(l)) bad |= 1;
                    if (l > mx) { mx = l; arg = v0 + 4 * i + k; }
                    mn = fminf(mn, l);
                }
            }
        }
        for (int j0 = v0 + tid; !bulk && j0 < v1; j0 += kBatch * kThreads) {
            float lv[kBatch];
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
                const int j = j0 + q * kThreads;
                lv[q] = j < v1 ? __ldg(L + j) : 0.0f;
            }
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
                const int j = j0 + q * kThreads;
                if (j < v1) {
                    const float l = lv[q];
                    if (cached) cache[j - v0] = l;
                    if (!isfinite(l)) bad |= 1;
                    if (l > mx) { mx = l; arg = j; }
                    mn = fminf(mn, l);
                }
            }
        }
        warp_max_min_arg(mx, arg, mn, bad);
        if (lane == 0) { s.red_f[wid] = mx; s.red_f2[wid] = mn; s.red_i[wid] = arg; s.red_i2[wid] = bad; }
        __syncthreads();
        // the CTA's result in every lane of warp 0, published into every CTA
        if (wid == 0) {
            float bm = lane < kWarps ? s.red_f[lane] : -INFINITY;
            int ba = lane < kWarps ? s.red_i[lane] : INT_MAX;
            float bn = lane < kWarps ? s.red_f2[lane] : INFINITY;
            int bb = lane < kWarps ? s.red_i2[lane] : 0;
            warp_max_min_arg(bm, ba, bn, bb);
            publish(cluster, s.all_max, rank, C, bm);
            publish(cluster, s.all_arg, rank, C, ba);
            publish(cluster, s.all_min, rank, C, bn);
            publish(cluster, s.all_bad, rank, C, bb);
        }
        cluster.sync();
        // every warp combines the cluster's values itself, in the same order
        // (so with the same result): no warp waits on another after the
        // cluster barrier
        float gm = lane < C ? s.all_max[lane] : -INFINITY;
        int ga = lane < C ? s.all_arg[lane] : INT_MAX;
        float gn = lane < C ? s.all_min[lane] : INFINITY;
        int gb = lane < C ? s.all_bad[lane] : 0;
        warp_max_min_arg(gm, ga, gn, gb);
        g_m = gm;
        g_min = gn;
        g_arg = ga;
        g_bad = gb;
    }
    const float m = g_m;
    const bool bad = g_bad != 0;

    RowStats st;
    st.m = m;
    st.lmin = g_min;
    st.argmax = g_arg;
    st.status = (g_bad & 2) ? MTPV_ROW_TIMEOUT : bad ? MTPV_ROW_NONFINITE : MTPV_ROW_OK;
    st.Z = 1.0;
    st.Zk = 1.0;
    st.lstar = -INFINITY;
    st.idxstar = INT_MAX;

    if (!bad && T > 0.0) {
        // ---------------- P2: exps, Z, level-1 histogram, e-cache ----------------
        const double md = (double)m;
        const float range = __fsub_rn(m, g_min);
        float inv_w = (range > 0.0f) ? __fdiv_rn((float)kBins, range) : 0.0f;
        if (!isfinite(inv_w)) inv_w = 0.0f;
        // The histogram only locates the crossing bin; the masses that decide
        // the cut are exact fp64 sums taken afterwards.  Per bin: the token
        // count and the tokens' excess over the bin's lower edge, e_j / e_lo - 1
        // as a fraction of the bin's span eps = e_hi / e_lo - 1, in fixed point
        // of at most qmax per token (32-bit integer atomics, exact and
        // order-independent).  Bin b spans logits (m - (b + 1) bw, m - b bw].
        const float bw = inv_w > 0.0f ? __frcp_rn(inv_w) : 0.0f;
        const float xw = __fmul_rn(bw, (float)invT);            // a bin's span in exponent units
        const float eps = xw > 0.0f ? expm1f(xw) : 0.0f;
        const unsigned qmax = (unsigned)min(65536, (int)(4294967295u / (unsigned)max(1, v1 - v0)));
        const float qscale = eps > 0.0f ? (float)qmax / eps : 0.0f;
        unsigned *hcnt = reinterpret_cast<unsigned *>(rg.hist_mass);  // [kBins] counts
        unsigned *hexc = hcnt + kBins;                                 // [kBins] excess
        if (!topp_all) {
            for (int b = tid; b < 2 * kBins; b += kThreads) hcnt[b] = 0u;
            __syncthreads();
        }
        double zt = 0.0;
        // NB tokens per thread at a time, loads before exps before the
        // histogram; full batches first, then the slice's tail in batches of
        // two, so that no exp is spent past its end
        auto p2_batch = [&](auto nb, int j0) {
            constexpr int NB = decltype(nb)::value;
            float lv[NB];
            double ev[NB];
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                const int j = j0 + q * kThreads;
                lv[q] = j < v1 ? lval(j) : m;
            }
#pragma unroll
            for (int q = 0; q < NB; ++q) ev[q] = e_of(lv[q], md, invT, s.exp_tab);
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                const int j = j0 + q * kThreads;
                if (j < v1) {
                    zt += ev[q];
                    if (cached_e) rg.ecache[j - v0] = ev[q];
                    if (!topp_all) {
                        const int b = bin_of(lv[q], m, inv_w);
                        // excess exp(x) - 1 over the lower edge, x in [0, xw] (xw is
                        // small: a third-order series is ample for locating)
                        const float lo = __fsub_rn(m, __fmul_rn(small_float(b + 1), bw));
                        const float x = fminf(xw, fmaxf(0.0f, __fmul_rn(__fsub_rn(lv[q], lo), (float)invT)));
                        const float ex = __fmul_rn(x, __fmaf_rn(x, __fmaf_rn(x, 0.16666667f, 0.5f), 1.0f));
                        atomicAdd(&hcnt[b], 1u);
                        atomicAdd(&hexc[b], min(qmax, rint_small(__fmul_rn(ex, qscale))));
                    }
                }
            }
        };
        int j0 = v0 + tid;
        for (; j0 + (kBatch - 1) * kThreads < v1; j0 += kBatch * kThreads)
            p2_batch(std::integral_constant<int, kBatch>{}, j0);
        for (; j0 < v1; j0 += 2 * kThreads) p2_batch(std::integral_constant<int, 2>{}, j0);
        const double zc = block_sum_d(zt, s);  // its barriers also complete the histogram
        // publish Z, and send every CTA the part of this CTA's histogram that
        // it owns (bins [r per, (r + 1) per) to CTA r, slot rank): warp r
        // copies one contiguous run into CTA r's scratch (the candidate area,
        // unused until the gather)
        const int per = kBins / C;
        if (wid == 0) publish(cluster, s.all_Z, rank, C, zc);
        if (tid == 0) s.cand_count = 0u;
        if (!topp_all) {
            for (int r = wid; r < C; r += kWarps) {
                uint2 *dst = reinterpret_cast<uint2 *>(cluster.map_shared_rank(rg.cand, r)) + rank * per;
                for (int i = lane; i < per; i += 32)
                    dst[i] = make_uint2(hcnt[r * per + i], hexc[r * per + i]);
            }
        }
        cluster.sync();
        st.Z = ordered_sum(s.all_Z, C, 0, nullptr);  // every warp, same order
        st.Zk = st.Z;

        if (!topp_all) {
            // ---------------- P3: crossing bin, exact cut ----------------
            const double thr = __dmul_rn((double)p.top_p, st.Z);
            const int base = rank * per;
            // masses of the bins this CTA owns (kBins / C of them), in the
            // histogram's region: its counts went to their owners before the
            // cluster barrier above, so the region is free
            double *own = rg.hist_mass;
            // the cluster's histogram on the bins this CTA owns: the C copies'
            // integer sums, turned into an approximate mass
            // e_lo (count + excess eps / qmax), e_lo = exp(-(b + 1) xw)
            {
                const uint2 *scr = reinterpret_cast<const uint2 *>(rg.cand);
                const double kex = (double)eps / (double)qmax;
                for (int b = tid; b < per; b += kThreads) {
                    unsigned long long cn = 0ull, ex = 0ull;
                    for (int r = 0; r < C; ++r) {
                        const uint2 v = scr[r * per + b];
                        cn += v.x;
                        ex += v.y;
                    }
                    const double elo = exp_neg(-(double)(base + b + 1) * (double)xw, s.exp_tab);
                    own[b] = elo * ((double)cn + (double)ex * kex);
                }
            }
            __syncthreads();
            if (wid == 0) {
                int f;
                double bef;
                const double t = warp_prefix_search(own, per, 0.0, 0.0, false, &f, &bef);
                publish(cluster, s.all_rt, rank, C, t);
            }
            cluster.sync();
            if (wid == 0) {
                // first range whose inclusive prefix reaches thr (same order everywhere)
                const double v = lane < C ? s.all_rt[lane] : 0.0;
                double P = 0.0, Pstar = 0.0;
                int cstar = -1;
                for (int r = 0; r < C; ++r) {
                    const double nx = __dadd_rn(P, __shfl_sync(0xffffffffu, v, r));
                    if (cstar < 0 && nx >= thr) { cstar = r; Pstar = P; }
                    P = nx;
                }
                int bstar = -2;
                if (cstar == rank) {
                    int f;
                    double bef;
                    warp_prefix_search(own, per, Pstar, thr, true, &f, &bef);
                    if (f < 0) f = per - 1;  // not reachable: the range total reached thr
                    bstar = base + f;
                } else if (cstar < 0 && rank == 0) {
                    bstar = -1;  // thr above the histogram total (top_p within its rounding of 1)
                }
                if (bstar != -2 && lane < C) *cluster.map_shared_rank(&s.bc_bin, lane) = bstar;
            }
            cluster.sync();
            const int bstar = s.bc_bin;
            // One pass over the slice: the exact mass above the located bin (A)
            // and in it (M), fp64 sums in a fixed order (each thread's tokens
            // in index order, then fixed trees, then the CTAs in rank order), so
            // they are the same bits in every run; and the located bin's tokens
            // gathered into CTA 0: staged locally, a range reserved with one
            // remote atomic, copied.  The bin's size is known once every CTA has
            // reserved its range.
            unsigned total = 0u;
            double A = 0.0, Mb = 0.0;
            if (bstar >= 0) {
                unsigned long long *stage = reinterpret_cast<unsigned long long *>(rg.cand_e);
                if (tid == 0) s.local_n = 0u;
                __syncthreads();
                double a_loc = 0.0, m_loc = 0.0;
                // each thread's tokens in ascending order (the sums' order);
                // kBatch logits loaded before any is used, and the weight
                // source chosen outside the loop (not per token)
                auto take = [&](float l, int j, double e) {
                    if (bin_of(l, m, inv_w) < bstar) {
                        a_loc = __dadd_rn(a_loc, e);
                    } else {
                        m_loc = __dadd_rn(m_loc, e);
                        const unsigned slot = atomicAdd(&s.local_n, 1u);
                        if (slot < (unsigned)kCandCap) stage[slot] = rank_key(l, j);
                    }
                };
                for (int j0 = v0 + tid; j0 < v1; j0 += kBatch * kThreads) {
                    float lv[kBatch];
#pragma unroll
                    for (int q = 0; q < kBatch; ++q) {
                        const int j = j0 + q * kThreads;
                        lv[q] = j < v1 ? lval(j) : 0.0f;
                    }
                    if (cached_e) {
#pragma unroll
                        for (int q = 0; q < kBatch; ++q) {
                            const int j = j0 + q * kThreads;
                            if (j < v1 && bin_of(lv[q], m, inv_w) <= bstar) take(lv[q], j, rg.ecache[j - v0]);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < kBatch; ++q) {
                            const int j = j0 + q * kThreads;
                            if (j < v1 && bin_of(lv[q], m, inv_w) <= bstar) take(lv[q], j, e_of(lv[q], md, invT, s.exp_tab));
                        }
                    }
                }
                double a_cta = a_loc, m_cta = m_loc;
                block_sum_d2(a_cta, m_cta, s);  // also completes the staging
                if (wid == 0) {
                    publish(cluster, s.all_part, rank, C, a_cta);
                    publish(cluster, s.all_M, rank, C, m_cta);
                }
                const unsigned nloc = min(s.local_n, (unsigned)kCandCap);
                if (tid == 0)
                    s.local_base = nloc ? atomicAdd(cluster.map_shared_rank(&s.cand_count, 0), nloc) : 0u;
                __syncthreads();
                {
                    unsigned long long *ck = cluster.map_shared_rank(rg.cand, 0);
                    const unsigned b0 = s.local_base;
                    for (unsigned i = tid; i < nloc; i += kThreads)
                        if (b0 + i < (unsigned)kCandCap) ck[b0 + i] = stage[i];
                }
                cluster.sync();
                total = *cluster.map_shared_rank(&s.cand_count, 0);
                A = ordered_sum(s.all_part, C, 0, nullptr);  // every warp, same order
                Mb = ordered_sum(s.all_M, C, 0, nullptr);
            }
            // The exact cut lies in the located bin iff A < thr <= A + M.  The
            // approximate histogram can miss by a bin when thr falls within its
            // rounding of a bin edge, and finds no bin when thr is within it of
            // the total: the radix select then finds the cut from scratch.
            const bool located = bstar >= 0 && total > 0u && A < thr && thr <= __dadd_rn(A, Mb);
            if (located && total <= (unsigned)kCandCap) {
                if (rank == 0 && (int)total <= kThreads) {
                    // one candidate per thread: its rank among the others (the
                    // keys are distinct, they carry the token index) places it
                    // and its exp in descending order; a block scan of the
                    // sorted exps gives every candidate its preceding mass
                    const int n = (int)total;
                    // with few candidates, `parts` threads share one: thread
                    // part * S + i counts the keys above candidate i in the
                    // part-th run of the list (runs of even length, so the
                    // 16-byte loads stay aligned); the counts are added below
                    const int parts = n <= kThreads / 4 ? 4 : n <= kThreads / 2 ? 2 : 1;
                    const int S = kThreads / parts, ci = tid % S, part = tid / S;
                    const int L = (((n + parts - 1) / parts) + 1) & ~1;
                    const int k0 = min(n, part * L), k1 = min(n, k0 + L);
                    const unsigned long long key = ci < n ? rg.cand[ci] : 0ull;
                    int r = 0;
                    if (ci < n) {
                        // 16-byte loads, four in flight, four independent
                        // counts: the loop is bound by shared-memory latency
                        const ulonglong2 *c2 = reinterpret_cast<const ulonglong2 *>(rg.cand);
                        int r0 = 0, r1 = 0, r2 = 0, r3 = 0, j = k0;
                        for (; j + 8 <= k1; j += 8) {
                            const ulonglong2 a = c2[j >> 1], b = c2[(j >> 1) + 1];
                            const ulonglong2 c = c2[(j >> 1) + 2], d = c2[(j >> 1) + 3];
                            r0 += (a.x > key ? 1 : 0) + (c.x > key ? 1 : 0);
                            r1 += (a.y > key ? 1 : 0) + (c.y > key ? 1 : 0);
                            r2 += (b.x > key ? 1 : 0) + (d.x > key ? 1 : 0);
                            r3 += (b.y > key ? 1 : 0) + (d.y > key ? 1 : 0);
                        }
                        for (; j < k1; ++j) r0 += rg.cand[j] > key ? 1 : 0;
                        r = (r0 + r1) + (r2 + r3);
                    }
                    if (parts > 1) {
                        int *rp = reinterpret_cast<int *>(s.thr_excl);
                        rp[tid] = r;
                        __syncthreads();
                        if (part == 0)
                            for (int q = 1; q < parts; ++q) r += rp[q * S + ci];
                    }
                    const double e = tid < n ? e_of(key_logit(key), md, invT, s.exp_tab) : 0.0;
                    __syncthreads();
                    if (tid < n) {
                        rg.cand[r] = key;
                        rg.cand_e[r] = e;
                    }
                    if (tid == 0) s.first_fail = INT_MAX;
                    __syncthreads();
                    double excl;
                    const double incl = block_scan_d(tid < n ? rg.cand_e[tid] : 0.0, s, &excl);
                    if (tid < n && __dadd_rn(A, excl) >= thr) atomicMin(&s.first_fail, tid);
                    __syncthreads();
                    int cut = (s.first_fail == INT_MAX) ? n - 1 : s.first_fail - 1;
                    if (cut < 0) cut = 0;  // A < thr by construction: the first is kept
                    if (tid == cut) {
                        s.cut_Zk = __dadd_rn(A, incl);
                        s.cut_pos = cut;
                        s.cut_idx = key_index(rg.cand[cut]);
                        s.cut_l = key_logit(rg.cand[cut]);
                    }
                    __syncthreads();
                    if (tid == 0) s.cut_n = n;
                } else if (rank == 0) {
                    // more candidates than threads: shared-memory bitonic sort
                    const int n = min((int)s.cand_count, kCandCap);
                    int n2 = 1;
                    while (n2 < n) n2 <<= 1;
                    for (int i = n + tid; i < n2; i += kThreads) rg.cand[i] = 0ull;
                    __syncthreads();
                    for (int k = 2; k <= n2; k <<= 1) {  // bitonic sort, descending
                        for (int jj = k >> 1; jj > 0; jj >>= 1) {
                            for (int i = tid; i < n2; i += kThreads) {
                                const int ix = i ^ jj;
                                if (ix > i) {
                                    unsigned long long a = rg.cand[i], b = rg.cand[ix];
                                    const bool desc = (i & k) == 0;
                                    if (desc ? (a < b) : (a > b)) { rg.cand[i] = b; rg.cand[ix] = a; }
                                }
                            }
                            __syncthreads();
                        }
                    }
                    for (int i = tid; i < n; i += kThreads) rg.cand_e[i] = e_of(key_logit(rg.cand[i]), md, invT, s.exp_tab);
                    // exclusive prefix over the sorted candidates: sequential
                    // chunks per thread, thread totals chained by warp 0
                    const int ch = (n + kThreads - 1) / kThreads;
                    const int i0 = min(n, tid * ch), i1 = min(n, i0 + ch);
                    __syncthreads();
                    double tt = 0.0;
                    for (int i = i0; i < i1; ++i) tt = __dadd_rn(tt, rg.cand_e[i]);
                    s.thr_excl[tid] = tt;
                    if (tid == 0) s.first_fail = INT_MAX;
                    __syncthreads();
                    if (wid == 0) {
                        constexpr int per_lane = kThreads / 32;
                        double lt = 0.0;
                        for (int q = 0; q < per_lane; ++q) lt = __dadd_rn(lt, s.thr_excl[lane * per_lane + q]);
                        double acc = 0.0, start = 0.0;
                        for (int r = 0; r < 32; ++r) {
                            const double v = __shfl_sync(0xffffffffu, lt, r);
                            if (r == lane) start = acc;
                            acc = __dadd_rn(acc, v);
                        }
                        for (int q = 0; q < per_lane; ++q) {
                            const double v = s.thr_excl[lane * per_lane + q];
                            s.thr_excl[lane * per_lane + q] = start;
                            start = __dadd_rn(start, v);
                        }
                    }
                    __syncthreads();
                    {
                        double ex = s.thr_excl[tid];
                        for (int i = i0; i < i1; ++i) {
                            if (__dadd_rn(A, ex) >= thr) { atomicMin(&s.first_fail, i); break; }
                            ex = __dadd_rn(ex, rg.cand_e[i]);
                        }
                    }
                    __syncthreads();
                    int cut = (s.first_fail == INT_MAX) ? n - 1 : s.first_fail - 1;
                    if (cut < 0) cut = 0;  // A < thr by construction: the first is kept
                    if (cut >= i0 && cut < i1) {
                        double ex = s.thr_excl[tid];
                        for (int i = i0; i < cut; ++i) ex = __dadd_rn(ex, rg.cand_e[i]);
                        s.cut_Zk = __dadd_rn(A, __dadd_rn(ex, rg.cand_e[cut]));
                        s.cut_pos = cut;
                        s.cut_idx = key_index(rg.cand[cut]);
                        s.cut_l = key_logit(rg.cand[cut]);
                    }
                    __syncthreads();
                    if (tid == 0) s.cut_n = n;
                }
                // Only CTA 0 needs the cut.  Meanwhile the weights go out
                // masked by bin (above the located bin kept, below it not, in
                // it kept for now): every other CTA stores its own slice and a
                // share of CTA 0's (read from CTA 0's shared memory, which the
                // cut does not touch), arrives on a cluster barrier and leaves.
                // CTA 0 waits there (the peers' stores and reads are done),
                // zeroes its candidates past the cut and writes the statistics.
                // (with a weight cache every slice fits shared memory with its
                // exps: the launch drops the cache otherwise, so the test is the
                // same in every CTA)
                const bool store = erow && slice <= kCacheFloats;
                if (store) {
                    auto store_masked = [&](const float *lc, const double *ec, int jb, int i0, int i1) {
                        for (int i = i0 + tid; i < i1; i += kThreads)
                            erow[jb + i] = bin_of(lc[i], m, inv_w) <= bstar ? ec[i] : 0.0;
                    };
                    const int n0 = min(V, slice);  // CTA 0's slice: [0, n0)
                    if (rank != 0) {
                        store_masked(rg.cache, rg.ecache, v0, 0, v1 - v0);
                        const int q = (((n0 + C - 2) / (C - 1)) + 31) & ~31;
                        store_masked(cluster.map_shared_rank(rg.cache, 0), cluster.map_shared_rank(rg.ecache, 0), 0,
                                     min(n0, (rank - 1) * q), min(n0, rank * q));
                    } else if (C == 1) {
                        store_masked(rg.cache, rg.ecache, v0, 0, v1 - v0);
                    }
                }
                cluster_arrive();
                if (rank != 0) return;
                cluster_wait();
                if (store) {
                    // candidates past the cut are not kept
                    for (int i = s.cut_pos + 1 + tid; i < s.cut_n; i += kThreads)
                        erow[key_index(rg.cand[i])] = 0.0;
                }
                st.Zk = s.cut_Zk;
                st.idxstar = s.cut_idx;
                st.lstar = s.cut_l;
                if (tid == 0) p.slots[row].st = st;
                return;
            } else {
                // weighted radix select on the 64-bit key, 8 bits per pass
                unsigned long long prefix = 0ull, mask = 0ull;
                double above = 0.0;
                for (int pass = 0; pass < 8; ++pass) {
                    const int shift = 56 - 8 * pass;
                    for (int d = tid; d < 256; d += kThreads) { s.rad_mass[d] = 0.0; s.rad_cnt[d] = 0; }
                    __syncthreads();
                    {
                        int cur = -1, ccnt = 0;
                        double cacc = 0.0;
                        for (int j = v0 + tid; j < v1; j += kThreads) {
                            const float l = lval(j);
                            const unsigned long long key = rank_key(l, j);
                            if ((key & mask) != prefix) continue;
                            const int d = (int)((key >> shift) & 255ull);
                            const double e = cached_e ? rg.ecache[j - v0] : e_of(l, md, invT, s.exp_tab);
                            if (d != cur) {
                                if (cur >= 0) { atomicAdd(&s.rad_mass[cur], cacc); atomicAdd(&s.rad_cnt[cur], ccnt); }
                                cur = d; cacc = 0.0; ccnt = 0;
                            }
                            cacc += e;
                            ++ccnt;
                        }
                        if (cur >= 0) { atomicAdd(&s.rad_mass[cur], cacc); atomicAdd(&s.rad_cnt[cur], ccnt); }
                    }
                    cluster.sync();
                    for (int d = tid; d < 256; d += kThreads) {
                        double ms = 0.0;
                        int cn = 0;
                        for (int r = 0; r < C; ++r) {
                            ms = __dadd_rn(ms, cluster.map_shared_rank(s.rad_mass, r)[d]);
                            cn += cluster.map_shared_rank(s.rad_cnt, r)[d];
                        }
                        s.own_mass[d] = ms;
                        s.own_cnt[d] = cn;
                    }
                    __syncthreads();
                    if (tid == 0) {
                        double acc = above, Asel = above, Alast = above;
                        int dsel = -1, dlast = -1;
                        for (int d = 255; d >= 0; --d) {
                            if (s.own_cnt[d] == 0) continue;
                            dlast = d;
                            Alast = acc;
                            const double nx = __dadd_rn(acc, s.own_mass[d]);
                            if (nx >= thr) { dsel = d; Asel = acc; break; }
                            acc = nx;
                        }
                        if (dsel < 0) { dsel = dlast; Asel = Alast; }
                        s.bc_bin = dsel;
                        s.bc_A = Asel;
                    }
                    cluster.sync();  // peers are done reading rad_* before the next pass clears them
                    prefix |= ((unsigned long long)s.bc_bin & 255ull) << shift;
                    mask |= 255ull << shift;
                    above = s.bc_A;
                }
                st.lstar = key_logit(prefix);
                st.idxstar = key_index(prefix);
                st.Zk = __dadd_rn(above, e_of(st.lstar, md, invT, s.exp_tab));
            }
        }
    }

    // the row's statistics, then its weights: e_j of kept tokens, 0 elsewhere
    if (rank == 0 && tid == 0) p.slots[row].st = st;
    if (erow && !bad && T > 0.0) {
        const double md = (double)m;
        if (cached_e) {  // coalesced 8-byte stores; they drain after the CTA has moved on
            for (int j = v0 + tid; j < v1; j += kThreads)
                erow[j] = is_kept(st, rg.cache[j - v0], j) ? rg.ecache[j - v0] : 0.0;
        } else {
            for (int j0 = v0 + tid; j0 < v1; j0 += kBatch * kThreads) {
                float lv[kBatch];
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const int j = j0 + q * kThreads;
                    lv[q] = j < v1 ? lval(j) : -INFINITY;
                }
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const int j = j0 + q * kThreads;
                    if (j < v1) erow[j] = is_kept(st, lv[q], j) ? e_of(lv[q], md, invT, s.exp_tab) : 0.0;
                }
            }
        }
    }
    // No closing cluster barrier: every access to a peer's shared memory above
    // is followed by a cluster barrier that the peer also passes, so no CTA can
    // leave while a peer still reads or writes its shared memory.
}

// ---------------------------------------------------------------------------
// draw kernel: one cluster per draft position (verify) or per row (sample)
// ---------------------------------------------------------------------------
// A verify call's per-position inputs, from the launch parameters or from memory.
__device__ __forceinline__ int32_t draft_at(const SamplerParams &p, size_t k) {
    return p.inline_inputs ? p.inl.drafts[k] : p.drafts[k];
}
__device__ __forceinline__ float u_acc_at(const SamplerParams &p, size_t k) {
    return p.inline_inputs ? p.inl.u_acc[k] : p.u_acc[k];
}
__device__ __forceinline__ float u_samp_at(const SamplerParams &p, size_t k) {
    return p.inline_inputs ? p.inl.u_samp[k] : p.u_samp[k];
}

__global__ void __launch_bounds__(kThreads, 1) sampler_draw_kernel(const __grid_constant__ SamplerParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SamplerSmem &s = *reinterpret_cast<SamplerSmem *>(smem_raw + kDrawBufBytes);
    double *wbuf = reinterpret_cast<double *>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x;
    const int V = p.V, K = p.K;
    const int slice = (V + C - 1) / C;
    const int v0 = min(V, rank * slice), v1 = min(V, v0 + slice);
    const double T = (double)p.T;
    const double invT = T > 0.0 ? 1.0 / T : 0.0;

    // this cluster's rows: verify position i of sequence b -> target row i and
    // (i < K) draft row i; sample -> one row
    const int c = blockIdx.y;
    int b = c, i = 0, rt = c, rd = c;
    if (p.verify) {
        const int S = 2 * K + 1;
        b = c / (K + 1);
        i = c - b * (K + 1);
        rt = b * S + i;
        rd = i < K ? b * S + K + 1 + i : rt;
    }
    const bool residual = p.verify && i < K;
    if (rank == 0 && tid == 0) s.res_acc = 0;
    build_exp_table(s.exp_tab);
    __syncthreads();
    wait_for_producer();  // the statistics kernel's rows and weights
    const float *Lt = row_ptr(p, rt), *Ld = row_ptr(p, rd);
    const double *Et = p.ecache ? p.ecache + (size_t)rt * V : nullptr;
    const double *Ed = p.ecache ? p.ecache + (size_t)rd * V : nullptr;

    // ---------------- the position's status, acceptance test of d_i ----------------
    // (verify: the slot of target row i becomes position i's record, whose
    // first 12 bytes are written after the last cluster barrier below; the
    // status field of the row statistics lies past them and is read first)
    int status = p.slots[rt].st.status;
    int d = 0;
    if (residual) {
        d = draft_at(p, (size_t)b * K + i);
        const int sd = p.slots[rd].st.status;
        if (d < 0 || d >= V) status = MTPV_ROW_BAD_DRAFT;
        else if (sd != MTPV_ROW_OK && status == MTPV_ROW_OK) status = sd;
    }
    const bool draws = status == MTPV_ROW_OK && T > 0.0;
    RowStats st_t = {}, st_d = {};
    if (draws || (rank == 0 && tid == 0)) {
        st_t = p.slots[rt].st;
        st_d = p.slots[rd].st;
    }
    if (residual && status == MTPV_ROW_OK && rank == 0 && tid == 0) {
        double pt, qd;  // p'_i(d_i), q'_i(d_i)
        if (Et && T > 0.0) {
            pt = Et[d] / st_t.Zk;
            qd = Ed[d] / st_d.Zk;
        } else {
            pt = warped_prob(st_t, Lt, d, T, invT, s.exp_tab);
            qd = warped_prob(st_d, Ld, d, T, invT, s.exp_tab);
        }
        const double ratio = (qd == 0.0) ? (pt > 0.0 ? INFINITY : 0.0) : pt / qd;
        s.res_acc = (double)u_acc_at(p, (size_t)b * K + i) < ratio ? 1 : 0;
    }

    // ---------------- this position's residual / bonus draw ----------------
    // The CTA that finds the token writes it to global memory itself (verify:
    // the record's x; sample: the output), so no CTA waits for another at the
    // end.  CTA 0 writes it instead when no draw runs or the draw timed out.
    int *x_dst = p.verify ? &p.slots[rt].rec.x : &p.out_tokens[c];
    int drew = kDrawNone;
    if (draws) {
        DrawSrc src;
        src.st_t = st_t;
        src.st_d = residual ? st_d : st_t;
        src.Lt = Lt;
        src.Ld = residual ? Ld : Lt;
        src.Et = Et;
        src.Ed = residual ? Ed : Et;
        src.tab = s.exp_tab;
        src.rho = residual ? st_t.Zk / st_d.Zk : 1.0;
        src.kind = residual ? 1 : 0;
        const float u = p.verify ? u_samp_at(p, (size_t)b * (K + 1) + i) : p.u_samp[c];
        drew = cluster_draw(cluster, s, wbuf, src, residual, invT, u, v0, v1, x_dst, p.wait_polls);
    }
    if (drew == kDrawTimeout) status = MTPV_ROW_TIMEOUT;
    const bool cta0_token = status != MTPV_ROW_OK || T == 0.0;
    unsigned tickets = 0u;
    if (rank == 0 && tid == 0) {
        if (cta0_token) *x_dst = status == MTPV_ROW_OK ? st_t.argmax : -1;
        if (!p.verify) {
            if (p.row_status) p.row_status[c] = status;
            return;
        }
        // the record's other fields, and one ticket for them (two when
        // this thread wrote the token as well)
        p.slots[rt].rec.accept = s.res_acc;
        p.slots[rt].rec.status = status;
        tickets = cta0_token ? 2u : 1u;
    }
    if (!p.verify) return;
    if (drew == kDrawWrote && tid == 0) tickets += 1u;  // the token's ticket
    if (tickets == 0u) return;

    // ---------------- tickets, and (last) the sequence's outputs ----------------
    // Two tickets per position; the thread that completes the sequence's
    // 2 (K + 1) writes its outputs (nobody waits for anybody).
    const int S = 2 * K + 1;
    __threadfence();
    const unsigned old = atomicAdd(&p.counters[b], tickets);
    if (old + tickets != 2u * (unsigned)(K + 1)) return;
    __threadfence();
    int seq_status = MTPV_ROW_OK, n = K;
    for (int k = 0; k <= K; ++k) {
        const int sk = __ldcg(&p.slots[b * S + k].rec.status);
        if (sk == MTPV_ROW_BAD_DRAFT) seq_status = MTPV_ROW_BAD_DRAFT;
        else if (sk != MTPV_ROW_OK && seq_status == MTPV_ROW_OK) seq_status = sk;
    }
    for (int k = 0; k < K; ++k)
        if (!__ldcg(&p.slots[b * S + k].rec.accept)) { n = k; break; }
    int32_t *ot = p.out_tokens + (size_t)b * (K + 1);
    if (seq_status != MTPV_ROW_OK) {
        for (int k = 0; k <= K; ++k) ot[k] = -1;
        p.out_acc[b] = -1;
    } else {
        for (int k = 0; k < n; ++k) ot[k] = draft_at(p, (size_t)b * K + k);
        ot[n] = __ldcg(&p.slots[b * S + n].rec.x);
        for (int k = n + 1; k <= K; ++k) ot[k] = -1;
        p.out_acc[b] = n;
    }
    if (p.row_status) p.row_status[b] = seq_status;
    p.counters[b] = 0u;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

// Cluster size of a sampler launch: the largest power of two up to 16 that
// can be resident on the device (the occupancy calculator is asked once per
// kernel and device); launch_sampler may halve it for many rows.  The kernels
// work with any power of two from 1 to 16, but smaller clusters only pay if a
// CTA's slice still fits its shared-memory cache: past it every pass re-reads
// the row from L2, which on B200 cost more than the waves it saves (8
// sequences x 3 drafts at vocabulary 248320, before the logits-only cache:
// 459 us with 16-CTA clusters in waves, 581 us with 2-CTA clusters in one).
int g_max_active[2][64][5];  // [kernel][device][log2 C]: clusters resident at once; -1 = cannot launch
bool g_known[2][64];
std::mutex g_cluster_mu;

template <typename Kern>
int cluster_size_for(int which, Kern kernel, size_t smem, int units) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 8;
    }
    std::lock_guard<std::mutex> lock(g_cluster_mu);
    if (!g_known[which][dev]) {
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        for (int lg = 0; lg < 5; ++lg) {
            const int c = 1 << lg;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(c, 1, 1);
            cfg.blockDim = dim3(kThreads, 1, 1);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = c;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
                cudaGetLastError();
                n = -1;
            }
            g_max_active[which][dev][lg] = n;
        }
        g_known[which][dev] = true;
    }
    (void)units;
    for (int lg = 4; lg >= 0; --lg)
        if (g_max_active[which][dev][lg] > 0) return 1 << lg;
    return 8;
}

// Clusters of size c (a power of two) of a kernel whose table is filled (by
// cluster_size_for) that the device holds at once; 0 if unknown.
int max_active_clusters(int which, int c) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 0;
    }
    int lg = 0;
    while ((1 << lg) < c && lg < 4) ++lg;
    std::lock_guard<std::mutex> lock(g_cluster_mu);
    return g_known[which][dev] ? std::max(0, g_max_active[which][dev][lg]) : 0;
}

// Both sampler kernels are launched as programmatic dependents of the work
// before them on the stream: their CTAs may be scheduled while that work
// drains, and each waits (griddepcontrol.wait) for it to complete before
// reading its results.
template <typename Kern>
cudaError_t launch_clusters(Kern kernel, int C, int clusters, size_t smem, const SamplerParams &p,
                            cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, clusters, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace

static std::atomic<int> g_wait_polls{-1};

void set_wait_polls(int polls) { g_wait_polls.store(polls); }

cudaError_t launch_sampler(const SamplerParams &params, int rows, cudaStream_t stream) {
    SamplerParams p = params;
    const int polls = g_wait_polls.load();
    p.wait_polls = polls < 0 ? kWaitLimit : polls;
    int C1 = cluster_size_for(0, sampler_stats_kernel, kStatsSmemBytes, rows);
    // When the rows need several waves of these clusters, halve the cluster
    // while the halved slices still keep their logits in shared memory and
    // more clusters fit at once: more rows per wave, each CTA twice the
    // tokens (and, past the exps' room, the draw kernel recomputing the kept
    // weights).  Measured per verify at vocabulary 151936: 2 / 4 / 8 / 16
    // sequences 63 -> 61, 117 -> 109, 237 -> 205, 467 -> 399 us; at vocabulary
    // 248320 and 8 sequences 347 -> 286 us; one sequence (7 rows, one wave)
    // keeps 16-CTA clusters.
    while (C1 > 1 && rows > max_active_clusters(0, C1) && (p.V + C1 / 2 - 1) / (C1 / 2) <= kCacheFloatsLogits &&
           max_active_clusters(0, C1 / 2) > max_active_clusters(0, C1))
        C1 /= 2;
    // The fp64 weight cache pays only while a CTA's slice (and its exps) stays
    // in shared memory: then the statistics kernel writes the masked exps it
    // already holds and the draw kernel bulk-loads them.  Past the slice
    // cache the statistics kernel would recompute every kept token's exp to
    // write it, and the draw kernel recomputing them from the logits was
    // measured faster (8 sequences x 3 drafts at vocabulary 248320: 404 vs
    // 453 us; at vocabulary 151936 and one sequence the cache wins, 39 vs
    // 46 us).
    if (p.ecache && (p.V + C1 - 1) / C1 > kCacheFloats) p.ecache = nullptr;
    cudaError_t e = launch_clusters(sampler_stats_kernel, C1, rows, kStatsSmemBytes, p, stream);
    if (e != cudaSuccess) return e;
    const int clusters = p.verify ? p.B * (p.K + 1) : rows;
    const int C2 = cluster_size_for(1, sampler_draw_kernel, kDrawSmemBytes, clusters);
    return launch_clusters(sampler_draw_kernel, C2, clusters, kDrawSmemBytes, p, stream);
}

}  // namespace mtpv
