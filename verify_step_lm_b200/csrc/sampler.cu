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
// Design for sm_100a.  One thread-block cluster of C CTAs (16, or 8 when a
// 16-CTA cluster cannot be resident) owns one row; each CTA owns a contiguous
// slice of the vocabulary.  Cross-CTA reductions go through distributed shared
// memory and hardware cluster barriers (no global flags, no spin loops):
//   P1  max / min / argmax / finiteness of the row
//   P2  e_j = exp((l_j - m)/T) in fp64, Z, and a 2048-bin mass histogram on
//       (m - l_j), binned linearly over the row's own range
//   P3  the bin where the descending cumulative mass reaches top_p * Z; its
//       tokens are gathered into CTA 0, sorted on a (logit desc, index asc)
//       64-bit key and scanned for the exact cut token.  A crossing bin with
//       more than kCandCap tokens (massive ties, degenerate ranges) falls back
//       to an 8-pass weighted radix select on the same key.
//   P4  verify: the last cluster of a sequence to finish its row (a global
//       ticket counter; nobody waits) runs the acceptance tests and the
//       residual / bonus draw.  sample: every cluster draws from its own row.
// The draw is a cluster-wide inverse CDF whose partial sums are formed in one
// fixed nested order (CTA slices, warp chunks, 32-wide steps), so the total,
// the prefix that picks the CTA and the prefix used inside it agree bit for
// bit.  All probability arithmetic is fp64 on the fp32 logits.
#include <cooperative_groups.h>
#include <float.h>
#include <limits.h>
#include <math.h>

#include "common.cuh"
#include "sampler.cuh"

namespace cg = cooperative_groups;

namespace mtpv {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kCandCap = 4096;
constexpr int kMaxK = 16;

struct SamplerSmem {
    double hist_mass[kBins];
    int hist_cnt[kBins];
    unsigned long long cand[kCandCap];
    double cand_e[kCandCap];
    double own_mass[kBins / 8];  // bins owned by this CTA (C >= 8), or radix digits
    int own_cnt[kBins / 8];
    double rad_mass[256];
    int rad_cnt[256];
    double red_d[kWarps];
    float red_f[kWarps];
    float red_f2[kWarps];
    int red_i[kWarps];
    int red_i2[kWarps];
    double warp_tot[kWarps];
    double thr_excl[kThreads];
    // published to the other CTAs of the cluster
    float pub_max, pub_min;
    int pub_arg, pub_bad;
    double pub_Z, pub_range_total, pub_partial;
    // broadcast into every CTA of the cluster
    int bc_bin, bc_cnt, bc_last;
    double bc_A;
    unsigned int cand_count;
    // derived by every CTA for itself
    float g_m, g_min;
    int g_arg, g_bad;
    double g_Z, draw_Pc, draw_total, cut_Zk;
    int wstar, x_found, first_fail, cut_idx;
    float cut_l;
    RowStats st[2 * kMaxK + 1];
    int seq_n, seq_status;
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

__device__ __forceinline__ double e_of(float l, double m, double T) {
    return exp(__dsub_rn((double)l, m) / T);
}

// Level-1 bin of a logit: linear in (m - l) over the row's range; monotone
// (non-increasing) in l, equal logits share a bin.
__device__ __forceinline__ int bin_of(float l, float m, float inv_w) {
    return min(kBins - 1, (int)__fmul_rn(__fsub_rn(m, l), inv_w));
}

__device__ __forceinline__ bool is_kept(const RowStats &st, float l, int j) {
    return (l > st.lstar) || (l == st.lstar && j <= st.idxstar);
}

// p'_j of one row given its statistics.
__device__ __forceinline__ double warped_prob(const RowStats &st, const float *L, int j, double T) {
    if (T == 0.0) return j == st.argmax ? 1.0 : 0.0;
    float l = L[j];
    if (!is_kept(st, l, j)) return 0.0;
    return e_of(l, (double)st.m, T) / st.Zk;
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

// Inclusive warp scan (Kogge-Stone) in fp64.
__device__ __forceinline__ double warp_incl_scan_d(double v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
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

// Weight of token j in a draw.  kind 0: p'_t(j); kind 1: max(0, p'_t(j) - q'_d(j)).
__device__ __forceinline__ double draw_weight(int kind, const RowStats &st_t, const float *Lt,
                                              const RowStats &st_d, const float *Ld, int j,
                                              double T) {
    double pt = warped_prob(st_t, Lt, j, T);
    if (kind == 0) return pt;
    double w = __dsub_rn(pt, warped_prob(st_d, Ld, j, T));
    return w > 0.0 ? w : 0.0;
}

// ---------------------------------------------------------------------------
// Cluster-wide inverse-CDF draw over the row: x = min{k : C_k > u * total}.
// Every CTA of the cluster calls it; the CTA holding the crossing writes
// *x_out.  With allow_fallback, a residual whose total is exactly zero
// (p' == q') is replaced by p'_t.
// ---------------------------------------------------------------------------
__device__ void cluster_draw(cg::cluster_group &cluster, SamplerSmem &s, int kind,
                             bool allow_fallback, const RowStats &st_t, const float *Lt,
                             const RowStats &st_d, const float *Ld, double T, float u, int v0,
                             int v1, int *x_out) {
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int n = v1 - v0;
    const int chunk = ((n + kWarps - 1) / kWarps + 31) & ~31;
    const int c0 = min(v1, v0 + w * chunk), c1 = min(v1, c0 + chunk);

    for (int attempt = 0; attempt < 2; ++attempt) {
        // pass A: warp totals (sequential over 32-wide steps), CTA partial
        double carry = 0.0;
        for (int b = c0; b < c1; b += 32) {
            const int j = b + lane;
            double wj = (j < c1) ? draw_weight(kind, st_t, Lt, st_d, Ld, j, T) : 0.0;
            double inc = warp_incl_scan_d(wj);
            carry = __dadd_rn(carry, __shfl_sync(0xffffffffu, inc, 31));
        }
        if (lane == 0) s.warp_tot[w] = carry;
        __syncthreads();
        if (threadIdx.x == 0) {
            double acc = 0.0;
            for (int i = 0; i < kWarps; ++i) acc = __dadd_rn(acc, s.warp_tot[i]);
            s.pub_partial = acc;
        }
        cluster.sync();
        if (threadIdx.x == 0) {
            double acc = 0.0, pc = 0.0;
            for (int r = 0; r < C; ++r) {
                double part = *cluster.map_shared_rank(&s.pub_partial, r);
                if (r == rank) pc = acc;
                acc = __dadd_rn(acc, part);
            }
            s.draw_Pc = pc;
            s.draw_total = acc;
        }
        cluster.sync();  // all peers have read pub_partial
        const double Pc = s.draw_Pc, total = s.draw_total;
        if (total == 0.0 && allow_fallback && kind == 1) {
            kind = 0;  // p' == q' exactly: draw from p'_n
            continue;
        }
        const double target = __dmul_rn((double)u, total);
        const double next = __dadd_rn(Pc, s.pub_partial);
        if (!(Pc <= target && target < next)) return;  // crossing is in another CTA
        if (threadIdx.x == 0) {
            double acc = 0.0, Wst = 0.0;
            int wst = kWarps - 1;
            for (int i = 0; i < kWarps; ++i) {
                double nx = __dadd_rn(acc, s.warp_tot[i]);
                if (__dadd_rn(Pc, nx) > target) { wst = i; Wst = acc; break; }
                acc = nx;
            }
            s.wstar = wst;
            s.draw_total = Wst;  // reused: prefix of the crossing warp
            s.x_found = -1;
        }
        __syncthreads();
        if (w == s.wstar) {
            const double Ww = s.draw_total;
            double cr = 0.0;
            int found = -1;
            for (int b = c0; b < c1 && found < 0; b += 32) {
                const int j = b + lane;
                double wj = (j < c1) ? draw_weight(kind, st_t, Lt, st_d, Ld, j, T) : 0.0;
                double inc = warp_incl_scan_d(wj);
                double val = __dadd_rn(Pc, __dadd_rn(Ww, __dadd_rn(cr, inc)));
                unsigned msk = __ballot_sync(0xffffffffu, (j < c1) && (val > target));
                if (msk) found = b + __ffs(msk) - 1;
                cr = __dadd_rn(cr, __shfl_sync(0xffffffffu, inc, 31));
            }
            if (lane == 0) s.x_found = found;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int x = s.x_found;
            if (x < 0) {  // not reachable with the consistent sums above; stay valid
                for (int j = v1 - 1; j >= v0; --j)
                    if (draw_weight(kind, st_t, Lt, st_d, Ld, j, T) > 0.0) { x = j; break; }
            }
            *x_out = x;
        }
        return;
    }
}

// ---------------------------------------------------------------------------
// the kernel: one cluster per row
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) sampler_kernel(SamplerParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SamplerSmem &s = *reinterpret_cast<SamplerSmem *>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int tid = threadIdx.x;
    const int lane = tid & 31, wid = tid >> 5;
    const int V = p.V;
    const int slice = (V + C - 1) / C;
    const int v0 = min(V, rank * slice), v1 = min(V, v0 + slice);
    const float *L = row_ptr(p, row);
    const double T = (double)p.T;
    const bool topp_all = !(p.top_p < 1.0f);

    // ---------------- P1: max, min, argmax, finiteness ----------------
    {
        float mx = -INFINITY, mn = INFINITY;
        int arg = INT_MAX, bad = 0;
        for (int j = v0 + tid; j < v1; j += kThreads) {
            float l = L[j];
            if (!isfinite(l)) bad = 1;
            if (l > mx) { mx = l; arg = j; }
            mn = fminf(mn, l);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float om = __shfl_xor_sync(0xffffffffu, mx, o);
            int oa = __shfl_xor_sync(0xffffffffu, arg, o);
            if (om > mx || (om == mx && oa < arg)) { mx = om; arg = oa; }
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            bad |= __shfl_xor_sync(0xffffffffu, bad, o);
        }
        if (lane == 0) { s.red_f[wid] = mx; s.red_f2[wid] = mn; s.red_i[wid] = arg; s.red_i2[wid] = bad; }
        __syncthreads();
        if (tid == 0) {
            mx = s.red_f[0]; arg = s.red_i[0]; mn = s.red_f2[0]; bad = s.red_i2[0];
            for (int i = 1; i < kWarps; ++i) {
                if (s.red_f[i] > mx || (s.red_f[i] == mx && s.red_i[i] < arg)) { mx = s.red_f[i]; arg = s.red_i[i]; }
                mn = fminf(mn, s.red_f2[i]);
                bad |= s.red_i2[i];
            }
            s.pub_max = mx; s.pub_min = mn; s.pub_arg = arg; s.pub_bad = bad;
        }
        cluster.sync();
        if (tid == 0) {
            float gm = -INFINITY, gn = INFINITY;
            int ga = INT_MAX, gb = 0;
            for (int r = 0; r < C; ++r) {
                float rm = *cluster.map_shared_rank(&s.pub_max, r);
                int ra = *cluster.map_shared_rank(&s.pub_arg, r);
                if (rm > gm || (rm == gm && ra < ga)) { gm = rm; ga = ra; }
                gn = fminf(gn, *cluster.map_shared_rank(&s.pub_min, r));
                gb |= *cluster.map_shared_rank(&s.pub_bad, r);
            }
            s.g_m = gm; s.g_min = gn; s.g_arg = ga; s.g_bad = gb;
        }
        __syncthreads();
    }
    const float m = s.g_m;
    const bool bad = s.g_bad != 0;

    RowStats st;
    st.m = m;
    st.lmin = s.g_min;
    st.argmax = s.g_arg;
    st.status = bad ? MTPV_ROW_NONFINITE : MTPV_ROW_OK;
    st.Z = 1.0;
    st.Zk = 1.0;
    st.lstar = -INFINITY;
    st.idxstar = INT_MAX;

    if (!bad && T > 0.0) {
        // ---------------- P2: exps, Z, level-1 histogram ----------------
        const double md = (double)m;
        const float range = __fsub_rn(m, s.g_min);
        float inv_w = (range > 0.0f) ? __fdiv_rn((float)kBins, range) : 0.0f;
        if (!isfinite(inv_w)) inv_w = 0.0f;
        if (!topp_all) {
            for (int b = tid; b < kBins; b += kThreads) { s.hist_mass[b] = 0.0; s.hist_cnt[b] = 0; }
            __syncthreads();
        }
        double zt = 0.0;
        {
            int cur = -1, ccnt = 0;
            double cacc = 0.0;
            for (int j = v0 + tid; j < v1; j += kThreads) {
                float l = L[j];
                double e = e_of(l, md, T);
                zt += e;
                if (!topp_all) {
                    int b = bin_of(l, m, inv_w);
                    if (b != cur) {
                        if (cur >= 0) { atomicAdd(&s.hist_mass[cur], cacc); atomicAdd(&s.hist_cnt[cur], ccnt); }
                        cur = b; cacc = 0.0; ccnt = 0;
                    }
                    cacc += e;
                    ++ccnt;
                }
            }
            if (cur >= 0) { atomicAdd(&s.hist_mass[cur], cacc); atomicAdd(&s.hist_cnt[cur], ccnt); }
        }
        double zc = block_sum_d(zt, s);
        if (tid == 0) { s.pub_Z = zc; s.cand_count = 0u; }
        cluster.sync();
        if (tid == 0) {
            double z = 0.0;
            for (int r = 0; r < C; ++r) z = __dadd_rn(z, *cluster.map_shared_rank(&s.pub_Z, r));
            s.g_Z = z;
        }
        __syncthreads();
        st.Z = s.g_Z;
        st.Zk = st.Z;

        if (!topp_all) {
            // ---------------- P3: crossing bin, exact cut ----------------
            const double thr = __dmul_rn((double)p.top_p, st.Z);
            const int per = kBins / C;
            const int base = rank * per;
            for (int b = tid; b < per; b += kThreads) {
                double ms = 0.0;
                int cn = 0;
                for (int r = 0; r < C; ++r) {
                    ms = __dadd_rn(ms, cluster.map_shared_rank(s.hist_mass, r)[base + b]);
                    cn += cluster.map_shared_rank(s.hist_cnt, r)[base + b];
                }
                s.own_mass[b] = ms;
                s.own_cnt[b] = cn;
            }
            __syncthreads();
            if (tid == 0) {
                double t = 0.0;
                for (int b = 0; b < per; ++b) t = __dadd_rn(t, s.own_mass[b]);
                s.pub_range_total = t;
            }
            cluster.sync();
            if (tid == 0) {
                // first range whose inclusive prefix reaches thr, then the bin
                double P = 0.0, Pstar = 0.0;
                int cstar = -1;
                for (int r = 0; r < C; ++r) {
                    double nxt = __dadd_rn(P, *cluster.map_shared_rank(&s.pub_range_total, r));
                    if (cstar < 0 && nxt >= thr) { cstar = r; Pstar = P; }
                    P = nxt;
                }
                if (cstar == rank) {
                    double loc = 0.0, A = Pstar;
                    int bstar = -1;
                    for (int b = 0; b < per; ++b) {
                        double nl = __dadd_rn(loc, s.own_mass[b]);
                        if (__dadd_rn(Pstar, nl) >= thr) { bstar = base + b; A = __dadd_rn(Pstar, loc); break; }
                        loc = nl;
                    }
                    if (bstar < 0) bstar = base + per - 1;  // unreachable: sums agree
                    const int cnt = s.own_cnt[bstar - base];
                    for (int r = 0; r < C; ++r) {
                        *cluster.map_shared_rank(&s.bc_bin, r) = bstar;
                        *cluster.map_shared_rank(&s.bc_cnt, r) = cnt;
                        *cluster.map_shared_rank(&s.bc_A, r) = A;
                    }
                } else if (cstar < 0 && rank == 0) {
                    // thr above the histogram total (top_p within rounding of 1): keep all
                    for (int r = 0; r < C; ++r) {
                        *cluster.map_shared_rank(&s.bc_bin, r) = -1;
                        *cluster.map_shared_rank(&s.bc_cnt, r) = 0;
                        *cluster.map_shared_rank(&s.bc_A, r) = P;
                    }
                }
            }
            cluster.sync();
            const int bstar = s.bc_bin;
            const int cnt = s.bc_cnt;
            const double A = s.bc_A;
            if (bstar < 0 || cnt == 0) {
                st.Zk = st.Z;  // nothing to cut (top_p within rounding of 1): keep all
            } else if (cnt <= kCandCap) {
                // gather the crossing bin's tokens into CTA 0
                unsigned int *cc = cluster.map_shared_rank(&s.cand_count, 0);
                unsigned long long *ck = cluster.map_shared_rank(s.cand, 0);
                for (int j = v0 + tid; j < v1; j += kThreads) {
                    float l = L[j];
                    if (bin_of(l, m, inv_w) == bstar) {
                        unsigned slot = atomicAdd(cc, 1u);
                        if (slot < (unsigned)kCandCap) ck[slot] = rank_key(l, j);
                    }
                }
                cluster.sync();
                if (rank == 0) {
                    const int n = min((int)s.cand_count, kCandCap);
                    int n2 = 1;
                    while (n2 < n) n2 <<= 1;
                    for (int i = n + tid; i < n2; i += kThreads) s.cand[i] = 0ull;
                    __syncthreads();
                    for (int k = 2; k <= n2; k <<= 1) {  // bitonic sort, descending
                        for (int jj = k >> 1; jj > 0; jj >>= 1) {
                            for (int i = tid; i < n2; i += kThreads) {
                                const int ix = i ^ jj;
                                if (ix > i) {
                                    unsigned long long a = s.cand[i], b = s.cand[ix];
                                    const bool desc = (i & k) == 0;
                                    if (desc ? (a < b) : (a > b)) { s.cand[i] = b; s.cand[ix] = a; }
                                }
                            }
                            __syncthreads();
                        }
                    }
                    for (int i = tid; i < n; i += kThreads) s.cand_e[i] = e_of(key_logit(s.cand[i]), md, T);
                    // exclusive prefix over the sorted candidates: sequential
                    // chunks per thread, thread totals scanned by warp 0
                    const int ch = (n + kThreads - 1) / kThreads;
                    const int i0 = min(n, tid * ch), i1 = min(n, i0 + ch);
                    __syncthreads();
                    double tt = 0.0;
                    for (int i = i0; i < i1; ++i) tt = __dadd_rn(tt, s.cand_e[i]);
                    s.thr_excl[tid] = tt;
                    if (tid == 0) s.first_fail = INT_MAX;
                    __syncthreads();
                    if (wid == 0) {
                        constexpr int per_lane = kThreads / 32;
                        double lt = 0.0;
                        for (int q = 0; q < per_lane; ++q) lt = __dadd_rn(lt, s.thr_excl[lane * per_lane + q]);
                        double inc = warp_incl_scan_d(lt);
                        double prev = __shfl_up_sync(0xffffffffu, inc, 1);
                        double acc = (lane == 0) ? 0.0 : prev;
                        for (int q = 0; q < per_lane; ++q) {
                            double v = s.thr_excl[lane * per_lane + q];
                            s.thr_excl[lane * per_lane + q] = acc;
                            acc = __dadd_rn(acc, v);
                        }
                    }
                    __syncthreads();
                    {
                        double ex = s.thr_excl[tid];
                        for (int i = i0; i < i1; ++i) {
                            if (__dadd_rn(A, ex) >= thr) { atomicMin(&s.first_fail, i); break; }
                            ex = __dadd_rn(ex, s.cand_e[i]);
                        }
                    }
                    __syncthreads();
                    int cut = (s.first_fail == INT_MAX) ? n - 1 : s.first_fail - 1;
                    if (cut < 0) cut = 0;  // A < thr by construction: the first is kept
                    if (cut >= i0 && cut < i1) {
                        double ex = s.thr_excl[tid];
                        for (int i = i0; i < cut; ++i) ex = __dadd_rn(ex, s.cand_e[i]);
                        s.cut_Zk = __dadd_rn(A, __dadd_rn(ex, s.cand_e[cut]));
                        s.cut_idx = key_index(s.cand[cut]);
                        s.cut_l = key_logit(s.cand[cut]);
                    }
                    __syncthreads();
                    st.Zk = s.cut_Zk;
                    st.idxstar = s.cut_idx;
                    st.lstar = s.cut_l;
                }
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
                            float l = L[j];
                            unsigned long long key = rank_key(l, j);
                            if ((key & mask) != prefix) continue;
                            const int d = (int)((key >> shift) & 255ull);
                            double e = e_of(l, md, T);
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
                            double nx = __dadd_rn(acc, s.own_mass[d]);
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
                st.Zk = __dadd_rn(above, e_of(st.lstar, md, T));
            }
        }
    }

    // publish the row statistics (CTA 0 of the cluster)
    if (rank == 0 && tid == 0) {
        p.stats[row] = st;
        __threadfence();
    }
    cluster.sync();

    if (!p.verify) {
        // ---------------- P4 (sample): draw from this row ----------------
        RowStats sr;
        sr.m = __ldcg(&p.stats[row].m);
        sr.Zk = __ldcg(&p.stats[row].Zk);
        sr.lstar = __ldcg(&p.stats[row].lstar);
        sr.idxstar = __ldcg(&p.stats[row].idxstar);
        sr.argmax = __ldcg(&p.stats[row].argmax);
        sr.status = __ldcg(&p.stats[row].status);
        if (sr.status != MTPV_ROW_OK) {
            if (rank == 0 && tid == 0) {
                p.out_tokens[row] = -1;
                if (p.row_status) p.row_status[row] = sr.status;
            }
        } else if (T == 0.0) {
            if (rank == 0 && tid == 0) {
                p.out_tokens[row] = sr.argmax;
                if (p.row_status) p.row_status[row] = MTPV_ROW_OK;
            }
        } else {
            cluster_draw(cluster, s, 0, false, sr, L, sr, L, T, p.u_samp[row], v0, v1, &p.out_tokens[row]);
            if (rank == 0 && tid == 0 && p.row_status) p.row_status[row] = MTPV_ROW_OK;
        }
        cluster.sync();
        return;
    }

    // ---------------- P4 (verify): the last cluster of the sequence ----------------
    const int S = 2 * p.K + 1;
    const int b = row / S;
    if (rank == 0 && tid == 0) {
        const unsigned old = atomicAdd(&p.counters[b], 1u);
        const int last = (old == (unsigned)(S - 1));
        for (int r = 0; r < C; ++r) *cluster.map_shared_rank(&s.bc_last, r) = last;
    }
    cluster.sync();
    if (!s.bc_last) {
        cluster.sync();
        return;
    }
    __threadfence();
    const int K = p.K;
    if (tid < S) {
        const RowStats *g = &p.stats[b * S + tid];
        RowStats r;
        r.Z = __ldcg(&g->Z);
        r.Zk = __ldcg(&g->Zk);
        r.m = __ldcg(&g->m);
        r.lmin = __ldcg(&g->lmin);
        r.lstar = __ldcg(&g->lstar);
        r.idxstar = __ldcg(&g->idxstar);
        r.argmax = __ldcg(&g->argmax);
        r.status = __ldcg(&g->status);
        s.st[tid] = r;
    }
    __syncthreads();
    const float *Lt0 = p.tl + (size_t)b * (K + 1) * V;
    const float *Ld0 = p.dl + (size_t)b * K * V;
    if (tid == 0) {
        int status = MTPV_ROW_OK;
        for (int i = 0; i < K; ++i) {
            const int d = p.drafts[b * K + i];
            if (d < 0 || d >= V) status = MTPV_ROW_BAD_DRAFT;
        }
        if (status == MTPV_ROW_OK)
            for (int i = 0; i < S; ++i)
                if (s.st[i].status != MTPV_ROW_OK) status = MTPV_ROW_NONFINITE;
        int n = K;
        if (status == MTPV_ROW_OK) {
            for (int i = 0; i < K; ++i) {
                const int d = p.drafts[b * K + i];
                const double pt = warped_prob(s.st[i], Lt0 + (size_t)i * V, d, T);
                const double qd = warped_prob(s.st[K + 1 + i], Ld0 + (size_t)i * V, d, T);
                const double r = (qd == 0.0) ? (pt > 0.0 ? INFINITY : 0.0) : pt / qd;
                if (!((double)p.u_acc[b * K + i] < r)) { n = i; break; }
            }
        }
        s.seq_n = n;
        s.seq_status = status;
    }
    __syncthreads();
    const int n = s.seq_n;
    const int status = s.seq_status;
    int32_t *ot = p.out_tokens + (size_t)b * (K + 1);
    if (status != MTPV_ROW_OK) {
        if (rank == 0 && tid <= K) ot[tid] = -1;
        if (rank == 0 && tid == 0) {
            p.out_acc[b] = -1;
            if (p.row_status) p.row_status[b] = status;
        }
    } else {
        if (rank == 0 && tid <= K) {
            if (tid < n) ot[tid] = p.drafts[b * K + tid];
            else if (tid > n) ot[tid] = -1;
        }
        if (rank == 0 && tid == 0) {
            p.out_acc[b] = n;
            if (p.row_status) p.row_status[b] = MTPV_ROW_OK;
        }
        if (T == 0.0) {
            if (rank == 0 && tid == 0) ot[n] = s.st[n].argmax;
        } else {
            const float *Lt = Lt0 + (size_t)n * V;
            const RowStats stt = s.st[n];
            if (n < K) {
                const RowStats std_ = s.st[K + 1 + n];
                cluster_draw(cluster, s, 1, true, stt, Lt, std_, Ld0 + (size_t)n * V, T,
                             p.u_samp[b * (K + 1) + n], v0, v1, &ot[n]);
            } else {
                cluster_draw(cluster, s, 0, false, stt, Lt, stt, Lt, T, p.u_samp[b * (K + 1) + n],
                             v0, v1, &ot[n]);
            }
        }
    }
    if (rank == 0 && tid == 0) p.counters[b] = 0u;
    cluster.sync();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t sampler_smem_bytes() { return sizeof(SamplerSmem); }

int sampler_cluster_size() {
    static int cached = 0;
    if (cached) return cached;
    const size_t smem = sizeof(SamplerSmem);
    cudaFuncSetAttribute(sampler_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(sampler_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    int best = 8;
    for (int c : {16, 8}) {
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
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, sampler_kernel, &cfg) == cudaSuccess &&
            nclusters > 0) {
            best = c;
            break;
        }
        cudaGetLastError();
    }
    cached = best;
    return best;
}

cudaError_t launch_sampler(const SamplerParams &p, int rows, cudaStream_t stream) {
    const int C = sampler_cluster_size();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, rows, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = sizeof(SamplerSmem);
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, sampler_kernel, p);
}

}  // namespace mtpv
