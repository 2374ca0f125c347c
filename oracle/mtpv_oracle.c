/*
 * mtpv_oracle.c -- plain, slow CPU oracle for the speculative-decoding verify
 * step.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call it; the library never does.  It shares
 * no code, header, table or helper with the CUDA path.
 *
 * What it computes, and where the pages say so:
 *   - LM-head projection of K+1 target rows through the bf16 head and of K
 *     draft rows through the draft-only 4-bit head (hazakura.dev MTPLX notes,
 *     "4-layer architecture", Layer 0: small-M shader, 4-bit draft LM head;
 *     devtrends.cc MTPLX overview: one forward pass verifies the whole batch).
 *   - Temperature softmax and top-p truncation of every row, applied alike to
 *     target and draft rows (devtrends.cc overview and devtrends.ru page:
 *     temperature=0.6, top_p=0.95 give the same distribution as sampling
 *     without MTP).
 *   - Leviathan-Chen rejection sampling with residual correction and a bonus
 *     token (devtrends.cc overview; hazakura.dev notes, Layer 2 cycle
 *     "draft -> parallel verify -> probability-ratio acceptance -> residual
 *     correction -> bonus token").
 * Precision: every sum, exp and ratio is fp64; inputs are bf16 / fp32 values
 * widened exactly.  The pages give no formula; where they stop, the readings
 * below are the textbook speculative-sampling rules:
 *   warp      p_j = exp((l_j - m)/T) / sum_i exp((l_i - m)/T), m = max l.
 *             T == 0: one-hot at the argmax (lowest index among equal maxima).
 *   top-p     order tokens by (logit desc, index asc); rank r is kept iff the
 *             probability mass of the ranks before it is < top_p (rank 0 is
 *             always kept); top_p >= 1 keeps every token with p > 0; kept
 *             probabilities are renormalised by their own sum.
 *   accept    draft d at position i is accepted iff u_acc[i] < r, with
 *             r = p'(d)/q'(d); r = +inf if q'(d) == 0 < p'(d); r = 0 if both
 *             are 0.  (u < 1, so u < r is the same test as u < min(1, r).)
 *   residual  at the first rejected position n: w = max(0, p'_n - q'_n); if
 *             sum w == 0 (p' == q'), w = p'_n.
 *   bonus     all K accepted: w = p'_K.
 *   draw      x = min{k : sum_{j<=k} w_j > u_samp[n] * sum w}, scanning in
 *             vocabulary-index order; if rounding leaves no such k, x is the
 *             last index with w > 0.
 *   outputs   tokens d_0..d_{n-1}, x, then -1 padding; accepted count n.
 *
 * Boundary flags (cases where a result may legitimately differ from an
 * implementation with different rounding): the acceptance uniform within
 * 1e-5 of r; the draw target within 1e-5 * w_x of an edge of the chosen bin;
 * a top-p cut within 1e-5 of the cut token's own mass AND the outcome changes
 * when that cut moves by one token.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define MTPVO_FLAG_RATIO 1
#define MTPVO_FLAG_DRAW 2
#define MTPVO_FLAG_TOPP 4
#define MTPVO_WINDOW 1e-5

/* ------------------------------------------------------------------ */
/* number formats                                                       */
/* ------------------------------------------------------------------ */
static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static uint16_t bf16_round_nearest_even(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)(u >> 16); /* inf/nan */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* target logits  y[m][n] = sum_k x[m][k] * W[n][k]                     */
/* ------------------------------------------------------------------ */
void mtpvo_lm_head_bf16(const uint16_t *x, int M, int Kd, int N, const uint16_t *W,
                        double *y, int n_begin, int n_end) {
    double *row = (double *)malloc(sizeof(double) * (size_t)Kd);
    double *xs = (double *)malloc(sizeof(double) * (size_t)M * (size_t)Kd);
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < Kd; ++k) xs[(size_t)m * Kd + k] = bf16_value(x[(size_t)m * Kd + k]);
    for (int n = n_begin; n < n_end; ++n) {
        for (int k = 0; k < Kd; ++k) row[k] = bf16_value(W[(size_t)n * Kd + k]);
        for (int m = 0; m < M; ++m) {
            double acc = 0.0;
            const double *xm = xs + (size_t)m * Kd;
            for (int k = 0; k < Kd; ++k) acc += xm[k] * row[k];
            y[(size_t)m * N + n] = acc;
        }
    }
    free(row);
    free(xs);
}

/* ------------------------------------------------------------------ */
/* draft logits through the int4 group-64 head.                         */
/* The stored nibble n of weight k of row v dequantises to              */
/* S[v][k/64] * (n - 8); y[m][v] = sum_k x[m][k] * deq(v, k).           */
/* ------------------------------------------------------------------ */
static int nibble_at(const uint8_t *rowbytes, int k) {
    uint8_t b = rowbytes[k >> 1];
    return (k & 1) ? (b >> 4) : (b & 0x0f);
}

void mtpvo_lm_head_int4g64(const uint16_t *x, int M, int Kd, int N, const uint8_t *Wq,
                           const uint16_t *S, double *y, int n_begin, int n_end) {
    const int G = Kd / 64;
    double *row = (double *)malloc(sizeof(double) * (size_t)Kd);
    double *xs = (double *)malloc(sizeof(double) * (size_t)M * (size_t)Kd);
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < Kd; ++k) xs[(size_t)m * Kd + k] = bf16_value(x[(size_t)m * Kd + k]);
    for (int n = n_begin; n < n_end; ++n) {
        const uint8_t *rb = Wq + (size_t)n * (Kd / 2);
        for (int k = 0; k < Kd; ++k) {
            double s = bf16_value(S[(size_t)n * G + k / 64]);
            row[k] = s * (double)(nibble_at(rb, k) - 8);
        }
        for (int m = 0; m < M; ++m) {
            double acc = 0.0;
            const double *xm = xs + (size_t)m * Kd;
            for (int k = 0; k < Kd; ++k) acc += xm[k] * row[k];
            y[(size_t)m * N + n] = acc;
        }
    }
    free(row);
    free(xs);
}

/* Independent restatement of the int4 group-64 storage format, used only to
 * cross-check the input generator byte for byte. */
void mtpvo_quantize_int4g64(const uint16_t *W, int N, int Kd, uint8_t *Wq, uint16_t *S) {
    const int G = Kd / 64;
    for (int n = 0; n < N; ++n) {
        for (int g = 0; g < G; ++g) {
            float amax = 0.0f;
            for (int j = 0; j < 64; ++j) {
                float a = fabsf((float)bf16_value(W[(size_t)n * Kd + g * 64 + j]));
                if (a > amax) amax = a;
            }
            uint16_t sb = bf16_round_nearest_even(amax / 7.0f);
            S[(size_t)n * G + g] = sb;
            float s = (float)bf16_value(sb);
            for (int j = 0; j < 64; ++j) {
                int k = g * 64 + j;
                int q = 0;
                if (s > 0.0f) {
                    float r = (float)bf16_value(W[(size_t)n * Kd + k]) / s;
                    q = (int)nearbyintf(r); /* default rounding: ties to even */
                    if (q > 7) q = 7;
                    if (q < -7) q = -7;
                }
                int nib = q + 8;
                uint8_t *b = Wq + (size_t)n * (Kd / 2) + (k >> 1);
                if (k & 1) *b = (uint8_t)((*b & 0x0f) | (nib << 4));
                else       *b = (uint8_t)((*b & 0xf0) | nib);
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* temperature softmax and top-p truncation of one row.                 */
/* ------------------------------------------------------------------ */
typedef struct {
    double m;        /* max logit                                   */
    double Z;        /* sum of exp((l - m)/T) over the whole row    */
    double kept_sum; /* sum of p over kept tokens                    */
    int kept;        /* number of kept tokens                        */
    int cut_token;   /* last kept token in (logit desc, idx asc)     */
    int next_token;  /* first dropped token (-1 if none)             */
    double gap_lo;   /* top_p - mass before the cut token            */
    double gap_hi;   /* mass up to and including the cut - top_p     */
    double p_cut, p_next;
} warp_info;

typedef struct {
    double l;
    int idx;
} ranked;

static int by_logit_desc_index_asc(const void *a, const void *b) {
    const ranked *x = (const ranked *)a, *y = (const ranked *)b;
    if (x->l > y->l) return -1;
    if (x->l < y->l) return 1;
    return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

/* Fills p_out (length V) with the warped distribution p'.  force_kept > 0
 * keeps exactly that many ranks (used to evaluate the alternative top-p cut
 * of an ambiguous row).  Returns 0, or 2 when a logit is not finite. */
static int warp_row(const double *l, int V, double T, double top_p, int force_kept,
                    double *p_out, warp_info *info) {
    memset(info, 0, sizeof *info);
    info->cut_token = -1;
    info->next_token = -1;
    if (V <= 0) return 3;
    for (int j = 0; j < V; ++j)
        if (!isfinite(l[j])) return 2;
    int am = 0;
    for (int j = 1; j < V; ++j)
        if (l[j] > l[am]) am = j;
    info->m = l[am];
    if (T == 0.0) { /* greedy: one-hot at the argmax */
        for (int j = 0; j < V; ++j) p_out[j] = 0.0;
        p_out[am] = 1.0;
        info->Z = 1.0;
        info->kept_sum = 1.0;
        info->kept = 1;
        info->cut_token = am;
        info->gap_lo = info->gap_hi = INFINITY;
        return 0;
    }
    double Z = 0.0;
    for (int j = 0; j < V; ++j) {
        p_out[j] = exp((l[j] - info->m) / T);
        Z += p_out[j];
    }
    info->Z = Z;
    for (int j = 0; j < V; ++j) p_out[j] = p_out[j] / Z;

    ranked *rk = (ranked *)malloc(sizeof(ranked) * (size_t)V);
    int *order = (int *)malloc(sizeof(int) * (size_t)V);
    unsigned char *keep = (unsigned char *)calloc((size_t)V, 1);
    for (int j = 0; j < V; ++j) {
        rk[j].l = l[j];
        rk[j].idx = j;
    }
    qsort(rk, (size_t)V, sizeof(ranked), by_logit_desc_index_asc);
    for (int r = 0; r < V; ++r) order[r] = rk[r].idx;
    free(rk);

    int kept = 0;
    double before_cut = 0.0, mass = 0.0;
    if (top_p >= 1.0 && force_kept <= 0) {
        for (int j = 0; j < V; ++j)
            if (p_out[j] > 0.0) keep[j] = 1;
        for (int r = 0; r < V; ++r)
            if (p_out[order[r]] > 0.0) kept = r + 1;
        info->gap_lo = info->gap_hi = INFINITY;
        if (kept > 0) info->cut_token = order[kept - 1];
        info->next_token = kept < V ? order[kept] : -1;
    } else {
        for (int r = 0; r < V; ++r) {
            int keep_r = force_kept > 0 ? (r < force_kept) : (mass < top_p);
            if (!keep_r) break;
            keep[order[r]] = 1;
            before_cut = mass;
            mass += p_out[order[r]];
            kept = r + 1;
        }
        info->cut_token = order[kept - 1];
        info->next_token = kept < V ? order[kept] : -1;
        info->p_cut = p_out[info->cut_token];
        info->p_next = info->next_token >= 0 ? p_out[info->next_token] : 0.0;
        info->gap_lo = (kept > 1) ? top_p - before_cut : INFINITY;
        info->gap_hi = (kept < V) ? mass - top_p : INFINITY;
    }
    double ks = 0.0;
    for (int j = 0; j < V; ++j)
        if (keep[j]) ks += p_out[j];
    for (int j = 0; j < V; ++j) p_out[j] = keep[j] ? p_out[j] / ks : 0.0;
    info->kept_sum = ks;
    info->kept = kept;
    free(order);
    free(keep);
    return 0;
}

/* Public single-row warp (for tests). info_out: m, Z, kept_sum, kept,
 * cut_token, next_token, gap_lo, gap_hi, p_cut, p_next. */
int mtpvo_warp(const double *l, int V, double T, double top_p, double *p_out, double *info_out) {
    warp_info wi;
    int st = warp_row(l, V, T, top_p, 0, p_out, &wi);
    if (info_out) {
        info_out[0] = wi.m;
        info_out[1] = wi.Z;
        info_out[2] = wi.kept_sum;
        info_out[3] = wi.kept;
        info_out[4] = wi.cut_token;
        info_out[5] = wi.next_token;
        info_out[6] = wi.gap_lo;
        info_out[7] = wi.gap_hi;
        info_out[8] = wi.p_cut;
        info_out[9] = wi.p_next;
    }
    return st;
}

/* ------------------------------------------------------------------ */
/* residual / bonus draw: inverse CDF in vocabulary-index order         */
/* ------------------------------------------------------------------ */
static int draw(const double *w, int V, double u, double *margin_rel) {
    double total = 0.0;
    for (int j = 0; j < V; ++j) total += w[j];
    double target = u * total;
    double c = 0.0;
    for (int j = 0; j < V; ++j) {
        double prev = c;
        c += w[j];
        if (c > target) {
            if (margin_rel) {
                double lo = target - prev, hi = c - target;
                *margin_rel = (lo < hi ? lo : hi) / w[j];
            }
            return j;
        }
    }
    int last = -1;
    for (int j = 0; j < V; ++j)
        if (w[j] > 0.0) last = j;
    if (margin_rel) *margin_rel = 0.0;
    return last;
}

int mtpvo_draw(const double *w, int V, double u, double *margin_rel) {
    return draw(w, V, u, margin_rel);
}

/* ------------------------------------------------------------------ */
/* acceptance, residual, bonus and outputs of one sequence, given its   */
/* warped rows.                                                         */
/* P: K+1 rows of p', Q: K rows of q' (each V long).                    */
/* ------------------------------------------------------------------ */
typedef struct {
    int n;            /* accepted drafts                      */
    int x;            /* residual or bonus token               */
    int flags;        /* MTPVO_FLAG_RATIO | MTPVO_FLAG_DRAW    */
    double ratio_margin, draw_margin;
} outcome;

static double accept_ratio(double p, double q) {
    if (q == 0.0) return p > 0.0 ? INFINITY : 0.0;
    return p / q;
}

static void decide(const double *P, const double *Q, const int32_t *d, const float *u_acc,
                   const float *u_samp, int K, int V, double *wbuf, outcome *o) {
    o->flags = 0;
    o->ratio_margin = INFINITY;
    o->draw_margin = INFINITY;
    int n = K;
    for (int i = 0; i < K; ++i) {
        double r = accept_ratio(P[(size_t)i * V + d[i]], Q[(size_t)i * V + d[i]]);
        double u = (double)u_acc[i];
        double gap = fabs(u - r);
        /* r == 0 (p'(d) == 0) and r == inf (q'(d) == 0) are decided by the
         * kept sets, not by rounding of the ratio. */
        if (isfinite(r) && r > 0.0 && gap < o->ratio_margin) o->ratio_margin = gap;
        if (isfinite(r) && r > 0.0 && gap < MTPVO_WINDOW) o->flags |= MTPVO_FLAG_RATIO;
        if (!(u < r)) { n = i; break; }
    }
    const double *w;
    if (n < K) {
        const double *p = P + (size_t)n * V, *q = Q + (size_t)n * V;
        double sw = 0.0;
        for (int j = 0; j < V; ++j) {
            double v = p[j] - q[j];
            wbuf[j] = v > 0.0 ? v : 0.0;
            sw += wbuf[j];
        }
        w = (sw == 0.0) ? p : wbuf;
    } else {
        w = P + (size_t)K * V;
    }
    double mr = 0.0;
    o->n = n;
    o->x = draw(w, V, (double)u_samp[n], &mr);
    o->draw_margin = mr;
    if (mr < MTPVO_WINDOW) o->flags |= MTPVO_FLAG_DRAW;
}

/* ------------------------------------------------------------------ */
/* Sampling mode: B sequences.                                          */
/*   tl [B][K+1][V], dl [B][K][V] logits (fp64), drafts [B][K],          */
/*   u_acc [B][K], u_samp [B][K+1].                                      */
/*   out_tokens [B][K+1], out_accepted [B], row_status [B],              */
/*   flags [B] (MTPVO_FLAG_*), margins [B][3] (ratio, draw, topp).       */
/* row_status: 0 ok, 1 draft id outside [0,V), 2 non-finite logit.       */
/* ------------------------------------------------------------------ */
void mtpvo_verify(const double *tl, const double *dl, const int32_t *drafts, const float *u_acc,
                  const float *u_samp, int B, int K, int V, double T, double top_p,
                  int32_t *out_tokens, int32_t *out_accepted, int32_t *row_status,
                  int32_t *flags, double *margins) {
    double *P = (double *)malloc(sizeof(double) * (size_t)(K + 1) * V);
    double *Q = (double *)malloc(sizeof(double) * (size_t)K * V);
    double *P2 = (double *)malloc(sizeof(double) * (size_t)(K + 1) * V);
    double *Q2 = (double *)malloc(sizeof(double) * (size_t)K * V);
    double *wbuf = (double *)malloc(sizeof(double) * (size_t)V);
    warp_info *pi = (warp_info *)malloc(sizeof(warp_info) * (size_t)(2 * K + 1));
    for (int b = 0; b < B; ++b) {
        const double *tlb = tl + (size_t)b * (K + 1) * V;
        const double *dlb = dl + (size_t)b * K * V;
        const int32_t *db = drafts + (size_t)b * K;
        int32_t *ot = out_tokens + (size_t)b * (K + 1);
        for (int i = 0; i <= K; ++i) ot[i] = -1;
        out_accepted[b] = -1;
        flags[b] = 0;
        int st = 0;
        for (int i = 0; i < K; ++i)
            if (db[i] < 0 || db[i] >= V) st = 1;
        for (int i = 0; i <= K && !st; ++i)
            if (warp_row(tlb + (size_t)i * V, V, T, top_p, 0, P + (size_t)i * V, &pi[i])) st = 2;
        for (int i = 0; i < K && !st; ++i)
            if (warp_row(dlb + (size_t)i * V, V, T, top_p, 0, Q + (size_t)i * V, &pi[K + 1 + i])) st = 2;
        row_status[b] = st;
        if (st) continue;

        outcome o;
        decide(P, Q, db, u_acc + (size_t)b * K, u_samp + (size_t)b * (K + 1), K, V, wbuf, &o);
        out_accepted[b] = o.n;
        for (int i = 0; i < o.n; ++i) ot[i] = db[i];
        ot[o.n] = o.x;
        flags[b] = o.flags;

        /* Top-p ambiguity: move each near-tie cut by one token and see whether
         * the outcome changes. */
        double topp_margin = INFINITY;
        if (T > 0.0 && top_p < 1.0) {
            for (int r = 0; r < 2 * K + 1; ++r) {
                warp_info *w = &pi[r];
                int alts[2], na = 0;
                if (w->gap_lo < MTPVO_WINDOW * w->p_cut) alts[na++] = w->kept - 1;
                if (w->gap_hi < MTPVO_WINDOW * w->p_next) alts[na++] = w->kept + 1;
                double rel_lo = w->p_cut > 0 ? w->gap_lo / w->p_cut : INFINITY;
                double rel_hi = w->p_next > 0 ? w->gap_hi / w->p_next : INFINITY;
                if (rel_lo < topp_margin) topp_margin = rel_lo;
                if (rel_hi < topp_margin) topp_margin = rel_hi;
                for (int a = 0; a < na; ++a) {
                    memcpy(P2, P, sizeof(double) * (size_t)(K + 1) * V);
                    memcpy(Q2, Q, sizeof(double) * (size_t)K * V);
                    warp_info tmp;
                    if (r <= K)
                        warp_row(tlb + (size_t)r * V, V, T, top_p, alts[a], P2 + (size_t)r * V, &tmp);
                    else
                        warp_row(dlb + (size_t)(r - K - 1) * V, V, T, top_p, alts[a],
                                 Q2 + (size_t)(r - K - 1) * V, &tmp);
                    outcome o2;
                    decide(P2, Q2, db, u_acc + (size_t)b * K, u_samp + (size_t)b * (K + 1), K, V,
                           wbuf, &o2);
                    if (o2.n != o.n || o2.x != o.x) flags[b] |= MTPVO_FLAG_TOPP;
                }
            }
        }
        if (margins) {
            margins[(size_t)b * 3 + 0] = o.ratio_margin;
            margins[(size_t)b * 3 + 1] = o.draw_margin;
            margins[(size_t)b * 3 + 2] = topp_margin;
        }
    }
    free(P); free(Q); free(P2); free(Q2); free(wbuf); free(pi);
}

/* ------------------------------------------------------------------ */
/* Distribution mode for one sequence: acceptance probabilities         */
/* acc[i] = min(1, p'_i(d_i)/q'_i(d_i)), residual distributions         */
/* res[i][:] = normalise(max(0, p'_i - q'_i)) (p'_i if that is all 0)   */
/* and the bonus distribution p'_K.  Returns row status.                */
/* ------------------------------------------------------------------ */
int mtpvo_verify_dist(const double *tl, const double *dl, const int32_t *d, int K, int V,
                      double T, double top_p, double *acc, double *res, double *bonus) {
    double *P = (double *)malloc(sizeof(double) * (size_t)(K + 1) * V);
    double *Q = (double *)malloc(sizeof(double) * (size_t)K * V);
    warp_info wi;
    int st = 0;
    for (int i = 0; i < K; ++i)
        if (d[i] < 0 || d[i] >= V) st = 1;
    for (int i = 0; i <= K && !st; ++i)
        if (warp_row(tl + (size_t)i * V, V, T, top_p, 0, P + (size_t)i * V, &wi)) st = 2;
    for (int i = 0; i < K && !st; ++i)
        if (warp_row(dl + (size_t)i * V, V, T, top_p, 0, Q + (size_t)i * V, &wi)) st = 2;
    if (!st) {
        for (int i = 0; i < K; ++i) {
            double r = accept_ratio(P[(size_t)i * V + d[i]], Q[(size_t)i * V + d[i]]);
            acc[i] = r < 1.0 ? r : 1.0;
            double *ri = res + (size_t)i * V;
            const double *p = P + (size_t)i * V, *q = Q + (size_t)i * V;
            double sw = 0.0;
            for (int j = 0; j < V; ++j) {
                double v = p[j] - q[j];
                ri[j] = v > 0.0 ? v : 0.0;
                sw += ri[j];
            }
            for (int j = 0; j < V; ++j) ri[j] = (sw == 0.0) ? p[j] : ri[j] / sw;
        }
        memcpy(bonus, P + (size_t)K * V, sizeof(double) * (size_t)V);
    }
    free(P);
    free(Q);
    return st;
}

/* ------------------------------------------------------------------ */
/* One sample from the warped distribution of each row (draft sampling). */
/* ------------------------------------------------------------------ */
void mtpvo_sample_rows(const double *l, int R, int V, double T, double top_p, const float *u,
                       int32_t *out, double *margin_rel, int32_t *row_status) {
    double *p = (double *)malloc(sizeof(double) * (size_t)V);
    warp_info wi;
    for (int r = 0; r < R; ++r) {
        int st = warp_row(l + (size_t)r * V, V, T, top_p, 0, p, &wi);
        if (row_status) row_status[r] = st;
        if (st) { out[r] = -1; continue; }
        double mr = 0.0;
        out[r] = draw(p, V, (double)u[r], &mr);
        if (margin_rel) margin_rel[r] = mr;
    }
    free(p);
}
