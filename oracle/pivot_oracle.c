/*
 * pivot_oracle.c -- plain, slow, double-precision CPU oracle for the PIVOT
 * group-shared indexer.  TEST INFRASTRUCTURE ONLY: it exists so that tests,
 * the smoke check and the bench's CPU-baseline leg can check and time the
 * CUDA library.  Nothing on the product path may link or call it, and it
 * shares no source, header, table or helper with the CUDA code.
 *
 * What it follows ("PIVOT", picx.dev summary of the paper, section
 * "Introduction and Theoretical Foundation" and "Methodology"):
 *   Eq. (1)  I_{t,s} = sum_j w_{t,j} ReLU(q_{t,j} . k_s),  T_t = TopK(I_{t,:}, k)
 *   Eq. (2)  prefill groups of g contiguous query positions
 *   Eq. (3)  decode group = current token + (g-1) MTP drafts
 *   Eq. (4)  proxy = per-head mean of q and of w over the group
 *   Eq. (5)  proxy score over the causal prefix
 *   Eq. (6)  PIVOT-Reuse: every member takes the proxy top-k under its own mask
 *   Eq. (7)  PIVOT-Refine candidates C = proxy top-c (c = 2k)
 *   Eq. (8)  member re-scoring over C
 *   Eq. (9)  member top-k over C
 *
 * Readings taken where the pages are silent (each one is also listed in the
 * design notes of the repository):
 *   - the proxy scans s <= e (the group's last position); each member t then
 *     masks s <= t.  This is the only reading under which Refine with c >= L
 *     equals the dense indexer.
 *   - the pooled query mean is rounded to nearest-even to the input dtype
 *     (bf16 or fp32) because that is the operand the scan multiplies; the
 *     pooled w stays in double.                     -> parity unpinned (a convention)
 *   - TopK order: larger score first; equal scores -> lower key index first.
 *     In double, -0.0 == +0.0, so signed zeros tie and fall to the index.
 *   - rows hold min(k, |eligible|) indices; the rest of the row is -1.
 *   - decode: sequence b holds P_b keys, its g members are positions
 *     P_b-g .. P_b-1 (current token, then drafts).  -> parity unpinned (a convention)
 *   - proxy aggregation (PIVOT paper, Ablation Studies, "Proxy aggregation
 *     (Table 2)": mean pooling against a first- or last-query proxy): the
 *     first- / last-query proxy is the pooling of that one member row (q as
 *     is, since rounding a value of the input dtype is exact; its w).
 *     Selected with orc_set_aggregation (0 mean, the default; 1 first; 2 last).
 *
 * Arithmetic: every score is accumulated in double from the exact values of
 * the bf16 / fp32 inputs.  Sorting is a full qsort per row (brute force).
 * OpenMP parallelises over independent rows / groups only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes of q and k: 0 = bf16 bit patterns (uint16), 1 = fp32 */
#define ORC_BF16 0
#define ORC_F32 1

/* ---------------------------------------------------------------- values */

/* Exact value of element i of a bf16 or fp32 array, as a double. */
static double orc_elem(const void *p, int dtype, int64_t i)
{
    if (dtype == ORC_BF16) {
        uint16_t h = ((const uint16_t *)p)[i];
        uint32_t u = (uint32_t)h << 16;
        float f;
        memcpy(&f, &u, 4);
        return (double)f;
    }
    return (double)((const float *)p)[i];
}

/* Round a double to the nearest bf16 value, ties to even (the rounding of
 * the pooled proxy, see the header).  Works on the exact double: frexp gives
 * x = m * 2^e with 0.5 <= |m| < 1; bf16 keeps 8 significant bits. */
static double orc_round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x))
        return x;
    int e;
    double m = frexp(x, &e);
    /* bf16 min normal is 2^-126 = 0.5 * 2^-125; below it the spacing is fixed 2^-133 */
    if (e < -125) {
        double q = ldexp(1.0, -133);
        return rint(x / q) * q; /* rint: round half to even in the default mode */
    }
    double r = rint(ldexp(m, 8)); /* 8 significant bits */
    return ldexp(r, e - 8);
}

static double orc_round_dtype(double x, int dtype)
{
    if (dtype == ORC_BF16)
        return orc_round_bf16(x);
    return (double)(float)x; /* C conversion double->float rounds to nearest even */
}

/* ---------------------------------------------------------------- scores */

/* Widen query row `row` of q [*, H, d] and w [*, H] to double. */
void orc_query_row(const void *q, const float *w, int dtype, int H, int d,
                   int64_t row, double *qv, double *wv)
{
    for (int j = 0; j < H; j++) {
        for (int x = 0; x < d; x++)
            qv[j * d + x] = orc_elem(q, dtype, (row * H + j) * (int64_t)d + x);
        wv[j] = (double)w[row * H + j];
    }
}

/* Proxy aggregation: 0 = mean of the members (Eq. 4), 1 = the first member's
 * query, 2 = the last member's.  Read by the calls below; set between calls. */
static int g_orc_agg = 0;
void orc_set_aggregation(int mode) { g_orc_agg = (mode >= 0 && mode <= 2) ? mode : 0; }

/* The member rows the proxy pools: all of them, or the first / last one. */
static const int64_t *orc_agg_rows(const int64_t *rows, int *nrows)
{
    if (g_orc_agg == 1) { *nrows = 1; return rows; }
    if (g_orc_agg == 2) { const int64_t *r = rows + (*nrows - 1); *nrows = 1; return r; }
    return rows;
}

/* Eq. (4): proxy = per-head mean over the member rows (listed in `rows`).
 * q-bar is rounded to the input dtype (reading above), w-bar stays double. */
void orc_proxy(const void *q, const float *w, int dtype, int H, int d,
               const int64_t *rows, int nrows, double *qbar, double *wbar)
{
    for (int j = 0; j < H; j++) {
        for (int x = 0; x < d; x++) {
            double s = 0.0;
            for (int r = 0; r < nrows; r++)
                s += orc_elem(q, dtype, (rows[r] * H + j) * (int64_t)d + x);
            qbar[j * d + x] = orc_round_dtype(s / (double)nrows, dtype);
        }
        double sw = 0.0;
        for (int r = 0; r < nrows; r++)
            sw += (double)w[rows[r] * H + j];
        wbar[j] = sw / (double)nrows;
    }
}

/* Eq. (1) / (5) / (8): score of one (query or proxy) against key k_s.
 * k is [*, d]; key row s.  The key row is widened to double first. */
static double orc_score_one(const double *qv, const double *wv, int H, int d,
                            const void *k, int dtype, int64_t s)
{
    double kr[1024];
    for (int x = 0; x < d; x++)
        kr[x] = orc_elem(k, dtype, s * (int64_t)d + x);
    double total = 0.0;
    for (int j = 0; j < H; j++) {
        double dot = 0.0;
        for (int x = 0; x < d; x++)
            dot += qv[j * d + x] * kr[x];
        double relu = dot > 0.0 ? dot : 0.0;
        total += wv[j] * relu;
    }
    return total;
}

/* Scores against n keys given by row numbers keys[i] (or keys key_lo+i when
 * keys == NULL). */
void orc_scores(const double *qv, const double *wv, int H, int d,
                const void *k, int dtype, const int64_t *keys, int64_t key_lo,
                int64_t n, double *out)
{
    for (int64_t i = 0; i < n; i++) {
        int64_t s = keys ? keys[i] : key_lo + i;
        out[i] = orc_score_one(qv, wv, H, d, k, dtype, s);
    }
}

/* Scores of n vectors (qv [n, H*d], wv [n, H]) against key rows, in parallel
 * over the vectors; out is [n, m].  Vector r reads keys from row
 * key_base[r] (0 when key_base == NULL) onward.  With key_rows ([n, m]) entry
 * i is the score against key key_rows[r*m+i] (NaN where that is < 0);
 * otherwise entry s < plen[r] is the score against key s (NaN beyond). */
void orc_scores_batch(const double *qv, const double *wv, int64_t n, int H, int d,
                      const void *k, int dtype, const int64_t *key_base,
                      const int64_t *key_rows, const int64_t *plen, int64_t m,
                      double *out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; r++) {
        int64_t base = key_base ? key_base[r] : 0;
        const double *q = qv + r * (int64_t)H * d;
        const double *w = wv + r * (int64_t)H;
        for (int64_t i = 0; i < m; i++) {
            int64_t s = key_rows ? key_rows[r * m + i] : i;
            int ok = key_rows ? (s >= 0) : (i < plen[r]);
            out[r * m + i] = ok ? orc_score_one(q, w, H, d, k, dtype, base + s) : NAN;
        }
    }
}

/* ---------------------------------------------------------------- TopK */

typedef struct {
    double v;
    int64_t idx;
} orc_pair;

/* larger score first; equal scores: lower index first */
static int orc_cmp(const void *a, const void *b)
{
    const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    if (x->idx < y->idx) return -1;
    if (x->idx > y->idx) return 1;
    return 0;
}

/* TopK by full sort: f[i] is the score of key index idx[i] (idx == NULL means
 * idx[i] = i).  Writes the first min(n, m) key indices in rank order to
 * out_idx (and their scores to out_val when non-NULL); returns that count. */
int64_t orc_topn(const double *f, const int64_t *idx, int64_t m, int64_t n,
                 int64_t *out_idx, double *out_val)
{
    orc_pair *p = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)(m > 0 ? m : 1));
    for (int64_t i = 0; i < m; i++) {
        p[i].v = f[i];
        p[i].idx = idx ? idx[i] : i;
    }
    qsort(p, (size_t)m, sizeof(orc_pair), orc_cmp);
    int64_t cnt = n < m ? n : m;
    for (int64_t i = 0; i < cnt; i++) {
        out_idx[i] = p[i].idx;
        if (out_val)
            out_val[i] = p[i].v;
    }
    free(p);
    return cnt;
}

/* write one output row: cnt indices, padded with -1 up to topk */
static void orc_write_row(int32_t *row_idx, double *row_val, int topk,
                          const int64_t *sel, const double *sel_val, int64_t cnt)
{
    for (int i = 0; i < topk; i++) {
        if (i < cnt) {
            row_idx[i] = (int32_t)sel[i];
            if (row_val) row_val[i] = sel_val[i];
        } else {
            row_idx[i] = -1;
            if (row_val) row_val[i] = NAN;
        }
    }
}

/* ---------------------------------------------------------------- methods */

/* Eq. (1): dense indexer for query rows t in [t0, t1) of a sequence of L
 * positions.  out_idx / out_val are [(t1 - t0), topk]; out_val may be NULL. */
void orc_dense(const void *q, const float *w, const void *k, int dtype,
               int64_t L, int H, int d, int topk, int64_t t0, int64_t t1,
               int32_t *out_idx, double *out_val)
{
    (void)L;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = t0; t < t1; t++) {
        double *qv = (double *)malloc(sizeof(double) * (size_t)H * d);
        double *wv = (double *)malloc(sizeof(double) * (size_t)H);
        double *f = (double *)malloc(sizeof(double) * (size_t)(t + 1));
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)topk);
        double *selv = (double *)malloc(sizeof(double) * (size_t)topk);
        orc_query_row(q, w, dtype, H, d, t, qv, wv);
        orc_scores(qv, wv, H, d, k, dtype, NULL, 0, t + 1, f); /* s <= t */
        int64_t cnt = orc_topn(f, NULL, t + 1, topk, sel, selv);
        orc_write_row(out_idx + (t - t0) * topk, out_val ? out_val + (t - t0) * topk : NULL,
                      topk, sel, selv, cnt);
        free(qv); free(wv); free(f); free(sel); free(selv);
    }
}

/* Eq. (2): members of prefill group i are [i*g, min(i*g + g, L)). */
static int orc_group_rows(int64_t L, int g, int64_t i, int64_t *rows)
{
    int n = 0;
    for (int64_t t = i * g; t < i * g + g && t < L; t++)
        rows[n++] = t;
    return n;
}

/* Proxy scores (Eq. 4 + 5) of prefill group i over its prefix s <= e_i.
 * out has e_i + 1 entries; returns e_i + 1. */
int64_t orc_proxy_scores(const void *q, const float *w, const void *k, int dtype,
                         int64_t L, int H, int d, int g, int64_t i, double *out)
{
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)g);
    int n = orc_group_rows(L, g, i, rows);
    double *qb = (double *)malloc(sizeof(double) * (size_t)H * d);
    double *wb = (double *)malloc(sizeof(double) * (size_t)H);
    int na = n;
    const int64_t *ar = orc_agg_rows(rows, &na);
    orc_proxy(q, w, dtype, H, d, ar, na, qb, wb);
    int64_t P = rows[n - 1] + 1;
    orc_scores(qb, wb, H, d, k, dtype, NULL, 0, P, out);
    free(rows); free(qb); free(wb);
    return P;
}

/* Eq. (6): PIVOT-Reuse for prefill groups [g0, g1).  Each member t sorts the
 * proxy scores over s <= t directly (no shortcut).  Output rows are the
 * member positions [g0*g, min(g1*g, L)) -> out_idx [(rows), topk]. */
void orc_reuse(const void *q, const float *w, const void *k, int dtype,
               int64_t L, int H, int d, int topk, int g, int64_t g0, int64_t g1,
               int32_t *out_idx, double *out_val)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = g0; i < g1; i++) {
        int64_t e = (i * g + g < L ? i * g + g : L) - 1;
        double *pf = (double *)malloc(sizeof(double) * (size_t)(e + 1));
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)topk);
        double *selv = (double *)malloc(sizeof(double) * (size_t)topk);
        orc_proxy_scores(q, w, k, dtype, L, H, d, g, i, pf);
        for (int64_t t = i * g; t <= e; t++) {
            int64_t cnt = orc_topn(pf, NULL, t + 1, topk, sel, selv); /* s <= t */
            int64_t r = t - g0 * (int64_t)g;
            orc_write_row(out_idx + r * topk, out_val ? out_val + r * topk : NULL,
                          topk, sel, selv, cnt);
        }
        free(pf); free(sel); free(selv);
    }
}

/* Eq. (7)-(9): PIVOT-Refine for prefill groups [g0, g1).
 * cand_in (may be NULL): [(g1-g0), c] int32, -1 padded; when given, these sets
 * replace the oracle's own C_i (used to check member rows against the GPU's
 * candidate set).  out_cand / out_cand_val (may be NULL): the oracle's C_i in
 * rank order, [(g1-g0), c].  Member rows as in orc_reuse. */
void orc_refine(const void *q, const float *w, const void *k, int dtype,
                int64_t L, int H, int d, int topk, int c, int g,
                int64_t g0, int64_t g1, const int32_t *cand_in,
                int32_t *out_idx, double *out_val,
                int32_t *out_cand, double *out_cand_val)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = g0; i < g1; i++) {
        int64_t e = (i * g + g < L ? i * g + g : L) - 1;
        int64_t P = e + 1;
        int64_t *cand = (int64_t *)malloc(sizeof(int64_t) * (size_t)(c > 0 ? c : 1));
        double *candv = (double *)malloc(sizeof(double) * (size_t)(c > 0 ? c : 1));
        int64_t nc = 0;
        if (cand_in) {
            const int32_t *ci = cand_in + (i - g0) * c;
            for (int x = 0; x < c; x++)
                if (ci[x] >= 0) cand[nc++] = ci[x];
        } else {
            double *pf = (double *)malloc(sizeof(double) * (size_t)P);
            orc_proxy_scores(q, w, k, dtype, L, H, d, g, i, pf);
            nc = orc_topn(pf, NULL, P, c, cand, candv); /* Eq. (7) over s <= e */
            free(pf);
        }
        if (out_cand) {
            int32_t *oc = out_cand + (i - g0) * c;
            for (int x = 0; x < c; x++) {
                oc[x] = x < nc ? (int32_t)cand[x] : -1;
                if (out_cand_val)
                    out_cand_val[(i - g0) * c + x] = (x < nc && !cand_in) ? candv[x] : NAN;
            }
        }
        double *qv = (double *)malloc(sizeof(double) * (size_t)H * d);
        double *wv = (double *)malloc(sizeof(double) * (size_t)H);
        double *f = (double *)malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1));
        int64_t *el = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nc > 0 ? nc : 1));
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)topk);
        double *selv = (double *)malloc(sizeof(double) * (size_t)topk);
        for (int64_t t = i * g; t <= e; t++) {
            orc_query_row(q, w, dtype, H, d, t, qv, wv);
            int64_t m = 0;
            for (int64_t x = 0; x < nc; x++)
                if (cand[x] <= t) el[m++] = cand[x]; /* causal mask per member */
            orc_scores(qv, wv, H, d, k, dtype, el, 0, m, f); /* Eq. (8) */
            int64_t cnt = orc_topn(f, el, m, topk, sel, selv); /* Eq. (9) */
            int64_t r = t - g0 * (int64_t)g;
            orc_write_row(out_idx + r * topk, out_val ? out_val + r * topk : NULL,
                          topk, sel, selv, cnt);
        }
        free(qv); free(wv); free(f); free(el); free(sel); free(selv);
        free(cand); free(candv);
    }
}

/* Eq. (3) decode: sequence b has P_b = off[b+1]-off[b] cached keys stored at
 * rows off[b].. of k_cache [sum P_b, d]; its g query rows are q rows
 * b*g .. b*g+g-1 (current token first, then drafts) at positions
 * P_b-g .. P_b-1.  variant 0 = Reuse, 1 = Refine.  Sequences [b0, b1).
 * out_idx [(b1-b0)*g, topk]; cand arrays [(b1-b0), c] as in orc_refine.
 * Index values are positions local to the sequence. */
void orc_decode(const void *q, const float *w, const void *kc, const int64_t *off,
                int dtype, int H, int d, int topk, int c, int g, int variant,
                int64_t b0, int64_t b1, const int32_t *cand_in,
                int32_t *out_idx, double *out_val,
                int32_t *out_cand, double *out_cand_val)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = b0; b < b1; b++) {
        int64_t P = off[b + 1] - off[b];
        const void *kb = (dtype == ORC_BF16)
                             ? (const void *)((const uint16_t *)kc + off[b] * d)
                             : (const void *)((const float *)kc + off[b] * d);
        int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)g);
        for (int r = 0; r < g; r++) rows[r] = b * g + r;
        double *qb = (double *)malloc(sizeof(double) * (size_t)H * d);
        double *wb = (double *)malloc(sizeof(double) * (size_t)H);
        double *pf = (double *)malloc(sizeof(double) * (size_t)P);
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * (size_t)(topk > c ? topk : c));
        double *selv = (double *)malloc(sizeof(double) * (size_t)(topk > c ? topk : c));
        int need_proxy = (variant == 0) || (cand_in == NULL);
        if (need_proxy) {
            int na = g;
            const int64_t *ar = orc_agg_rows(rows, &na);
            orc_proxy(q, w, dtype, H, d, ar, na, qb, wb);
            orc_scores(qb, wb, H, d, kb, dtype, NULL, 0, P, pf); /* s <= P_b - 1 */
        }
        if (variant == 0) {
            for (int r = 0; r < g; r++) {
                int64_t t = P - g + r;
                int64_t cnt = orc_topn(pf, NULL, t + 1, topk, sel, selv);
                int64_t orow = (b - b0) * g + r;
                orc_write_row(out_idx + orow * topk, out_val ? out_val + orow * topk : NULL,
                              topk, sel, selv, cnt);
            }
        } else {
            int64_t *cand = (int64_t *)malloc(sizeof(int64_t) * (size_t)c);
            double *candv = (double *)malloc(sizeof(double) * (size_t)c);
            int64_t nc = 0;
            if (cand_in) {
                const int32_t *ci = cand_in + (b - b0) * c;
                for (int x = 0; x < c; x++)
                    if (ci[x] >= 0) cand[nc++] = ci[x];
            } else {
                nc = orc_topn(pf, NULL, P, c, cand, candv);
            }
            if (out_cand) {
                int32_t *oc = out_cand + (b - b0) * c;
                for (int x = 0; x < c; x++) {
                    oc[x] = x < nc ? (int32_t)cand[x] : -1;
                    if (out_cand_val)
                        out_cand_val[(b - b0) * c + x] = (x < nc && !cand_in) ? candv[x] : NAN;
                }
            }
            double *qv = (double *)malloc(sizeof(double) * (size_t)H * d);
            double *wv = (double *)malloc(sizeof(double) * (size_t)H);
            double *f = (double *)malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1));
            int64_t *el = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nc > 0 ? nc : 1));
            for (int r = 0; r < g; r++) {
                int64_t t = P - g + r;
                orc_query_row(q, w, dtype, H, d, b * g + r, qv, wv);
                int64_t m = 0;
                for (int64_t x = 0; x < nc; x++)
                    if (cand[x] <= t) el[m++] = cand[x];
                orc_scores(qv, wv, H, d, kb, dtype, el, 0, m, f);
                int64_t cnt = orc_topn(f, el, m, topk, sel, selv);
                int64_t orow = (b - b0) * g + r;
                orc_write_row(out_idx + orow * topk, out_val ? out_val + orow * topk : NULL,
                              topk, sel, selv, cnt);
            }
            free(qv); free(wv); free(f); free(el); free(cand); free(candv);
        }
        free(rows); free(qb); free(wb); free(pf); free(sel); free(selv);
    }
}

/* Threads the OpenMP loops above will use (1 without OpenMP). */
int orc_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
