/*
 * csa_oracle.c -- plain, slow, fp64 CPU definition of one decode step of
 * combined sparse attention (pinned prefix + sliding window + Quest-style
 * top-k pages) over a paged GQA KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity oracle for the CUDA
 * library in long_context_decoding_b200/.  Only the tests, the smoke check
 * and the CPU-baseline leg of the benchmark may load it.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * Sources (titles of the pages this follows):
 *  - "Accelerating Long-Context Decoding in Large-Scale Hybrid LLMs Without
 *    Retraining", abstract: every full-attention layer attends to a sliding
 *    window of recent tokens, a pinned prefix and a fixed budget of the most
 *    relevant tokens of the context.
 *  - arxivlens analysis of the same paper, "Methodology": the budgeted tokens
 *    are picked by query-aware top-k selection (Quest).
 *  - roboaidigest post, "The Move" (Quest-style *paged* top-k) and "Why It
 *    Matters" (the KV cache stays full size, so any page can be selected).
 * The page score used for the top-k is the Quest upper bound
 *     s_h(p) = sum_i max(q_{h,i} * max_{p,i}, q_{h,i} * min_{p,i})
 * over the per-page, per-channel key minimum and maximum.
 *
 * Readings taken where the pages are silent:
 *  - GQA: the page score of a kv-head is the max over the query heads of its
 *    group of the per-head bound (keeps the bound valid for every head).
 *  - prefix and window are token-exact; a page is a top-k candidate unless
 *    every one of its valid tokens is already in prefix or window.
 *  - k = floor(budget / page_size) pages; all candidates when |C| <= k.
 *  - equal scores: the lower logical page index wins.
 *  - the softmax scale is an argument (callers pass 1/sqrt(D)).
 *  - metadata and scores cover valid tokens (t < seq_len) only.
 *
 * Layouts (all row-major, bf16 passed as raw uint16 bit patterns):
 *  q          [B][Hq][D]
 *  k_cache    [num_pages][Hkv][ps][D]      (same for v_cache)
 *  meta       [num_pages][Hkv][2][D]       (row 0 = min, row 1 = max)
 *  page_table [B][max_pages]               (logical page -> physical page)
 *  seq_lens   [B]
 *  query head h belongs to kv-head h / (Hq / Hkv).
 *
 * All functions return 0 on success and a negative number on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_EINVAL (-1)

/* bf16 bit pattern -> double (bf16 is the top half of an IEEE binary32). */
static double bf(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int dims_ok(const int *d)
{
    /* d = {B, Hq, Hkv, D, ps, max_pages, num_pages} */
    if (d[0] < 0 || d[1] <= 0 || d[2] <= 0 || d[3] <= 0 || d[4] <= 0 ||
        d[5] < 0 || d[6] < 0)
        return 0;
    if (d[1] % d[2] != 0)
        return 0;
    return 1;
}

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* Token ranges of one sequence: effective prefix Pe and window We, and the
 * candidate page range [c_lo, c_hi) (empty when prefix and window already
 * cover every token, i.e. Pe >= L - We).                                    */
static void ranges(int L, int prefix, int window, int ps, int *Pe, int *We,
                   int *c_lo, int *c_hi)
{
    int pe = prefix < L ? prefix : L;
    int we = window < L ? window : L;
    *Pe = pe;
    *We = we;
    if (pe < L - we) {
        *c_lo = pe / ps;                      /* page holding token Pe        */
        *c_hi = (L - we + ps - 1) / ps;       /* one past page of token L-We-1 */
    } else {
        *c_lo = 0;
        *c_hi = 0;
    }
}

/* Step 1 -- page metadata: per (physical page, kv-head, channel) the minimum
 * and maximum key over the valid tokens of the page, recomputed from the
 * cache.  Physical pages that the page table does not reach through a valid
 * token are left untouched.                                                 */
int oracle_meta(const int *d, const uint16_t *k_cache, const int32_t *page_table,
                const int32_t *seq_lens, uint16_t *meta)
{
    if (!dims_ok(d))
        return ORACLE_EINVAL;
    const int B = d[0], Hkv = d[2], D = d[3], ps = d[4], MP = d[5], NPG = d[6];
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        if (L < 0 || L > MP * ps)
            return ORACLE_EINVAL;
        int np = (L + ps - 1) / ps;
        for (int p = 0; p < np; ++p) {
            int phys = page_table[(size_t)b * MP + p];
            if (phys < 0 || phys >= NPG)
                return ORACLE_EINVAL;
            int ntok = L - p * ps < ps ? L - p * ps : ps;
            for (int g = 0; g < Hkv; ++g) {
                const uint16_t *kp = k_cache + (((size_t)phys * Hkv + g) * ps) * D;
                uint16_t *mn = meta + (((size_t)phys * Hkv + g) * 2 + 0) * D;
                uint16_t *mx = meta + (((size_t)phys * Hkv + g) * 2 + 1) * D;
                for (int i = 0; i < D; ++i) {
                    uint16_t lo = kp[i], hi = kp[i];
                    for (int t = 1; t < ntok; ++t) {
                        uint16_t v = kp[(size_t)t * D + i];
                        if (bf(v) < bf(lo))
                            lo = v;
                        if (bf(v) > bf(hi))
                            hi = v;
                    }
                    mn[i] = lo;
                    mx[i] = hi;
                }
            }
        }
    }
    return 0;
}

/* Steps 2-3 -- Quest page scores for the candidate pages of every
 * (sequence, kv-head).  Per page the min/max come straight from the cache
 * (the definition, not a stored summary).  scores [B][Hkv][max_pages]; pages
 * that are not candidates get NaN.                                          */
int oracle_scores(const int *d, const uint16_t *q, const uint16_t *k_cache,
                  const int32_t *page_table, const int32_t *seq_lens, int prefix,
                  int window, double *scores)
{
    if (!dims_ok(d) || prefix < 0 || window < 0)
        return ORACLE_EINVAL;
    const int B = d[0], Hq = d[1], Hkv = d[2], D = d[3], ps = d[4], MP = d[5],
              NPG = d[6];
    const int G = Hq / Hkv;
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 0 || seq_lens[b] > MP * ps)
            return ORACLE_EINVAL;
        int np = (seq_lens[b] + ps - 1) / ps;
        for (int p = 0; p < np; ++p) {
            int phys = page_table[(size_t)b * MP + p];
            if (phys < 0 || phys >= NPG)
                return ORACLE_EINVAL;
        }
    }
    const double nan = NAN;
    for (size_t i = 0; i < (size_t)B * Hkv * MP; ++i)
        scores[i] = nan;

    int units = B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < units; ++u) {
        int b = u / Hkv, g = u % Hkv;
        int L = seq_lens[b];
        int Pe, We, c_lo, c_hi;
        ranges(L, prefix, window, ps, &Pe, &We, &c_lo, &c_hi);
        double *mn = (double *)malloc(sizeof(double) * (size_t)D);
        double *mx = (double *)malloc(sizeof(double) * (size_t)D);
        for (int p = c_lo; p < c_hi; ++p) {
            int phys = page_table[(size_t)b * MP + p];
            int ntok = L - p * ps < ps ? L - p * ps : ps;
            const uint16_t *kp = k_cache + (((size_t)phys * Hkv + g) * ps) * D;
            for (int i = 0; i < D; ++i) {
                mn[i] = bf(kp[i]);
                mx[i] = mn[i];
                for (int t = 1; t < ntok; ++t) {
                    double v = bf(kp[(size_t)t * D + i]);
                    if (v < mn[i])
                        mn[i] = v;
                    if (v > mx[i])
                        mx[i] = v;
                }
            }
            double best = -INFINITY;
            for (int j = 0; j < G; ++j) {
                const uint16_t *qh = q + ((size_t)b * Hq + (size_t)g * G + j) * D;
                double s = 0.0;
                for (int i = 0; i < D; ++i) {
                    double qi = bf(qh[i]);
                    double a = qi * mx[i], c = qi * mn[i];
                    s += a > c ? a : c;
                }
                if (s > best)
                    best = s;
            }
            scores[((size_t)b * Hkv + g) * MP + p] = best;
        }
        free(mn);
        free(mx);
    }
    return 0;
}

typedef struct {
    double s;
    int p;
} scored_page;

/* descending score, then ascending page index */
static int by_score_then_index(const void *x, const void *y)
{
    const scored_page *a = (const scored_page *)x, *b = (const scored_page *)y;
    if (a->s > b->s)
        return -1;
    if (a->s < b->s)
        return 1;
    return (a->p > b->p) - (a->p < b->p);
}

static int ascending_int(const void *x, const void *y)
{
    int a = *(const int *)x, b = *(const int *)y;
    return (a > b) - (a < b);
}

/* Step 4 -- top-k pages: the first k' = min(floor(budget/ps), |C|)
 * candidates in the order (score descending, page ascending), returned in
 * ascending page order.  A full sort, not a selection algorithm.
 * scores are read as written by oracle_scores (NaN = not a candidate); any
 * other array of the same shape may be passed.  sel [B][Hkv][max_sel].     */
int oracle_select(const int *d, const double *scores, const int32_t *seq_lens,
                  int prefix, int window, int budget, int max_sel, int32_t *sel,
                  int32_t *nsel)
{
    if (!dims_ok(d) || prefix < 0 || window < 0 || budget < 0 || max_sel < 0)
        return ORACLE_EINVAL;
    const int B = d[0], Hkv = d[2], ps = d[4], MP = d[5];
    int k = budget / ps;
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        if (L < 0 || L > MP * ps)
            return ORACLE_EINVAL;
        int Pe, We, c_lo, c_hi;
        ranges(L, prefix, window, ps, &Pe, &We, &c_lo, &c_hi);
        int n = c_hi - c_lo;
        int kk = k < n ? k : n;
        if (kk > max_sel)
            return ORACLE_EINVAL;
        for (int g = 0; g < Hkv; ++g) {
            const double *sc = scores + ((size_t)b * Hkv + g) * MP;
            scored_page *cand = (scored_page *)malloc(sizeof(scored_page) * (size_t)(n > 0 ? n : 1));
            for (int i = 0; i < n; ++i) {
                cand[i].s = sc[c_lo + i];
                cand[i].p = c_lo + i;
            }
            qsort(cand, (size_t)n, sizeof(scored_page), by_score_then_index);
            int32_t *out = sel + ((size_t)b * Hkv + g) * max_sel;
            for (int i = 0; i < kk; ++i)
                out[i] = cand[i].p;
            qsort(out, (size_t)kk, sizeof(int32_t), ascending_int);
            nsel[b * Hkv + g] = kk;
            free(cand);
        }
    }
    return 0;
}

/* Step 5 -- the attended token set A of one (sequence, kv-head):
 * t < L and (t < Pe or t >= L - We or page(t) is selected).  With dense != 0
 * it is every t < L.  mask [B][Hkv][max_pages * ps], 1 = attended.         */
int oracle_token_mask(const int *d, const int32_t *seq_lens, int prefix, int window,
                      const int32_t *sel, const int32_t *nsel, int max_sel, int dense,
                      uint8_t *mask)
{
    if (!dims_ok(d) || prefix < 0 || window < 0 || max_sel < 0)
        return ORACLE_EINVAL;
    const int B = d[0], Hkv = d[2], ps = d[4], MP = d[5];
    const size_t T = (size_t)MP * ps;
    memset(mask, 0, (size_t)B * Hkv * T);
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        if (L < 0 || L > MP * ps)
            return ORACLE_EINVAL;
        int Pe = prefix < L ? prefix : L;
        int We = window < L ? window : L;
        for (int g = 0; g < Hkv; ++g) {
            uint8_t *m = mask + ((size_t)b * Hkv + g) * T;
            for (int t = 0; t < L; ++t)
                m[t] = (uint8_t)(dense || t < Pe || t >= L - We);
            if (dense)
                continue;
            int n = nsel[b * Hkv + g];
            if (n < 0 || n > max_sel)
                return ORACLE_EINVAL;
            const int32_t *s = sel + ((size_t)b * Hkv + g) * max_sel;
            for (int i = 0; i < n; ++i) {
                int p = s[i];
                if (p < 0 || p >= MP)
                    return ORACLE_EINVAL;
                for (int t = p * ps; t < (p + 1) * ps && t < L; ++t)
                    m[t] = 1;
            }
        }
    }
    return 0;
}

/* Step 6 -- softmax attention of every query head over its kv-head's set A:
 *   z_t = scale * q_h . k_t,  o_h = sum_t exp(z_t - max z) v_t / sum_t exp(z_t - max z)
 * and lse_h = max z + log(sum_t exp(z_t - max z)).  An empty set gives o = 0
 * and lse = -inf.  out [B][Hq][D], lse [B][Hq] (nullable).
 * dense != 0 attends to every valid token (the unmodified layer).          */
int oracle_attend(const int *d, const uint16_t *q, const uint16_t *k_cache,
                  const uint16_t *v_cache, const int32_t *page_table,
                  const int32_t *seq_lens, int prefix, int window, const int32_t *sel,
                  const int32_t *nsel, int max_sel, int dense, double scale, double *out,
                  double *lse)
{
    if (!dims_ok(d))
        return ORACLE_EINVAL;
    const int B = d[0], Hq = d[1], Hkv = d[2], D = d[3], ps = d[4], MP = d[5],
              NPG = d[6];
    const int G = Hq / Hkv;
    const size_t T = (size_t)MP * ps;
    uint8_t *mask = (uint8_t *)malloc((size_t)(B > 0 ? B : 1) * Hkv * (T > 0 ? T : 1));
    int rc = oracle_token_mask(d, seq_lens, prefix, window, sel, nsel, max_sel, dense, mask);
    if (rc != 0) {
        free(mask);
        return rc;
    }
    for (int b = 0; b < B; ++b) {
        int np = (seq_lens[b] + ps - 1) / ps;
        for (int p = 0; p < np; ++p) {
            int phys = page_table[(size_t)b * MP + p];
            if (phys < 0 || phys >= NPG) {
                free(mask);
                return ORACLE_EINVAL;
            }
        }
    }
    int heads = B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < heads; ++bh) {
        int b = bh / Hq, h = bh % Hq, g = h / G;
        int L = seq_lens[b];
        const uint8_t *m = mask + ((size_t)b * Hkv + g) * T;
        const uint16_t *qh = q + ((size_t)b * Hq + h) * D;
        double *z = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        double zmax = -INFINITY;
        for (int t = 0; t < L; ++t) {
            if (!m[t])
                continue;
            int phys = page_table[(size_t)b * MP + t / ps];
            const uint16_t *kt = k_cache + (((size_t)phys * Hkv + g) * ps + t % ps) * D;
            double dot = 0.0;
            for (int i = 0; i < D; ++i)
                dot += bf(qh[i]) * bf(kt[i]);
            z[t] = scale * dot;
            if (z[t] > zmax)
                zmax = z[t];
        }
        double *o = out + ((size_t)b * Hq + h) * D;
        for (int i = 0; i < D; ++i)
            o[i] = 0.0;
        double denom = 0.0;
        for (int t = 0; t < L; ++t) {
            if (!m[t])
                continue;
            double w = exp(z[t] - zmax);
            denom += w;
            int phys = page_table[(size_t)b * MP + t / ps];
            const uint16_t *vt = v_cache + (((size_t)phys * Hkv + g) * ps + t % ps) * D;
            for (int i = 0; i < D; ++i)
                o[i] += w * bf(vt[i]);
        }
        if (denom > 0.0) {
            for (int i = 0; i < D; ++i)
                o[i] /= denom;
        }
        if (lse)
            lse[(size_t)b * Hq + h] = denom > 0.0 ? zmax + log(denom) : -INFINITY;
        free(z);
    }
    free(mask);
    return 0;
}

/* ------------------------------------------------------------------------
 * fp8 page metadata (an optional variant of the scoring input, not a step of
 * the pages' method: a lower-precision copy of the exact bf16 min/max that
 * halves the bytes the scoring reads).  Each metadata row pair (the D minima
 * and D maxima of one physical page and kv-head) is stored as
 *     2*D bytes of OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7,
 *     3 mantissa bits; largest finite value 448; subnormals k * 2^-9)
 *     followed by a 16-byte trailer: int32 e, then 12 zero bytes,
 * and encodes min * 2^-e rounded toward -inf and max * 2^-e rounded toward
 * +inf, so the decoded box [2^e * min8, 2^e * max8] contains the exact one
 * and the Quest bound computed from it is still an upper bound for every
 * head.  e is the smallest integer with max_i |value_i| * 2^-e <= 448 over
 * the row pair (0 for an all-zero row pair).  Zero is encoded as 0x00.
 * ------------------------------------------------------------------------ */

/* Largest (up = 0) or smallest (up = 1) E4M3 value <= (>=) y, |y| <= 448.  */
static double fp8_round(double y, int up)
{
    if (y < 0.0)
        return -fp8_round(-y, !up);
    const double sub = ldexp(1.0, -9);     /* subnormal quantum             */
    double quantum;
    if (y < ldexp(1.0, -6)) {
        quantum = sub;
    } else {
        int ex;
        frexp(y, &ex);                     /* y = f * 2^ex, f in [0.5, 1)   */
        quantum = ldexp(1.0, ex - 1 - 3);  /* 3 mantissa bits below 2^(ex-1) */
    }
    double k = up ? ceil(y / quantum) : floor(y / quantum);
    return k * quantum;
}

/* E4M3 bit pattern of a value of the grid (zero -> 0x00).                  */
static uint8_t fp8_encode(double v)
{
    if (v == 0.0)
        return 0;
    uint8_t s = v < 0.0 ? 0x80 : 0x00;
    double a = fabs(v);
    if (a < ldexp(1.0, -6))
        return (uint8_t)(s | (uint8_t)(a / ldexp(1.0, -9)));
    int ex;
    frexp(a, &ex);
    int E = ex - 1;                        /* a = m * 2^(E-3), m in [8, 15] */
    int m = (int)(a / ldexp(1.0, E - 3));
    return (uint8_t)(s | (uint8_t)((E + 7) << 3) | (uint8_t)(m - 8));
}

/* Value of an E4M3 bit pattern (0x7f / 0xff, NaN, never occur here).        */
static double fp8_decode(uint8_t x)
{
    double sgn = (x & 0x80) ? -1.0 : 1.0;
    int E = (x >> 3) & 0xF, m = x & 7;
    if (E == 0)
        return sgn * ldexp((double)m, -9);
    return sgn * ldexp((double)(8 + m), E - 7 - 3);
}

/* Smallest e with a * 2^-e <= 448 (a = max |value| >= 0); 0 for a = 0.     */
static int fp8_row_exponent(double a)
{
    if (a == 0.0)
        return 0;
    int ex;
    double f = frexp(a, &ex);              /* a = f * 2^ex = (2f) * 2^(ex-1) */
    int k = ex - 1;
    return k - 8 + (2.0 * f > 1.75 ? 1 : 0);
}

/* Exported for the tests' pins.                                             */
double oracle_fp8_round(double y, int up) { return fp8_round(y, up); }
int oracle_fp8_encode(double v) { return fp8_encode(v); }
double oracle_fp8_decode(int x) { return fp8_decode((uint8_t)x); }
int oracle_fp8_row_exponent(double a) { return fp8_row_exponent(a); }

/* fp8 copy of the metadata of every physical page that a sequence reaches
 * through a valid token.  meta: [num_pages][Hkv][2][D] bf16 (exact min/max);
 * meta8: [num_pages][Hkv][2*D + 16] bytes; untouched pages keep their bytes. */
int oracle_meta_fp8(const int *d, const uint16_t *meta, const int32_t *page_table,
                    const int32_t *seq_lens, uint8_t *meta8)
{
    if (!dims_ok(d))
        return ORACLE_EINVAL;
    const int B = d[0], Hkv = d[2], D = d[3], ps = d[4], MP = d[5], NPG = d[6];
    const size_t row = (size_t)2 * D + 16;
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        if (L < 0 || L > MP * ps)
            return ORACLE_EINVAL;
        int np = (L + ps - 1) / ps;
        for (int p = 0; p < np; ++p) {
            int phys = page_table[(size_t)b * MP + p];
            if (phys < 0 || phys >= NPG)
                return ORACLE_EINVAL;
            for (int g = 0; g < Hkv; ++g) {
                const uint16_t *mn = meta + (((size_t)phys * Hkv + g) * 2 + 0) * D;
                const uint16_t *mx = meta + (((size_t)phys * Hkv + g) * 2 + 1) * D;
                uint8_t *out = meta8 + ((size_t)phys * Hkv + g) * row;
                double amax = 0.0;
                for (int i = 0; i < D; ++i) {
                    if (fabs(bf(mn[i])) > amax)
                        amax = fabs(bf(mn[i]));
                    if (fabs(bf(mx[i])) > amax)
                        amax = fabs(bf(mx[i]));
                }
                int e = fp8_row_exponent(amax);
                for (int i = 0; i < D; ++i) {
                    out[i] = fp8_encode(fp8_round(ldexp(bf(mn[i]), -e), 0));
                    out[D + i] = fp8_encode(fp8_round(ldexp(bf(mx[i]), -e), 1));
                }
                int32_t e32 = e;
                memcpy(out + 2 * D, &e32, 4);
                memset(out + 2 * D + 4, 0, 12);
            }
        }
    }
    return 0;
}

/* Quest scores from fp8 metadata (the stored box, decoded and scaled by 2^e):
 * same candidates, layout and NaN convention as oracle_scores.              */
int oracle_scores_fp8(const int *d, const uint16_t *q, const uint8_t *meta8,
                      const int32_t *page_table, const int32_t *seq_lens, int prefix,
                      int window, double *scores)
{
    if (!dims_ok(d) || prefix < 0 || window < 0)
        return ORACLE_EINVAL;
    const int B = d[0], Hq = d[1], Hkv = d[2], D = d[3], ps = d[4], MP = d[5],
              NPG = d[6];
    const int G = Hq / Hkv;
    const size_t row = (size_t)2 * D + 16;
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 0 || seq_lens[b] > MP * ps)
            return ORACLE_EINVAL;
        int np = (seq_lens[b] + ps - 1) / ps;
        for (int p = 0; p < np; ++p) {
            int phys = page_table[(size_t)b * MP + p];
            if (phys < 0 || phys >= NPG)
                return ORACLE_EINVAL;
        }
    }
    for (size_t i = 0; i < (size_t)B * Hkv * MP; ++i)
        scores[i] = NAN;
    int units = B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < units; ++u) {
        int b = u / Hkv, g = u % Hkv;
        int Pe, We, c_lo, c_hi;
        ranges(seq_lens[b], prefix, window, ps, &Pe, &We, &c_lo, &c_hi);
        for (int p = c_lo; p < c_hi; ++p) {
            int phys = page_table[(size_t)b * MP + p];
            const uint8_t *r = meta8 + ((size_t)phys * Hkv + g) * row;
            int32_t e;
            memcpy(&e, r + 2 * D, 4);
            double best = -INFINITY;
            for (int j = 0; j < G; ++j) {
                const uint16_t *qh = q + ((size_t)b * Hq + (size_t)g * G + j) * D;
                double s = 0.0;
                for (int i = 0; i < D; ++i) {
                    double qi = bf(qh[i]);
                    double lo = ldexp(fp8_decode(r[i]), e), hi = ldexp(fp8_decode(r[D + i]), e);
                    double a = qi * hi, c = qi * lo;
                    s += a > c ? a : c;
                }
                if (s > best)
                    best = s;
            }
            scores[((size_t)b * Hkv + g) * MP + p] = best;
        }
    }
    return 0;
}
