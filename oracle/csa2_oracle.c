/*
 * csa2_oracle.c -- plain, slow CPU oracle for the CSA2 FP4 sparse-decode
 * path. TEST INFRASTRUCTURE ONLY (see csa2_oracle.h for who may load it and
 * for the citation tags [INF], [NEO], [ZUL]).
 *
 * All arithmetic is fp64 or exact integers. Built with -ffp-contract=off and
 * no fast-math so that every fp64 operation is the IEEE operation written.
 *
 * The "omp parallel for" lines mark outer loops whose iterations are
 * independent (tokens, rows, heads): each iteration does the same operations
 * in the same order whichever thread runs it, so the OpenMP build (used only
 * to time the oracle on every host core) gives bit-identical results. The
 * test build ignores them.
 *
 * Parity status of each function (what pins it) is listed in the header of
 * tests/test_oracle_pins.py. The indexer formula itself is not printed on the
 * pages (parity unpinned: it is the DSA-style reading, see below).
 */
#include "csa2_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

double orc_bf16_value(uint16_t bits)
{
    /* bf16 is the upper half of an IEEE binary32. */
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E2M1 (OCP microscaling FP4): bit 3 sign, bits 2..1 exponent with bias 1,
 * bit 0 mantissa. Exponent field 0 is subnormal: value = m * 2^-1.
 * [NEO part 3] names the format; the value table follows from it. */
double orc_e2m1_value(uint8_t code)
{
    int sign = (code >> 3) & 1;
    int exp_field = (code >> 1) & 3;
    int mant = code & 1;
    double mag;
    if (exp_field == 0)
        mag = mant * 0.5;
    else
        mag = ldexp(1.0 + 0.5 * mant, exp_field - 1);
    return sign ? -mag : mag;
}

/* E4M3FN (OCP FP8): bit 7 sign, bits 6..3 exponent with bias 7, bits 2..0
 * mantissa. Exponent field 0 is subnormal (m/8 * 2^-6). Exponent 15 with
 * mantissa 7 is NaN; there are no infinities, so 448 is the largest value. */
double orc_e4m3_value(uint8_t byte)
{
    int sign = (byte >> 7) & 1;
    int exp_field = (byte >> 3) & 15;
    int mant = byte & 7;
    double mag;
    if (exp_field == 15 && mant == 7)
        return NAN;
    if (exp_field == 0)
        mag = ldexp(mant / 8.0, -6);
    else
        mag = ldexp(1.0 + mant / 8.0, exp_field - 7);
    return sign ? -mag : mag;
}

/* Encode a non-negative value that is exactly on the E4M3FN grid. */
static uint8_t e4m3_encode_exact(double v)
{
    if (v < ldexp(1.0, -6)) {
        /* subnormal: v = m * 2^-9 */
        return (uint8_t)(int)(v / ldexp(1.0, -9));
    }
    int e;
    frexp(v, &e);              /* v = f * 2^e, f in [0.5, 1) */
    int E = e - 1;             /* v = (1 + m/8) * 2^E */
    int mant = (int)((v / ldexp(1.0, E) - 1.0) * 8.0);
    return (uint8_t)(((E + 7) << 3) | mant);
}

/* ------------------------------------------------------------------------ */
/* Quantizer                                                                 */
/* ------------------------------------------------------------------------ */

/*
 * Scale of one 16-channel group. [NEO part 3] fixes only "one E4M3 scale per
 * 16 channels"; the reading taken is s = the E4M3FN value nearest to amax/6,
 * so that the largest magnitude lands on the top E2M1 magnitude 6.
 *
 * Method: textbook round-to-nearest-even onto the E4M3FN grid. In the binade
 * [2^E, 2^(E+1)) with E >= -6 the grid step is 2^(E-3); below 2^-6 the
 * subnormal step 2^-9 continues. t = amax/6 is formed in fp64; amax has at
 * most 8 significant bits and every E4M3 midpoint times 6 has at most 7, so
 * amax/6 is either exactly a midpoint or at least 2^-8 (relative) away from
 * one, far more than the 2^-53 fp64 rounding of t. Rounding t therefore
 * equals rounding the exact quotient.
 */
uint8_t orc_group_scale(double amax)
{
    double t = amax / 6.0;
    if (!(t > 0.0))
        return 0;
    if (t >= 448.0)
        return 0x7E;           /* saturate to the largest finite value */
    int e;
    frexp(t, &e);
    int E = e - 1;             /* t in [2^E, 2^(E+1)) */
    if (E < -6)
        E = -6;                /* subnormal range shares the 2^-9 step */
    double step = ldexp(1.0, E - 3);
    double n = nearbyint(t / step);   /* default mode: nearest, ties even */
    return e4m3_encode_exact(n * step);
}

/*
 * E2M1 code of x under scale s. Reading: |x|/s rounded to nearest on the E2M1
 * magnitude grid {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even code,
 * saturating at 6; negative sign only for a non-zero magnitude.
 *
 * Method: round-to-nearest-even onto the grid. For r = |x|/s in [2^E,
 * 2^(E+1)) with E >= 0 the step is 2^(E-1); below 1 the subnormal step 0.5
 * continues. Ties-to-even on the step count is ties-to-even-code because the
 * code's low bit is the mantissa bit. As for the scale, |x| has 8 significant
 * bits and s*midpoint at most 7, so r lies exactly on a midpoint or far from
 * it compared with the fp64 rounding of the quotient.
 */
uint8_t orc_e2m1_code(double x, double s)
{
    if (s == 0.0)
        return 0;
    double r = fabs(x) / s;
    double mag;
    if (r >= 6.0) {
        mag = 6.0;
    } else {
        int e;
        frexp(r, &e);
        int E = (r == 0.0) ? 0 : e - 1;
        if (E < 0)
            E = 0;
        double step = ldexp(1.0, E - 1);
        mag = nearbyint(r / step) * step;
    }
    uint8_t code;
    if (mag == 0.0) {
        code = 0;              /* canonical +0, also for negative x */
    } else if (mag == 0.5) {
        code = 1;              /* the one subnormal magnitude */
    } else {
        int e;
        frexp(mag, &e);
        int E = e - 1;                       /* 0, 1 or 2 */
        int mant = (mag / ldexp(1.0, E) == 1.5) ? 1 : 0;
        code = (uint8_t)(((E + 1) << 1) | mant);
    }
    if (code != 0 && x < 0.0)
        code |= 8;
    return code;
}

void orc_group_scale_n(const double *amax, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_group_scale(amax[i]);
}

void orc_e2m1_code_n(const double *x, const double *s, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_e2m1_code(x[i], s[i]);
}

void orc_quant_fp4(const uint16_t *x_bf16, int64_t n, int dim,
                   uint8_t *codes, uint8_t *scales)
{
    int groups = dim / 16;
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t *row = x_bf16 + t * dim;
        uint8_t *crow = codes + t * (dim / 2);
        uint8_t *srow = scales + t * groups;
        for (int g = 0; g < groups; ++g) {
            double amax = 0.0;
            for (int c = 0; c < 16; ++c) {
                double v = fabs(orc_bf16_value(row[g * 16 + c]));
                if (v > amax)
                    amax = v;
            }
            uint8_t sb = orc_group_scale(amax);
            double s = orc_e4m3_value(sb);
            srow[g] = sb;
            for (int c = 0; c < 16; c += 2) {
                int ch = g * 16 + c;
                uint8_t lo = orc_e2m1_code(orc_bf16_value(row[ch]), s);
                uint8_t hi = orc_e2m1_code(orc_bf16_value(row[ch + 1]), s);
                crow[ch / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

void orc_dequant_fp4(const uint8_t *codes, const uint8_t *scales, int64_t n,
                     int dim, double *out)
{
    int groups = dim / 16;
    for (int64_t t = 0; t < n; ++t) {
        for (int ch = 0; ch < dim; ++ch) {
            uint8_t byte = codes[t * (dim / 2) + ch / 2];
            uint8_t code = (ch & 1) ? (byte >> 4) : (byte & 15);
            double s = orc_e4m3_value(scales[t * groups + ch / 16]);
            out[t * dim + ch] = orc_e2m1_value(code) * s;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Indexer FP8 quantiser                                                     */
/* ------------------------------------------------------------------------ */

/*
 * E4M3FN code of the exact quotient x / sigma, for a finite x and a binary32
 * sigma > 0: the grid value nearest to x / sigma, ties to the even mantissa,
 * saturating at +-448 (the largest finite value: anything above it is
 * nearest to it), canonical +0 when the magnitude rounds to 0.
 *
 * The quotient itself is never formed, so nothing is rounded before the one
 * rounding onto the E4M3 grid. The grid values v_0 = 0 < v_1 < ... < v_126 =
 * 448 are the non-negative codes 0x00..0x7E in order. The nearest value is
 * found by comparing |x| with products v_i * sigma and with the midpoints
 * (v_i + v_(i+1)) / 2 * sigma: a grid value has at most 4 significant bits, a
 * midpoint at most 5, sigma at most 24, so every product is exact in fp64,
 * and every comparison below is an exact comparison of real numbers.
 */
uint8_t orc_e4m3_code_quotient(double x, float sigma)
{
    double a = fabs(x);
    double s = (double)sigma;
    /* i = the largest grid index with v_i * sigma <= |x| (v_0 = 0 always is) */
    int i = 0;
    while (i < 126 && orc_e4m3_value((uint8_t)(i + 1)) * s <= a)
        ++i;
    int code;
    if (i == 126) {
        code = 126;                               /* at or above 448: saturate */
    } else {
        double mid = 0.5 * (orc_e4m3_value((uint8_t)i) + orc_e4m3_value((uint8_t)(i + 1)));
        double ms = mid * s;
        if (a < ms)
            code = i;
        else if (a > ms)
            code = i + 1;
        else
            code = (i % 2 == 0) ? i : i + 1;      /* exact tie: even mantissa */
    }
    if (code == 0)
        return 0;
    return (x < 0.0) ? (uint8_t)(code | 0x80) : (uint8_t)code;
}

/*
 * Indexer key / query quantiser. [ZUL section 3] lists "indexer K / scale"
 * among the state a KV owner hands to its consumer layers, and [NEO part 2]
 * has the indexer read FP8 operands; the pages give no rule for the scale.
 * Reading: one binary32 scale per row of `dim` channels,
 *     sigma = the binary32 value nearest to amax / 448 (0 for an all-zero
 *             row), so that the row's largest magnitude lands on the top
 *             E4M3 value,
 * and code_c = the E4M3FN value nearest to the exact quotient x_c / sigma
 * (orc_e4m3_code_quotient: one rounding, ties to even, saturating, canonical
 * +0; all codes 0 when sigma = 0). The dequantised value is
 * sigma * e4m3(code).
 */
void orc_quant_index_fp8(const uint16_t *x_bf16, int64_t n_rows, int dim,
                         uint8_t *codes, float *sigma)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_rows; ++t) {
        const uint16_t *row = x_bf16 + t * dim;
        double amax = 0.0;
        for (int c = 0; c < dim; ++c) {
            double v = fabs(orc_bf16_value(row[c]));
            if (v > amax)
                amax = v;
        }
        /* amax is a bf16 value, exact in binary32; the IEEE binary32 division
         * rounds the exact quotient amax / 448 to nearest (even). */
        float sg = (float)amax / 448.0f;
        sigma[t] = sg;
        for (int c = 0; c < dim; ++c)
            codes[t * dim + c] = (sg == 0.0f) ? 0 : orc_e4m3_code_quotient(orc_bf16_value(row[c]), sg);
    }
}

/* ------------------------------------------------------------------------ */
/* Indexer                                                                   */
/* ------------------------------------------------------------------------ */

/*
 * The pages name a lightweight indexer with "indexer K / scale" owned by the
 * Full layer ([ZUL section 3]) and the DSA lineage, but print no formula.
 * Reading (parity unpinned): the DSA-style weighted sum of per-head ReLU dot
 * products, s_t = sum_h w_h * relu(sigma_t * <q_h, k_t>), with one shared
 * indexer key per token and a per-token scale sigma_t.
 *
 * Exactness: each E4M3 product has at most 8 significant bits and exponent in
 * [-18, 10]; a sum of 64 of them needs at most 42 bits, so the dot product is
 * exact in fp64. With sigma = 1 and power-of-two w (the workloads' inputs) the
 * score is exact too.
 */
void orc_indexer_scores(const uint8_t *q, const float *w, int n_heads,
                        int idim, const uint8_t *k, const float *sigma,
                        int64_t n, int relu, double *s)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        double score = 0.0;
        for (int h = 0; h < n_heads; ++h) {
            double dot = 0.0;
            for (int c = 0; c < idim; ++c)
                dot += orc_e4m3_value(q[h * idim + c]) *
                       orc_e4m3_value(k[t * idim + c]);
            double v = (double)sigma[t] * dot;
            if (relu && v < 0.0)
                v = 0.0;
            score += (double)w[h] * v;
        }
        s[t] = score;
    }
}

/* ------------------------------------------------------------------------ */
/* Top-k                                                                     */
/* ------------------------------------------------------------------------ */

typedef struct {
    double score;
    int32_t index;
} scored_t;

/* Order: higher score first; equal scores: lower index first. */
static int by_score_desc_index_asc(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->index > b->index) - (a->index < b->index);
}

static int by_int_asc(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * "Top-K sparse addressing index" ([NEO part 2]; [ZUL section 3]: Full and
 * Reindex layers run the selection). Reading: the k largest scores, ties to
 * the lower token index, returned in ascending token order, -1 padded.
 */
int orc_topk(const double *s, int64_t n_valid, int k, int32_t *out)
{
    if (k <= 0)
        return 0;
    if (n_valid <= k) {
        for (int i = 0; i < k; ++i)
            out[i] = (i < n_valid) ? i : -1;
        return (int)n_valid;
    }
    scored_t *all = (scored_t *)malloc((size_t)n_valid * sizeof *all);
    for (int64_t t = 0; t < n_valid; ++t) {
        all[t].score = s[t] + 0.0;   /* -0 and +0 are the same score */
        all[t].index = (int32_t)t;
    }
    qsort(all, (size_t)n_valid, sizeof *all, by_score_desc_index_asc);
    for (int i = 0; i < k; ++i)
        out[i] = all[i].index;
    free(all);
    qsort(out, (size_t)k, sizeof *out, by_int_asc);
    return k;
}

/*
 * Top-k inside a candidate pool ([NEO part 2]: the hierarchical sparse
 * indexer lets later indexing layers filter only within the candidate pool
 * built by the first Full layer, so their cost no longer grows with the
 * context). pool[i] is a token index (-1 entries are skipped) and s[i] its
 * score under the filtering layer's own indexer query. The k best pool
 * entries by (score desc, token index asc) are emitted in ascending token
 * order, -1 padded when the pool holds fewer than k valid entries. Reading:
 * the pool is the Full layer's top-C under its own scores (C >= k, a
 * parameter: the pages give no size).
 */
int orc_pool_topk(const double *s, const int32_t *pool, int n_pool, int k, int32_t *out)
{
    if (k <= 0)
        return 0;
    scored_t *all = (scored_t *)malloc((size_t)(n_pool > 0 ? n_pool : 1) * sizeof *all);
    int n = 0;
    for (int i = 0; i < n_pool; ++i) {
        if (pool[i] < 0)
            continue;
        all[n].score = s[i] + 0.0;
        all[n].index = pool[i];
        ++n;
    }
    qsort(all, (size_t)n, sizeof *all, by_score_desc_index_asc);
    int m = n < k ? n : k;
    for (int i = 0; i < m; ++i)
        out[i] = all[i].index;
    free(all);
    qsort(out, (size_t)m, sizeof *out, by_int_asc);
    for (int i = m; i < k; ++i)
        out[i] = -1;
    return m;
}

/* ------------------------------------------------------------------------ */
/* Sparse attention + sliding window                                         */
/* ------------------------------------------------------------------------ */

/*
 * One query token. Keys and values: the selected FP4 entries, dequantized
 * exactly, together with the SWA rows (bf16). Reading: the two sources are
 * different tensors ([ZUL section 4]: global compressed state and local SWA
 * state have separate lifetimes), so nothing is de-duplicated and one softmax
 * runs over their union. The same 576-channel vector serves as key and value.
 */
void orc_sparse_attn(const uint16_t *q, int n_heads, int dim,
                     const uint8_t *codes, const uint8_t *scales,
                     int64_t n_cache, const int32_t *idx, int k,
                     const uint16_t *swa, int n_swa, double softmax_scale,
                     double *o, double *lse)
{
    int n_keys = 0;
    for (int i = 0; i < k; ++i)
        if (idx[i] >= 0 && idx[i] < n_cache)
            ++n_keys;
    n_keys += n_swa;

    double *keys = (double *)malloc((size_t)(n_keys > 0 ? n_keys : 1) * dim * sizeof(double));
    int r = 0;
    for (int i = 0; i < k; ++i) {
        if (idx[i] < 0 || idx[i] >= n_cache)
            continue;
        orc_dequant_fp4(codes + (int64_t)idx[i] * (dim / 2),
                        scales + (int64_t)idx[i] * (dim / 16), 1, dim,
                        keys + (int64_t)r * dim);
        ++r;
    }
    for (int i = 0; i < n_swa; ++i, ++r)
        for (int c = 0; c < dim; ++c)
            keys[(int64_t)r * dim + c] = orc_bf16_value(swa[(int64_t)i * dim + c]);

    #pragma omp parallel for schedule(static)
    for (int h = 0; h < n_heads; ++h) {
        double *oh = o + (int64_t)h * dim;
        if (n_keys == 0) {
            for (int c = 0; c < dim; ++c)
                oh[c] = 0.0;
            lse[h] = -INFINITY;
            continue;
        }
        double *logit = (double *)malloc((size_t)n_keys * sizeof(double));
        double m = -INFINITY;
        for (int i = 0; i < n_keys; ++i) {
            double dot = 0.0;
            for (int c = 0; c < dim; ++c)
                dot += orc_bf16_value(q[(int64_t)h * dim + c]) * keys[(int64_t)i * dim + c];
            logit[i] = softmax_scale * dot;
            if (logit[i] > m)
                m = logit[i];
        }
        double l = 0.0;
        for (int c = 0; c < dim; ++c)
            oh[c] = 0.0;
        for (int i = 0; i < n_keys; ++i) {
            double p = exp(logit[i] - m);
            l += p;
            for (int c = 0; c < dim; ++c)
                oh[c] += p * keys[(int64_t)i * dim + c];
        }
        for (int c = 0; c < dim; ++c)
            oh[c] /= l;
        lse[h] = m + log(l);
        free(logit);
    }
    free(keys);
}

/* ------------------------------------------------------------------------ */
/* Static modes and ownership                                                */
/* ------------------------------------------------------------------------ */

/*
 * [ZUL section 3]: Full builds the compressed KV and indexer state and becomes
 * the physical cache owner; Reindex reuses the KV but recomputes the index;
 * Reuse reuses the KV and the existing top-K. [NEO part 2]: the main KV tensor
 * and indexer keys are shared across layers and top-K indices are reused.
 * Reading: every non-Full layer reads the KV of the nearest Full layer before
 * it, and a Reuse layer takes that Full layer's indices (even if a Reindex
 * layer sits between them).
 */
int orc_plan(const int *modes, int n_layers, int *kv_owner, int *index_src)
{
    int last_full = -1;
    for (int i = 0; i < n_layers; ++i) {
        switch (modes[i]) {
        case 0: /* Full */
            last_full = i;
            kv_owner[i] = i;
            index_src[i] = i;
            break;
        case 1: /* Reindex */
            if (last_full < 0)
                return -1 - i;
            kv_owner[i] = last_full;
            index_src[i] = i;
            break;
        case 2: /* Reuse */
            if (last_full < 0)
                return -1 - i;
            kv_owner[i] = last_full;
            index_src[i] = last_full;
            break;
        default:
            return -1 - i;
        }
    }
    return 0;
}
