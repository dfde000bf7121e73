/*
 * csa2_oracle.c -- plain, slow, single-threaded CPU oracle for the CSA2
 * sparse FP4-KV decode path. TEST INFRASTRUCTURE: see csa2_oracle.h for the
 * sources, the rules on who may call it, and the readings it takes.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math
 * (oracle/build.py). Nothing here is blocked, fused or reordered: each
 * function is the definition written out.
 */
#include "csa2_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* [OCP-MX] FP4 E2M1: exponent bias 1; exponent field 0 is subnormal with
 * value m * 2^(1-1) / 2; otherwise 2^(e-1) * (1 + m/2). */
double orc_e2m1_value(uint32_t code) {
    uint32_t s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* [OCP-FP8] E4M3: bias 7; exponent field 0 is subnormal with value
 * 2^-6 * m/8; S.1111.111 is NaN; no infinities. */
double orc_e4m3_value(uint32_t byte) {
    uint32_t s = (byte >> 7) & 1u, e = (byte >> 3) & 15u, m = byte & 7u;
    double mag;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* Round |x| onto the grid of a minifloat binade by binade. The spacing of
 * representable values in the binade [2^E, 2^(E+1)) is 2^(E - mbits); below
 * the smallest normal binade emin the spacing stays 2^(emin - mbits). a/q is
 * exact in double (a has 24 significant bits, q is a power of two) and
 * nearbyint() rounds it to the nearest integer with ties to even, which is
 * ties to the even mantissa because the integer is 2^mbits + mantissa. */
static double round_to_minifloat_grid(double a, int emin, int mbits) {
    int e2;
    if (a == 0.0) return 0.0;
    (void)frexp(a, &e2);      /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;           /* a in [2^E, 2^(E+1)) */
    if (E < emin) E = emin;
    double q = ldexp(1.0, E - mbits);
    return nearbyint(a / q) * q;
}

uint32_t orc_e4m3_rne_sat(float xf) {
    double x = (double)xf;
    uint32_t sign = signbit(x) ? 0x80u : 0u;
    double a = fabs(x);
    if (isnan(a)) return sign | 0x7Fu;
    if (a >= 448.0) return sign | 0x7Eu;             /* satfinite */
    double v = round_to_minifloat_grid(a, -6, 3);     /* v <= 448 here */
    if (v == 0.0) return sign;
    if (v < ldexp(1.0, -6)) {                         /* subnormal: m * 2^-9 */
        return sign | (uint32_t)(v / ldexp(1.0, -9));
    }
    int e2;
    (void)frexp(v, &e2);
    int E = e2 - 1;
    uint32_t m = (uint32_t)(v / ldexp(1.0, E - 3)) - 8u;
    return sign | ((uint32_t)(E + 7) << 3) | m;
}

uint32_t orc_e2m1_rne_sat(float yf) {
    double y = (double)yf;
    uint32_t sign = signbit(y) ? 8u : 0u;
    double a = fabs(y);
    if (isnan(a)) return sign;
    if (a >= 6.0) return sign | 7u;                   /* satfinite */
    double v = round_to_minifloat_grid(a, 0, 1);      /* v <= 6 here */
    if (v == 0.0) return sign;
    if (v < 1.0) return sign | 1u;                    /* only subnormal: 0.5 */
    int e2;
    (void)frexp(v, &e2);
    int E = e2 - 1;
    uint32_t m = (uint32_t)(v / ldexp(1.0, E - 1)) - 2u;
    return sign | ((uint32_t)(E + 1) << 1) | m;
}

/* ------------------------------------------------------------------------ */
/* FP4 quantise + append                                                     */
/* ------------------------------------------------------------------------ */

static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

void orc_quantize_block16(const uint16_t *x_bf16, uint8_t *packed8, uint8_t *scale) {
    float x[16];
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        x[i] = bf16_to_float(x_bf16[i]);
        float a = fabsf(x[i]);
        if (a > amax) amax = a;                       /* NaN never compares greater */
    }
    volatile float t = amax / 6.0f;                   /* binary32 division */
    uint32_t s = orc_e4m3_rne_sat(t);
    float sd = (float)orc_e4m3_value(s);              /* exact in binary32 */
    uint32_t c[16];
    for (int i = 0; i < 16; ++i) {
        if (sd == 0.0f) {
            c[i] = 0u;
        } else {
            volatile float y = x[i] / sd;             /* binary32 division */
            c[i] = orc_e2m1_rne_sat(y);
        }
    }
    for (int j = 0; j < 8; ++j) packed8[j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
    *scale = (uint8_t)s;
}

void orc_quantize_row(const uint16_t *x_bf16, int32_t d, uint8_t *codes, uint8_t *scales) {
    for (int32_t b = 0; b < d / 16; ++b)
        orc_quantize_block16(x_bf16 + 16 * b, codes + 8 * b, scales + b);
}

int64_t orc_physical_row(const int32_t *page_table_seq, int32_t page_size, int64_t t) {
    return (int64_t)page_table_seq[t / page_size] * page_size + t % page_size;
}

void orc_append_fp4(const uint16_t *x_bf16, int32_t n, int32_t d,
                    const int32_t *seq, const int64_t *pos,
                    const int32_t *page_table, int32_t max_pages, int32_t page_size,
                    uint8_t *codes, uint8_t *scales) {
    for (int32_t i = 0; i < n; ++i) {
        int64_t row = orc_physical_row(page_table + (int64_t)seq[i] * max_pages, page_size, pos[i]);
        orc_quantize_row(x_bf16 + (int64_t)i * d, d,
                         codes + row * (d / 2), scales + row * (d / 16));
    }
}

void orc_e4m3_row(const uint16_t *x_bf16, int32_t width, uint8_t *out) {
    for (int32_t i = 0; i < width; ++i) out[i] = (uint8_t)orc_e4m3_rne_sat(bf16_to_float(x_bf16[i]));
}

void orc_append_swa_e4m3(const uint16_t *x_bf16, int32_t n, const int32_t *seq, const int64_t *pos,
                         int64_t ring_rows, uint8_t *swa) {
    for (int32_t i = 0; i < n; ++i) {
        int64_t slot = pos[i] % ring_rows;
        orc_e4m3_row(x_bf16 + (int64_t)i * 512, 512, swa + ((int64_t)seq[i] * ring_rows + slot) * 512);
    }
}

void orc_append_kidx_e4m3(const uint16_t *x_bf16, int32_t n, int32_t di, const int32_t *seq,
                          const int64_t *pos, const int32_t *page_table, int32_t max_pages,
                          int32_t page_size, uint8_t *kidx) {
    for (int32_t i = 0; i < n; ++i) {
        int64_t row = orc_physical_row(page_table + (int64_t)seq[i] * max_pages, page_size, pos[i]);
        orc_e4m3_row(x_bf16 + (int64_t)i * di, di, kidx + row * di);
    }
}

void orc_dequant_row(const uint8_t *codes, const uint8_t *scales, int32_t d, double *out) {
    for (int32_t i = 0; i < d; ++i) {
        uint32_t c = (codes[i / 2] >> (4 * (i % 2))) & 15u;
        out[i] = orc_e2m1_value(c) * orc_e4m3_value(scales[i / 16]);
    }
}

/* ------------------------------------------------------------------------ */
/* Indexer and Top-k                                                         */
/* ------------------------------------------------------------------------ */

double orc_index_score(const uint8_t *q, const float *w, int32_t hi, int32_t di,
                       const uint8_t *k) {
    double s = 0.0;
    for (int32_t h = 0; h < hi; ++h) {
        double dot = 0.0;
        for (int32_t i = 0; i < di; ++i)
            dot += orc_e4m3_value(q[h * di + i]) * orc_e4m3_value(k[i]);
        s += (double)w[h] * (dot > 0.0 ? dot : 0.0);
    }
    return s + 0.0;                                   /* -0 becomes +0 */
}

typedef struct {
    double score;
    int32_t id;
} orc_pair;

static int cmp_pair(const void *pa, const void *pb) {
    const orc_pair *a = (const orc_pair *)pa, *b = (const orc_pair *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->id > b->id) - (a->id < b->id);
}

int32_t orc_select_topk(const double *score, const int32_t *ids, int64_t n,
                        int32_t k, int32_t *out) {
    orc_pair *v = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        v[i].score = score[i];
        v[i].id = ids[i];
    }
    qsort(v, (size_t)n, sizeof(orc_pair), cmp_pair);
    int32_t m = (int64_t)k < n ? k : (int32_t)n;
    for (int32_t j = 0; j < m; ++j) out[j] = v[j].id;
    for (int32_t j = m; j < k; ++j) out[j] = -1;
    free(v);
    return m;
}

void orc_index_full(const uint8_t *qidx, const float *w, int32_t hi, int32_t di,
                    const uint8_t *kidx, const int32_t *page_table_seq, int32_t page_size,
                    int64_t n_visible, int32_t k, int32_t p,
                    int32_t *topk, int32_t *pool, double *scores_out) {
    int64_t n = n_visible > 0 ? n_visible : 0;
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t t = 0; t < n; ++t) {
        int64_t row = orc_physical_row(page_table_seq, page_size, t);
        s[t] = orc_index_score(qidx, w, hi, di, kidx + row * di);
        ids[t] = (int32_t)t;
        if (scores_out) scores_out[t] = s[t];
    }
    orc_select_topk(s, ids, n, k, topk);
    if (p > 0 && pool) orc_select_topk(s, ids, n, p, pool);
    free(s);
    free(ids);
}

void orc_index_reindex(const uint8_t *qidx, const float *w, int32_t hi, int32_t di,
                       const uint8_t *kidx, const int32_t *page_table_seq, int32_t page_size,
                       const int32_t *pool, int32_t p, int32_t k, int32_t *topk) {
    double *s = (double *)malloc(sizeof(double) * (size_t)(p > 0 ? p : 1));
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)(p > 0 ? p : 1));
    int64_t n = 0;
    for (int32_t j = 0; j < p; ++j) {
        if (pool[j] < 0) continue;
        int64_t row = orc_physical_row(page_table_seq, page_size, pool[j]);
        s[n] = orc_index_score(qidx, w, hi, di, kidx + row * di);
        ids[n] = pool[j];
        ++n;
    }
    orc_select_topk(s, ids, n, k, topk);
    free(s);
    free(ids);
}

/* ------------------------------------------------------------------------ */
/* Sparse + sliding-window attention                                         */
/* ------------------------------------------------------------------------ */

void orc_sparse_attn(const uint16_t *q_bf16, int32_t h, int32_t d,
                     const uint8_t *codes, const uint8_t *scales,
                     const int32_t *page_table_seq, int32_t page_size,
                     const int32_t *topk, int32_t k,
                     const uint8_t *swa_rows, int32_t nw,
                     double softmax_scale, double *o, double *lse) {
    /* gather the attended rows: selected global entries, then the window */
    int32_t nsel = 0;
    for (int32_t j = 0; j < k; ++j) nsel += topk[j] >= 0;
    int32_t nrow = nsel + nw;
    double *v = (double *)malloc(sizeof(double) * (size_t)(nrow > 0 ? nrow : 1) * (size_t)d);
    int32_t r = 0;
    for (int32_t j = 0; j < k; ++j) {
        if (topk[j] < 0) continue;
        int64_t row = orc_physical_row(page_table_seq, page_size, topk[j]);
        orc_dequant_row(codes + row * (d / 2), scales + row * (d / 16), d, v + (size_t)r * d);
        ++r;
    }
    for (int32_t j = 0; j < nw; ++j, ++r)
        for (int32_t i = 0; i < d; ++i)
            v[(size_t)r * d + i] = orc_e4m3_value(swa_rows[(size_t)j * d + i]);

    double *z = (double *)malloc(sizeof(double) * (size_t)(nrow > 0 ? nrow : 1));
    for (int32_t hh = 0; hh < h; ++hh) {
        double *oh = o + (size_t)hh * d;
        for (int32_t i = 0; i < d; ++i) oh[i] = 0.0;
        if (nrow == 0) {
            lse[hh] = -INFINITY;
            continue;
        }
        double m = -INFINITY;
        for (int32_t j = 0; j < nrow; ++j) {
            double dot = 0.0;
            for (int32_t i = 0; i < d; ++i)
                dot += (double)bf16_to_float(q_bf16[(size_t)hh * d + i]) * v[(size_t)j * d + i];
            z[j] = softmax_scale * dot;
            if (z[j] > m) m = z[j];
        }
        double l = 0.0;
        for (int32_t j = 0; j < nrow; ++j) {
            double pj = exp(z[j] - m);
            l += pj;
            for (int32_t i = 0; i < d; ++i) oh[i] += pj * v[(size_t)j * d + i];
        }
        for (int32_t i = 0; i < d; ++i) oh[i] /= l;
        lse[hh] = m + log(l);
    }
    free(z);
    free(v);
}
