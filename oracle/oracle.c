/*
 * oracle.c -- CPU oracle for the scaled FP8 / MXFP8 GEMM and its quantizers.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h): plain loops, fp64 arithmetic,
 * pthreads over output rows.  Build with strict IEEE semantics (no
 * -ffast-math): the fp32 steps below rely on IEEE single-precision division.
 */
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- formats */

double orc_e4m3_decode(uint8_t code) {
    int s = code >> 7;
    int E = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (E == 15 && m == 7) return NAN;
    if (E == 0)
        mag = ldexp((double)m, -9);              /* m/8 * 2^(1-7) */
    else
        mag = ldexp(1.0 + m / 8.0, E - 7);
    return s ? -mag : mag;
}

uint8_t orc_e4m3_encode(double v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;          /* saturate to the max finite */
    /* largest code c in [0, 0x7E] with decode(c) <= a (decode is increasing) */
    int lo = 0, hi = 0x7E;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (orc_e4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid - 1;
    }
    int c = lo;
    double d0 = orc_e4m3_decode((uint8_t)c);
    if (d0 == a) return sign | (uint8_t)c;
    double d1 = orc_e4m3_decode((uint8_t)(c + 1));
    double halfway = 0.5 * (d0 + d1);            /* exact: both are short dyadics */
    int pick;
    if (a < halfway) pick = c;
    else if (a > halfway) pick = c + 1;
    else pick = (c % 2 == 0) ? c : c + 1;        /* tie: even code */
    return sign | (uint8_t)pick;
}

int orc_mx_exponent(double amax) {
    if (amax == 0.0) return 127;
    double e = ceil(log2(amax / 448.0)) + 127.0;
    if (e < 0.0) e = 0.0;
    if (e > 254.0) e = 254.0;
    return (int)e;
}

static float bf16_to_float(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* --------------------------------------------------------------- threading */

typedef void (*row_fn)(void* ctx, int64_t row);
typedef struct { row_fn fn; void* ctx; int64_t r0, r1; } span_t;

static void* run_span(void* p) {
    span_t* s = (span_t*)p;
    for (int64_t r = s->r0; r < s->r1; ++r) s->fn(s->ctx, r);
    return NULL;
}

static void parallel_rows(int64_t rows, int nthreads, row_fn fn, void* ctx) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > rows) nthreads = (int)(rows > 0 ? rows : 1);
    pthread_t th[256];
    span_t sp[256];
    for (int t = 0; t < nthreads; ++t) {
        sp[t].fn = fn; sp[t].ctx = ctx;
        sp[t].r0 = rows * t / nthreads;
        sp[t].r1 = rows * (t + 1) / nthreads;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, run_span, &sp[t]);
    run_span(&sp[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------- quantizers */

typedef struct {
    const uint16_t* x; int64_t k, ld_x; uint8_t* q; int64_t ld_q; float* s; uint8_t* sf;
} quant_ctx;

static void rowwise_row(void* p, int64_t r) {
    quant_ctx* c = (quant_ctx*)p;
    const uint16_t* xr = c->x + r * c->ld_x;
    float amax = 0.0f;
    for (int64_t j = 0; j < c->k; ++j) {
        float a = fabsf(bf16_to_float(xr[j]));
        if (a > amax) amax = a;
    }
    /* scale = amax / 448, held as an fp32 tensor element */
    float s = (amax == 0.0f) ? 1.0f : (float)((double)amax / 448.0);
    c->s[r] = s;
    for (int64_t j = 0; j < c->k; ++j) {
        float v = bf16_to_float(xr[j]) / s;      /* fp32 quotient, IEEE RN */
        c->q[r * c->ld_q + j] = orc_e4m3_encode((double)v);
    }
}

void orc_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t k, int64_t ld_x,
                          uint8_t* q, int64_t ld_q, float* s, int nthreads) {
    quant_ctx c = {x, k, ld_x, q, ld_q, s, NULL};
    parallel_rows(rows, nthreads, rowwise_row, &c);
}

float orc_tensor_scale(const uint16_t* x, int64_t rows, int64_t k, int64_t ld_x) {
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            float a = fabsf(bf16_to_float(x[r * ld_x + j]));
            if (a > amax) amax = a;
        }
    return (amax == 0.0f) ? 1.0f : (float)((double)amax / 448.0);
}

typedef struct { const uint16_t* x; int64_t k, ld_x; float s; uint8_t* q; int64_t ld_q; } static_ctx;

static void static_row(void* p, int64_t r) {
    static_ctx* c = (static_ctx*)p;
    for (int64_t j = 0; j < c->k; ++j) {
        float v = bf16_to_float(c->x[r * c->ld_x + j]) / c->s;   /* fp32 quotient, IEEE RN */
        c->q[r * c->ld_q + j] = orc_e4m3_encode((double)v);
    }
}

void orc_quantize_static(const uint16_t* x, int64_t rows, int64_t k, int64_t ld_x, float s,
                         uint8_t* q, int64_t ld_q, int nthreads) {
    static_ctx c = {x, k, ld_x, s, q, ld_q};
    parallel_rows(rows, nthreads, static_row, &c);
}

static void mx_row(void* p, int64_t r) {
    quant_ctx* c = (quant_ctx*)p;
    const uint16_t* xr = c->x + r * c->ld_x;
    int64_t nkb = c->k / 32;
    for (int64_t b = 0; b < nkb; ++b) {
        double amax = 0.0;
        for (int j = 0; j < 32; ++j) {
            double a = fabs((double)bf16_to_float(xr[b * 32 + j]));
            if (a > amax) amax = a;
        }
        int e = orc_mx_exponent(amax);
        c->sf[r * nkb + b] = (uint8_t)e;
        for (int j = 0; j < 32; ++j) {
            double v = (double)bf16_to_float(xr[b * 32 + j]) * ldexp(1.0, 127 - e);
            c->q[r * c->ld_q + b * 32 + j] = orc_e4m3_encode(v);
        }
    }
}

void orc_mx_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld_x,
                     uint8_t* q, int64_t ld_q, uint8_t* sf, int nthreads) {
    quant_ctx c = {x, k, ld_x, q, ld_q, NULL, sf};
    parallel_rows(rows, nthreads, mx_row, &c);
}

/* ------------------------------------------------------------------ GEMMs */

typedef struct {
    const uint8_t *qa, *qb, *sfa, *sfb;
    int64_t n, k;
    const float *sa, *sb;
    double *c, *bound;
    double dec[256];
} gemm_ctx;

static void gemm_rowwise_row(void* p, int64_t i) {
    gemm_ctx* g = (gemm_ctx*)p;
    const uint8_t* a = g->qa + i * g->k;
    for (int64_t j = 0; j < g->n; ++j) {
        const uint8_t* b = g->qb + j * g->k;
        double d = 0.0, dabs = 0.0;
        for (int64_t t = 0; t < g->k; ++t) {
            double prod = g->dec[a[t]] * g->dec[b[t]];
            d += prod;
            dabs += fabs(prod);
        }
        double sab = (double)g->sa[i] * (double)g->sb[j];
        g->c[i * g->n + j] = sab * d;
        if (g->bound) g->bound[i * g->n + j] = fabs(sab) * dabs;
    }
}

void orc_gemm_rowwise(const uint8_t* qa, const uint8_t* qb, int64_t m, int64_t n, int64_t k,
                      const float* sa, const float* sb, double* c_ref, double* bound,
                      int nthreads) {
    gemm_ctx* g = (gemm_ctx*)calloc(1, sizeof(gemm_ctx));
    g->qa = qa; g->qb = qb; g->n = n; g->k = k; g->sa = sa; g->sb = sb;
    g->c = c_ref; g->bound = bound;
    for (int v = 0; v < 256; ++v) g->dec[v] = orc_e4m3_decode((uint8_t)v);
    parallel_rows(m, nthreads, gemm_rowwise_row, g);
    free(g);
}

static void gemm_mx_row(void* p, int64_t i) {
    gemm_ctx* g = (gemm_ctx*)p;
    int64_t nkb = g->k / 32;
    const uint8_t* a = g->qa + i * g->k;
    for (int64_t j = 0; j < g->n; ++j) {
        const uint8_t* b = g->qb + j * g->k;
        double acc = 0.0, accabs = 0.0;
        for (int64_t blk = 0; blk < nkb; ++blk) {
            double d = 0.0, dabs = 0.0;
            for (int t = 0; t < 32; ++t) {
                double prod = g->dec[a[blk * 32 + t]] * g->dec[b[blk * 32 + t]];
                d += prod;
                dabs += fabs(prod);
            }
            int ex = (int)g->sfa[i * nkb + blk] + (int)g->sfb[j * nkb + blk] - 254;
            acc += ldexp(d, ex);
            accabs += ldexp(dabs, ex);
        }
        g->c[i * g->n + j] = acc;
        if (g->bound) g->bound[i * g->n + j] = accabs;
    }
}

void orc_gemm_mx(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb, const uint8_t* sfb,
                 int64_t m, int64_t n, int64_t k, double* c_ref, double* bound, int nthreads) {
    gemm_ctx* g = (gemm_ctx*)calloc(1, sizeof(gemm_ctx));
    g->qa = qa; g->qb = qb; g->sfa = sfa; g->sfb = sfb; g->n = n; g->k = k;
    g->c = c_ref; g->bound = bound;
    for (int v = 0; v < 256; ++v) g->dec[v] = orc_e4m3_decode((uint8_t)v);
    parallel_rows(m, nthreads, gemm_mx_row, g);
    free(g);
}
