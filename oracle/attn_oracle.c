/*
 * attn_oracle.c -- the parity oracle for the attention forward pass.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the package
 * smoke check and the benchmark's CPU-baseline / reference arm load this
 * library.  It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes (plain definition, fp64 throughout):
 *
 *   for every batch b, head h and query row i
 *     s_ij  = scale * sum_d q[b,h,i,d] * k[b,h,j,d]     over the visible keys j
 *     M_i   = max_j s_ij
 *     L_i   = sum_j exp(s_ij - M_i)
 *     O_i,: = sum_j exp(s_ij - M_i) * v[b,h,j,:] / L_i
 *     LSE_i = M_i + ln(L_i)
 *
 *   visible keys: all j < Sk; with the causal flag only j <= i (the mask is
 *   aligned at the top-left corner when Sq != Sk, so every row sees key 0).
 *
 * Sources on the pages:
 *   - the standard, materialised attention that FlashAttention must reproduce:
 *     page "FlashAttention in ops-transformer on Ascend NPU" (ai6s.net/6a0d3bfb),
 *     section "why standard attention stalls", the standard_attention snippet
 *     (scores = Q K^T / sqrt(d), softmax over the last axis, times V); and
 *     page "FlashAttention: long-text inference without running out of memory"
 *     (ai6s.net/6a0d42d8), section "the memory black hole",
 *     Attention(Q,K,V) = Softmax(QK^T/sqrt(d)) V with its three steps.
 *   - the accuracy check that compares against exactly this routine: page
 *     "ops-transformer FlashAttention on Atlas 800" (hwcomputing.csdn.net/6a0d4444),
 *     section "accuracy check".
 *   - the causal flag instead of a mask tensor, with the mask
 *     triu(ones(S,S), diagonal=1) as its meaning: page ai6s.net/6a0d3bfb,
 *     section "how FlashAttention runs on the Ascend NPU".
 *   - the log-sum-exp per row, natural log: page "64K long-sequence
 *     FlashAttention" (ai6s.net/6a140d07), section "layer 2: numerical
 *     stability" (the lse accumulator of shape [B, H, block_i] and torch.log).
 *   - BSND / BNSD (= BHSD) layouts: page hwcomputing.csdn.net/6a0d4444,
 *     sections "minimal runnable code" and the error table; page
 *     "catlass FlashAttention template tuning" (hwcomputing.csdn.net/6a0d4681),
 *     section "data layout".
 *
 * The score row is materialised in full (Sk doubles per row) and the softmax
 * takes two passes over it (max, then exp-sum), as the standard routine does.
 * Rows are independent; OpenMP splits them across threads.  No blocking, no
 * online rescaling, no reordering of the sums beyond the definition.
 *
 * Inputs are the same 16-bit tensors the GPU receives, decoded exactly to
 * fp64 (fp16 through a 65536-entry table filled by the decoder below; bf16 by
 * widening its bits to an IEEE binary32), or fp64 arrays.
 *
 * ORACLE_PLANT (compile-time, tests only): plants one deliberate mistake so
 * the test suite can show that its pins catch it.  Never set in the normal
 * build.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

enum { ORACLE_FP16 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 };
enum { ORACLE_BSND = 0, ORACLE_BHSD = 1 };
enum { ORACLE_OK = 0, ORACLE_EINVAL = 1, ORACLE_ENOMEM = 2 };

/* IEEE 754 binary16: sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_fp16_to_f64(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double mag;
    if (e == 0)
        mag = ldexp((double)f, -24);              /* subnormal: f * 2^-24 */
    else if (e == 31)
        mag = f ? NAN : INFINITY;
    else
        mag = ldexp((double)(1024 + f), e - 25);  /* (1 + f/1024) * 2^(e-15) */
    return sign ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE 754 binary32. */
double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double g_fp16_table[65536];
static int g_fp16_table_ready = 0;

static void fill_fp16_table(void)
{
    if (g_fp16_table_ready)
        return;
    for (uint32_t u = 0; u < 65536u; ++u)
        g_fp16_table[u] = oracle_fp16_to_f64((uint16_t)u);
    g_fp16_table_ready = 1;
}

typedef struct {
    const void *p;
    int dtype;
    int layout;
    int64_t H, S, D;
} view_t;

/* Flat element index of (b, h, s, d) in the stated layout. */
static int64_t elem_index(const view_t *t, int64_t b, int64_t h, int64_t s, int64_t d)
{
#if ORACLE_PLANT == 6
    /* planted: BSND addressed as if it were BHSD */
    return ((b * t->H + h) * t->S + s) * t->D + d;
#else
    if (t->layout == ORACLE_BSND)
        return ((b * t->S + s) * t->H + h) * t->D + d;
    return ((b * t->H + h) * t->S + s) * t->D + d;
#endif
}

static double load(const view_t *t, int64_t idx)
{
    switch (t->dtype) {
    case ORACLE_FP16: return g_fp16_table[((const uint16_t *)t->p)[idx]];
    case ORACLE_BF16: return oracle_bf16_to_f64(((const uint16_t *)t->p)[idx]);
    default:          return ((const double *)t->p)[idx];
    }
}

/* Decodes one D-long row (b, h, s, :) into dst. */
static void load_row(const view_t *t, int64_t b, int64_t h, int64_t s, double *dst)
{
    for (int64_t d = 0; d < t->D; ++d)
        dst[d] = load(t, elem_index(t, b, h, s, d));
}

/* Number of keys that query row i may attend to. */
static int64_t visible_keys(int64_t i, int64_t Sk, int causal)
{
    if (!causal)
        return Sk;
#if ORACLE_PLANT == 2
    /* planted: causal off by one (j < i instead of j <= i) */
    return i < Sk ? i : Sk;
#else
    return i + 1 < Sk ? i + 1 : Sk;
#endif
}

/*
 * One query row, straight from the definition.  scores has room for Sk
 * doubles, qrow and vrow for D doubles, o_out receives D doubles.
 * weights_out, when not NULL, receives the Sk softmax weights (0 where masked).
 */
static void attend_row(const view_t *q, const view_t *k, const view_t *v,
                       int64_t b, int64_t h, int64_t i, int64_t Sk, int causal,
                       double scale, double *scores, double *qrow, double *vrow,
                       double *o_out, double *lse_out, double *weights_out)
{
    const int64_t D = q->D;
    const int64_t n = visible_keys(i, Sk, causal);

    load_row(q, b, h, i, qrow);

    /* step 1: the full (visible part of the) score row */
    for (int64_t j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) {
#if ORACLE_PLANT == 1
            /* planted: query and key swapped for the row index */
            dot += load(q, elem_index(q, b, h, j < q->S ? j : 0, d)) *
                   load(k, elem_index(k, b, h, i < k->S ? i : 0, d));
#else
            dot += qrow[d] * load(k, elem_index(k, b, h, j, d));
#endif
        }
#if ORACLE_PLANT == 3
        scores[j] = scale * scale * dot;   /* planted: scale applied twice */
#else
        scores[j] = scale * dot;
#endif
    }

    /* step 2: softmax, first pass = row max, second pass = exp-sum */
    double M = -INFINITY;
    for (int64_t j = 0; j < n; ++j)
        if (scores[j] > M)
            M = scores[j];
    double L = 0.0;
    for (int64_t j = 0; j < n; ++j) {
#if ORACLE_PLANT == 5
        scores[j] = exp(M - scores[j]);    /* planted: sign of the exponent flipped */
#else
        scores[j] = exp(scores[j] - M);
#endif
        L += scores[j];
    }

    /* step 3: weights times V */
    for (int64_t d = 0; d < D; ++d)
        o_out[d] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
#if ORACLE_PLANT == 4
        load_row(v, b, h, i < v->S ? i : 0, vrow);   /* planted: V row of the query */
#else
        load_row(v, b, h, j, vrow);
#endif
        const double w = scores[j];
        for (int64_t d = 0; d < D; ++d)
            o_out[d] += w * vrow[d];
    }
#if ORACLE_PLANT != 7
    for (int64_t d = 0; d < D; ++d)
        o_out[d] /= L;                     /* plant 7 drops this normalisation */
#endif

#if ORACLE_PLANT == 8
    *lse_out = log(L);                     /* planted: the max is not added back */
#else
    *lse_out = M + log(L);
#endif

    if (weights_out) {
        for (int64_t j = 0; j < Sk; ++j)
            weights_out[j] = j < n ? scores[j] / L : 0.0;
    }
}

static int check_args(const void *q, const void *k, const void *v, int64_t B, int64_t H,
                      int64_t Sq, int64_t Sk, int64_t D, int layout, int dtype)
{
    if (!q || !k || !v)
        return ORACLE_EINVAL;
    if (B <= 0 || H <= 0 || Sq <= 0 || Sk <= 0 || D <= 0)
        return ORACLE_EINVAL;
    if (layout != ORACLE_BSND && layout != ORACLE_BHSD)
        return ORACLE_EINVAL;
    if (dtype != ORACLE_FP16 && dtype != ORACLE_BF16 && dtype != ORACLE_F64)
        return ORACLE_EINVAL;
    return ORACLE_OK;
}

/*
 * Attention forward for a list of query rows.
 *
 * rows[r] is a flat row id (b * H + h) * Sq + i.  For each r the output row
 * goes to o_out[r * D .. r * D + D) and its log-sum-exp to lse_out[r].
 * With rows == NULL every row is computed and o_out / lse_out are laid out
 * as [B, H, Sq, D] and [B, H, Sq] (row-major), whatever the input layout.
 * nthreads <= 0 lets OpenMP choose.
 */
int oracle_attn_fwd_rows(const void *q, const void *k, const void *v,
                         int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                         int layout, int causal, double scale, int dtype,
                         const int64_t *rows, int64_t nrows,
                         double *o_out, double *lse_out, int nthreads)
{
    int rc = check_args(q, k, v, B, H, Sq, Sk, D, layout, dtype);
    if (rc != ORACLE_OK)
        return rc;
    if (!o_out || !lse_out)
        return ORACLE_EINVAL;
    if (dtype == ORACLE_FP16)
        fill_fp16_table();

    const view_t vq = {q, dtype, layout, H, Sq, D};
    const view_t vk = {k, dtype, layout, H, Sk, D};
    const view_t vv = {v, dtype, layout, H, Sk, D};
    const int64_t total = rows ? nrows : B * H * Sq;
    int failed = 0;

#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads) reduction(| : failed)
#endif
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)Sk);
        double *qrow = (double *)malloc(sizeof(double) * (size_t)D);
        double *vrow = (double *)malloc(sizeof(double) * (size_t)D);
        if (!scores || !qrow || !vrow) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
            for (int64_t r = 0; r < total; ++r) {
                const int64_t flat = rows ? rows[r] : r;
                if (flat < 0 || flat >= B * H * Sq) {
                    failed = 1;
                    continue;
                }
                const int64_t i = flat % Sq;
                const int64_t bh = flat / Sq;
                attend_row(&vq, &vk, &vv, bh / H, bh % H, i, Sk, causal, scale,
                           scores, qrow, vrow, o_out + r * D, lse_out + r, NULL);
            }
        }
        free(scores);
        free(qrow);
        free(vrow);
    }
    return failed ? ORACLE_EINVAL : ORACLE_OK;
}

/* The softmax weights of one query row (Sk doubles, zero where masked). */
int oracle_attn_weights(const void *q, const void *k, const void *v,
                        int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                        int layout, int causal, double scale, int dtype,
                        int64_t row, double *weights_out)
{
    int rc = check_args(q, k, v, B, H, Sq, Sk, D, layout, dtype);
    if (rc != ORACLE_OK)
        return rc;
    if (!weights_out || row < 0 || row >= B * H * Sq)
        return ORACLE_EINVAL;
    if (dtype == ORACLE_FP16)
        fill_fp16_table();
    const view_t vq = {q, dtype, layout, H, Sq, D};
    const view_t vk = {k, dtype, layout, H, Sk, D};
    const view_t vv = {v, dtype, layout, H, Sk, D};
    double *scores = (double *)malloc(sizeof(double) * (size_t)Sk);
    double *buf = (double *)malloc(sizeof(double) * (size_t)(3 * D));
    if (!scores || !buf) {
        free(scores);
        free(buf);
        return ORACLE_ENOMEM;
    }
    double lse;
    const int64_t i = row % Sq, bh = row / Sq;
    attend_row(&vq, &vk, &vv, bh / H, bh % H, i, Sk, causal, scale,
               scores, buf, buf + D, buf + 2 * D, &lse, weights_out);
    free(scores);
    free(buf);
    return ORACLE_OK;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int oracle_plant(void) { return ORACLE_PLANT; }
