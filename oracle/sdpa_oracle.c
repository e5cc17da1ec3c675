/*
 * Plain fp64 CPU oracle for the scaled-dot-product attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file;
 * only tests/, the smoke check and the CPU-baseline leg of the benchmark load
 * it.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (one query row at a time, no tiling, no online softmax):
 *
 *   g    = h / (headNum / kvHeadNum)                        GQA grouping
 *   s_j  = qkScale * ( sum_d q[i,h,d] k[j,g,d]
 *                    + sum_r qRope[i,h,r] kRope[j,g,r] )     MLA split contraction
 *          + addmask[i,j]                                   float mask is added
 *   keep_j = keepmask[i,j] != 0                              bool mask: true = keep
 *            and (causal => j <= i + Lk - Lq)                bottom-right causal
 *   out[i,h,:] = sum_keep exp(s_j - m) v[j,g,:] / sum_keep exp(s_j - m),
 *   m = max_keep s_j;  a row with no kept key gives out = 0, lse = -inf.
 *
 * Sources:
 *  - "Core 注意力" (WorldFoundry docs), section "选择最窄的入口": the entry
 *    follows the PyTorch SDPA contract with GQA expansion.
 *  - same page, section "一个可以在 CPU 或 GPU 上运行的例子", closing
 *    paragraph: a boolean mask marks the scores that are kept, a float mask
 *    is added to the score matrix.
 *  - "MLA Prefill" (CANN ATB docs), parameter table: Q/QRope/K/kRope/V
 *    shapes, qSeqLen/kvSeqLen per sequence, headNum/kvHeadNum, qkScale is
 *    multiplied after Q*K^T, maskType causal variants.
 *
 * Readings where the pages are silent: causal is aligned bottom-right
 * (identical to top-left when Lq == Lk); a fully masked row yields zeros.
 *
 * Built with:  gcc -O2 -fopenmp -shared -fPIC sdpa_oracle.c -o liboracle.so -lm
 * A second build with -DORACLE_PLANT=<n> carries one deliberately planted
 * mistake; the pin tests use those builds to show that every pin is able to
 * catch a plausible error.  The faithful build defines no ORACLE_PLANT.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

typedef struct {
    const double *ptr;   /* element (b,h,row,d) at ptr + b*sb + h*sh + row*si + d */
    int64_t sb, sh, si;  /* element strides; sb is ignored for packed (varlen) input */
} ora_tensor;

typedef struct {
    int32_t batch, head_num, kv_head_num;
    int32_t dqk, drope, dv;      /* drope = 0 when there is no rope part */
    int32_t varlen;              /* 0: [B,H,L,D] dense, 1: packed [T,H,D] */
    int64_t lq, lk;              /* dense lengths (ignored when varlen) */
    const int32_t *q_seqlen;     /* [batch], varlen only */
    const int32_t *kv_seqlen;    /* [batch], varlen only */
    ora_tensor q, qrope, k, krope, v;
    double *out;                 /* full-forward output, addressed with out_t's strides */
    ora_tensor out_t;
    int32_t mask_kind;           /* 0 none, 1 causal, 2 bool keep, 3 additive */
    const uint8_t *keep;         /* mask_kind 2 */
    const double *add;           /* mask_kind 3 */
    int64_t mb, mh, mi, mj;      /* mask element strides, 0 = broadcast */
    double qk_scale;
    double *lse;                 /* optional natural-log LSE: [B,H,Lq] dense, [H,T] packed */
    int64_t lse_ld;              /* packed only: T, the row count of one head's LSE run */
} ora_args;

enum { ORA_OK = 0, ORA_BAD_ARG = 1, ORA_NO_MEMORY = 2 };

static const double *row_ptr(const ora_tensor *t, int64_t b, int64_t h, int64_t row)
{
    return t->ptr + b * t->sb + h * t->sh + row * t->si;
}

/* One (sequence, head, query row): the definition written out directly. */
static void one_row(const ora_args *a, int64_t b, int64_t h, int64_t i,
                    int64_t q_off, int64_t k_off, int64_t Lq, int64_t Lk,
                    int64_t seq_b, double *s, unsigned char *kept,
                    double *oi, double *lse_i)
{
    int64_t group = a->head_num / a->kv_head_num;
    int64_t g = h / group;
#if ORACLE_PLANT == 1
    g = h % a->kv_head_num;                     /* planted: wrong GQA index */
#endif
    const double *qi = row_ptr(&a->q, seq_b, h, q_off + i);
    const double *qri = a->drope ? row_ptr(&a->qrope, seq_b, h, q_off + i) : NULL;
    int64_t any = 0;
    double m = -INFINITY;

    for (int64_t j = 0; j < Lk; ++j) {
        const double *kj = row_ptr(&a->k, seq_b, g, k_off + j);
        double dot = 0.0;
        for (int d = 0; d < a->dqk; ++d) dot += qi[d] * kj[d];
#if ORACLE_PLANT != 3                           /* planted 3: rope term dropped */
        if (a->drope) {
            const double *krj = row_ptr(&a->krope, seq_b, g, k_off + j);
            for (int r = 0; r < a->drope; ++r) dot += qri[r] * krj[r];
        }
#endif
        double sj = a->qk_scale * dot;
        int keep = 1;
        if (a->mask_kind == 1) {
#if ORACLE_PLANT == 2
            keep = (j <= i);                    /* planted: top-left causal */
#else
            keep = (j <= i + Lk - Lq);
#endif
        } else if (a->mask_kind == 2) {
            uint8_t kv = a->keep[b * a->mb + h * a->mh + i * a->mi + j * a->mj];
#if ORACLE_PLANT == 4
            keep = (kv == 0);                   /* planted: polarity flipped */
#else
            keep = (kv != 0);
#endif
        } else if (a->mask_kind == 3) {
            double add = a->add[b * a->mb + h * a->mh + i * a->mi + j * a->mj];
#if ORACLE_PLANT == 5
            sj = a->qk_scale * (dot + add);     /* planted: mask added before scaling */
#else
            sj += add;
#endif
        }
        s[j] = sj;
        kept[j] = (unsigned char)keep;
        if (keep) {
            any = 1;
            if (sj > m) m = sj;
        }
    }

    for (int e = 0; e < a->dv; ++e) oi[e] = 0.0;
    double denom = 0.0;
    if (any) {
        for (int64_t j = 0; j < Lk; ++j) {
#if ORACLE_PLANT == 7
            denom += exp(s[j] - m);             /* planted: masked keys in the normaliser */
#endif
            if (!kept[j]) continue;
#if ORACLE_PLANT == 6
            double p = exp(m - s[j]);           /* planted: sign flipped in the exponent */
#else
            double p = exp(s[j] - m);
#endif
#if ORACLE_PLANT != 7
            denom += p;
#endif
            const double *vj = row_ptr(&a->v, seq_b, g, k_off + j);
            for (int e = 0; e < a->dv; ++e) oi[e] += p * vj[e];
        }
        for (int e = 0; e < a->dv; ++e) oi[e] /= denom;
    }
    if (lse_i) *lse_i = any ? m + log(denom) : -INFINITY;
}

/* Full forward.  Rows are independent, so OpenMP splits (sequence, head, row). */
int ora_sdpa_fwd(const ora_args *a)
{
    if (!a || a->batch < 0 || a->head_num <= 0 || a->kv_head_num <= 0) return ORA_BAD_ARG;
    if (a->head_num % a->kv_head_num != 0) return ORA_BAD_ARG;
    if (a->varlen && (a->mask_kind == 2 || a->mask_kind == 3)) return ORA_BAD_ARG;

    int64_t B = a->batch, H = a->head_num;
    int64_t *q_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B + 1));
    int64_t *k_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B + 1));
    if (!q_off || !k_off) { free(q_off); free(k_off); return ORA_NO_MEMORY; }
    /* Per-sequence start rows: running sums of the lengths (packed layout). */
    q_off[0] = 0; k_off[0] = 0;
    int64_t max_lk = 0;
    for (int64_t b = 0; b < B; ++b) {
        int64_t lq = a->varlen ? a->q_seqlen[b] : a->lq;
        int64_t lk = a->varlen ? a->kv_seqlen[b] : a->lk;
        if (lq < 0 || lk < 0) { free(q_off); free(k_off); return ORA_BAD_ARG; }
        q_off[b + 1] = a->varlen ? q_off[b] + lq : 0;
        k_off[b + 1] = a->varlen ? k_off[b] + lk : 0;
        if (lk > max_lk) max_lk = lk;
    }
    int64_t max_lq = 0;
    for (int64_t b = 0; b < B; ++b) {
        int64_t lq = a->varlen ? a->q_seqlen[b] : a->lq;
        if (lq > max_lq) max_lq = lq;
    }
    int err = ORA_OK;
    int64_t total = B * H * max_lq;

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_lk + 1));
        unsigned char *kept = (unsigned char *)malloc((size_t)(max_lk + 1));
        if (!s || !kept) {
#pragma omp atomic write
            err = ORA_NO_MEMORY;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < total; ++t) {
                int64_t b = t / (H * max_lq);
                int64_t h = (t / max_lq) % H;
                int64_t i = t % max_lq;
                int64_t lq = a->varlen ? a->q_seqlen[b] : a->lq;
                int64_t lk = a->varlen ? a->kv_seqlen[b] : a->lk;
                if (i >= lq) continue;
                int64_t seq_b = a->varlen ? 0 : b;     /* packed input has no batch stride */
                double *oi = a->out + seq_b * a->out_t.sb + h * a->out_t.sh
                             + (q_off[b] + i) * a->out_t.si;
                double *lse_i = NULL;
                if (a->lse)
                    lse_i = a->varlen ? a->lse + h * a->lse_ld + q_off[b] + i   /* [H, T] */
                                      : a->lse + (b * H + h) * lq + i;          /* [B, H, Lq] */
                one_row(a, b, h, i, q_off[b], k_off[b], lq, lk, seq_b, s, kept, oi, lse_i);
            }
        }
        free(s);
        free(kept);
    }
    free(q_off);
    free(k_off);
    return err;
}

/* A subset of rows: rows[n] = (sequence, head, row-within-sequence).  Used on
 * workloads whose full fp64 evaluation would take too long; each listed row is
 * still evaluated over its complete key range.  Row t's output goes to
 * out_rows[t*dv .. t*dv+dv) and its LSE (if lse_rows) to lse_rows[t]. */
int ora_sdpa_fwd_rows(const ora_args *a, const int64_t *rows, int64_t n,
                      double *out_rows, double *lse_rows)
{
    if (!a || a->head_num <= 0 || a->kv_head_num <= 0) return ORA_BAD_ARG;
    if (a->head_num % a->kv_head_num != 0) return ORA_BAD_ARG;
    if (a->varlen && (a->mask_kind == 2 || a->mask_kind == 3)) return ORA_BAD_ARG;
    int64_t B = a->batch;
    int64_t *q_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B + 1));
    int64_t *k_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(B + 1));
    if (!q_off || !k_off) { free(q_off); free(k_off); return ORA_NO_MEMORY; }
    q_off[0] = 0; k_off[0] = 0;
    int64_t max_lk = 0;
    for (int64_t b = 0; b < B; ++b) {
        int64_t lq = a->varlen ? a->q_seqlen[b] : a->lq;
        int64_t lk = a->varlen ? a->kv_seqlen[b] : a->lk;
        q_off[b + 1] = a->varlen ? q_off[b] + lq : 0;
        k_off[b + 1] = a->varlen ? k_off[b] + lk : 0;
        if (lk > max_lk) max_lk = lk;
    }
    int err = ORA_OK;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_lk + 1));
        unsigned char *kept = (unsigned char *)malloc((size_t)(max_lk + 1));
        if (!s || !kept) {
#pragma omp atomic write
            err = ORA_NO_MEMORY;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < n; ++t) {
                int64_t b = rows[3 * t], h = rows[3 * t + 1], i = rows[3 * t + 2];
                int64_t lq = a->varlen ? a->q_seqlen[b] : a->lq;
                int64_t lk = a->varlen ? a->kv_seqlen[b] : a->lk;
                if (b < 0 || b >= B || h < 0 || h >= a->head_num || i < 0 || i >= lq) continue;
                int64_t seq_b = a->varlen ? 0 : b;
                one_row(a, b, h, i, q_off[b], k_off[b], lq, lk, seq_b, s, kept,
                        out_rows + t * a->dv, lse_rows ? lse_rows + t : NULL);
            }
        }
        free(s);
        free(kept);
    }
    free(q_off);
    free(k_off);
    return err;
}

int ora_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
