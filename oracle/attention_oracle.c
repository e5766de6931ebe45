/*
 * attention_oracle.c -- plain fp64 CPU oracle for decode / small-Q attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the bench's CPU
 * baseline use it.  It shares no code, header or constant with the CUDA
 * library; it decodes fp16/bf16 bit patterns itself from the IEEE / bfloat16
 * format definitions.
 *
 * What it computes (the plain definition, no tiling, no online rescaling):
 *
 *   O = softmax(Q K^T * scale) V,  scale defaults to 1/sqrt(headDim)
 *     -- "SmallQ FlashAttention for Ascend 910B", section "接口" (interface):
 *        O = softmax(Q·Kᵀ/√headDim)·V;
 *     -- "昇腾CANN上的FlashAttention工程实战", section on standard attention:
 *        scores are divided by the scaling factor, soft-maxed, then times V.
 *
 * For every requested output row (b, hq, i):
 *   hkv = hq / (Hq / Hkv)                      grouped-query map (GQA)
 *   n   = seqlens ? seqlens[b] : Lk            keys present for batch b
 *   key j is visible iff j < n and (not causal or j <= i + n - Lq)
 *                                              (causal mask aligned to the
 *                                               bottom-right corner)
 *   s_j = scale * sum_d q[b,i,hq,d] * k[b,j,hkv,d]
 *   m   = max_j s_j,  l = sum_j exp(s_j - m)
 *   O[b,i,hq,:] = sum_j exp(s_j - m) v[b,j,hkv,:] / l
 *   lse[b,hq,i] = m + ln(l)                    natural log-sum-exp
 * A row with no visible key gets O = 0 and lse = -inf.
 *
 * Subtracting m is an exact identity of softmax (it only keeps exp() in
 * range); it is not a reformulation of the method.
 *
 * Inputs are raw element arrays addressed by element strides
 * ([B, L, H, D] order), of type fp16 (0), bf16 (1) or fp64 (2).
 * Rows are processed in parallel with POSIX threads, one row at a time per
 * thread; every sum is a plain left-to-right fp64 loop.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 };

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double x;
    if (e == 0) {
        x = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
    } else if (e == 31) {
        x = f ? NAN : INFINITY;
    } else {
        x = ldexp((double)(1024 + f), e - 25); /* (1 + f/2^10) * 2^(e-15) */
    }
    return sign ? -x : x;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double oracle_bf16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int f = h & 0x7f;
    double x;
    if (e == 0) {
        x = ldexp((double)f, -133); /* subnormal: f * 2^-126 * 2^-7 */
    } else if (e == 255) {
        x = f ? NAN : INFINITY;
    } else {
        x = ldexp((double)(128 + f), e - 134); /* (1 + f/2^7) * 2^(e-127) */
    }
    return sign ? -x : x;
}

static double load_elem(const void *base, int dtype, int64_t idx) {
    if (dtype == ORACLE_F64) return ((const double *)base)[idx];
    uint16_t bits = ((const uint16_t *)base)[idx];
    return dtype == ORACLE_F16 ? oracle_f16_to_f64(bits) : oracle_bf16_to_f64(bits);
}

typedef struct {
    const void *q, *k, *v;
    const int64_t *qs, *ks, *vs; /* element strides, 4 each, [B, L, H, D] */
    int dtype;
    int64_t B, Lq, Hq, Lk, Hkv, Dqk, Dv;
    const int32_t *seqlens;
    int causal;
    double scale;
    int64_t nrows;
    const int64_t *rows; /* nrows x (b, hq, i), or NULL for all rows */
    double *o;           /* nrows x Dv */
    double *lse;         /* nrows */
    int nthreads;
    int tid;
    int status;
} job_t;

/* One output row by the definition. scores: scratch of >= Lk doubles. */
static void one_row(const job_t *J, int64_t b, int64_t hq, int64_t i, double *scores,
                    double *o_row, double *lse_row) {
    int64_t g = J->Hq / J->Hkv;
    int64_t hkv = hq / g;
    int64_t n = J->seqlens ? (int64_t)J->seqlens[b] : J->Lk;
    int64_t last = n - 1; /* last visible key, inclusive */
    if (J->causal && i + n - J->Lq < last) last = i + n - J->Lq;

    for (int64_t d = 0; d < J->Dv; ++d) o_row[d] = 0.0;
    if (last < 0) {
        *lse_row = -INFINITY;
        return;
    }
    int64_t qoff = b * J->qs[0] + i * J->qs[1] + hq * J->qs[2];
    double m = -INFINITY;
    for (int64_t j = 0; j <= last; ++j) {
        int64_t koff = b * J->ks[0] + j * J->ks[1] + hkv * J->ks[2];
        double dot = 0.0;
        for (int64_t d = 0; d < J->Dqk; ++d)
            dot += load_elem(J->q, J->dtype, qoff + d * J->qs[3]) *
                   load_elem(J->k, J->dtype, koff + d * J->ks[3]);
        scores[j] = J->scale * dot;
        if (scores[j] > m) m = scores[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j <= last; ++j) {
        double p = exp(scores[j] - m);
        l += p;
        int64_t voff = b * J->vs[0] + j * J->vs[1] + hkv * J->vs[2];
        for (int64_t d = 0; d < J->Dv; ++d)
            o_row[d] += p * load_elem(J->v, J->dtype, voff + d * J->vs[3]);
    }
    for (int64_t d = 0; d < J->Dv; ++d) o_row[d] /= l;
    *lse_row = m + log(l);
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(J->Lk > 0 ? J->Lk : 1));
    if (!scores) {
        J->status = -2;
        return NULL;
    }
    for (int64_t r = J->tid; r < J->nrows; r += J->nthreads) {
        int64_t b, hq, i;
        if (J->rows) {
            b = J->rows[3 * r];
            hq = J->rows[3 * r + 1];
            i = J->rows[3 * r + 2];
        } else { /* all rows in (b, hq, i) order */
            i = r % J->Lq;
            hq = (r / J->Lq) % J->Hq;
            b = r / (J->Lq * J->Hq);
        }
        one_row(J, b, hq, i, scores, J->o + r * J->Dv, J->lse + r);
    }
    free(scores);
    return NULL;
}

/*
 * Returns 0 on success, -1 on an invalid argument, -2 when memory or a
 * thread could not be obtained.
 */
int oracle_attention(const void *q, const int64_t *q_stride, const void *k,
                     const int64_t *k_stride, const void *v, const int64_t *v_stride, int dtype,
                     int64_t B, int64_t Lq, int64_t Hq, int64_t Lk, int64_t Hkv, int64_t Dqk,
                     int64_t Dv, const int32_t *seqlens, int causal, double scale,
                     int64_t nrows, const int64_t *rows, double *o, double *lse, int nthreads) {
    if (dtype < 0 || dtype > 2 || B < 0 || Lq < 0 || Hq <= 0 || Lk < 0 || Hkv <= 0 ||
        Dqk <= 0 || Dv <= 0 || Hq % Hkv != 0 || nrows < 0 || nthreads < 1)
        return -1;
    if (!rows && nrows != B * Hq * Lq) return -1;
    if (seqlens)
        for (int64_t b = 0; b < B; ++b)
            if (seqlens[b] < 0 || seqlens[b] > Lk) return -1;
    if (rows)
        for (int64_t r = 0; r < nrows; ++r)
            if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 ||
                rows[3 * r + 1] >= Hq || rows[3 * r + 2] < 0 || rows[3 * r + 2] >= Lq)
                return -1;
    if (nrows == 0) return 0;
    if (nthreads > nrows) nthreads = (int)nrows;

    job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return -2;
    }
    int status = 0;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        job_t *J = &jobs[t];
        J->q = q; J->k = k; J->v = v;
        J->qs = q_stride; J->ks = k_stride; J->vs = v_stride;
        J->dtype = dtype;
        J->B = B; J->Lq = Lq; J->Hq = Hq; J->Lk = Lk; J->Hkv = Hkv; J->Dqk = Dqk; J->Dv = Dv;
        J->seqlens = seqlens; J->causal = causal; J->scale = scale;
        J->nrows = nrows; J->rows = rows; J->o = o; J->lse = lse;
        J->nthreads = nthreads; J->tid = t; J->status = 0;
    }
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, worker, &jobs[t]) != 0) {
            status = -2;
            break;
        }
        ++started;
    }
    if (status == 0) {
        worker(&jobs[0]);
    }
    for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
    for (int t = 0; t < nthreads && status == 0; ++t)
        if (jobs[t].status) status = jobs[t].status;
    free(jobs);
    free(th);
    return status;
}
