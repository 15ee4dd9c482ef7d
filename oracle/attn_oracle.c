/*
 * attn_oracle.c -- plain, slow, fp64 CPU reference for exact scaled-dot-product
 * attention forward.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; the product path never does.  It shares no
 * code, header, table or helper with the CUDA library.
 *
 * What it computes (one query row at a time, nothing blocked, fused or reordered):
 *
 *   s_j  = scale * sum_c q_c * k_jc                 for every visible key j
 *   m    = max_j s_j
 *   l    = sum_j exp(s_j - m)
 *   P_j  = exp(s_j - m) / l
 *   O_c  = sum_j P_j * v_jc
 *   LSE  = m + ln(l)
 *
 * Sources, by page and section:
 *  - "FlashAttention" (fp-ai-systems), section "The problem: the n x n score matrix":
 *    S = Q K^T, P = softmax(S), O = P V per head.
 *  - "Flash Attention -- Module 12.3" (aicurriculum), section "Definition": the same
 *    math with the 1/sqrt(d) scale, softmax(Q K^T / sqrt(d)) V; here the caller passes
 *    the scale.
 *  - "FlashAttention 1-2-3" (myaihardware), section "The Math Behind the Online Softmax
 *    Trick": the two-pass stable softmax (subtract the row maximum, exponentiate, sum,
 *    divide), which is what this file does per row.
 *  - Same page, section "FlashAttention-1": the causal mask zeroes the upper triangle.
 *    With Nq != Nkv the pages are silent; this oracle aligns the mask bottom-right:
 *    query i sees key j iff j <= i + (Nkv - Nq).  A query that sees no key gets O = 0
 *    and LSE = -inf (also a reading: the pages never reach that case).
 *  - LSE is not on the pages; it is the natural log of sum_j exp(s_j) over the scaled
 *    scores.
 *
 * Inputs are 16-bit (fp16 or bf16 bit patterns) or fp64 arrays; every 16-bit element is
 * converted exactly to double before use.  Layout: q [B,H,Nq,d], k and v [B,H,Nkv,d],
 * all contiguous with d innermost.  Outputs are fp64: o [rows, d], lse [rows].
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORC_F64 = 0, ORC_F16 = 1, ORC_BF16 = 2 };

/* IEEE binary16 -> double, exactly (normal, subnormal, zero, inf, nan). */
static double half_bits_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double r;
    if (e == 0)
        r = ldexp((double)man, -24);
    else if (e == 31)
        r = man ? NAN : INFINITY;
    else
        r = ldexp((double)(man + 1024), e - 25);
    return sign ? -r : r;
}

/* bfloat16 is the upper half of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double elem(const void* base, int dtype, size_t i) {
    if (dtype == ORC_F64) return ((const double*)base)[i];
    uint16_t bits = ((const uint16_t*)base)[i];
    return dtype == ORC_F16 ? half_bits_to_double(bits) : bf16_bits_to_double(bits);
}

typedef struct {
    const void *q, *k, *v;
    int dtype;
    double *o, *lse;
    int64_t B, H, Nq, Nkv, d;
    double scale;
    int causal;
    const int64_t* rows; /* global row ids (bh * Nq + i), or NULL for all rows */
    int64_t nrows;
    int64_t next;        /* shared work counter */
    pthread_mutex_t mu;
} job_t;

/* One query row, straight from the definition. */
static void one_row(const job_t* J, int64_t grow, double* s, double* qrow, double* out,
                    double* lse_out) {
    const int64_t d = J->d, Nq = J->Nq, Nkv = J->Nkv;
    const int64_t bh = grow / Nq, i = grow % Nq;
    int64_t last = Nkv - 1;                       /* last visible key */
    if (J->causal) {
        int64_t lim = i + (Nkv - Nq);
        if (lim < last) last = lim;
    }
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    if (last < 0) { *lse_out = -INFINITY; return; }

    for (int64_t c = 0; c < d; ++c) qrow[c] = elem(J->q, J->dtype, (size_t)(grow * d + c));

    const size_t kv0 = (size_t)(bh * Nkv * d);
    double m = -INFINITY;
    for (int64_t j = 0; j <= last; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c)
            acc += qrow[c] * elem(J->k, J->dtype, kv0 + (size_t)(j * d + c));
        s[j] = J->scale * acc;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j <= last; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int64_t j = 0; j <= last; ++j) {
        const double p = s[j] / l;
        for (int64_t c = 0; c < d; ++c)
            out[c] += p * elem(J->v, J->dtype, kv0 + (size_t)(j * d + c));
    }
    *lse_out = m + log(l);
}

static void* worker(void* arg) {
    job_t* J = (job_t*)arg;
    double* s = (double*)malloc(sizeof(double) * (size_t)(J->Nkv > 0 ? J->Nkv : 1));
    double* qrow = (double*)malloc(sizeof(double) * (size_t)J->d);
    if (!s || !qrow) { free(s); free(qrow); return (void*)1; }
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int64_t r = J->next;
        J->next += 16;
        pthread_mutex_unlock(&J->mu);
        if (r >= J->nrows) break;
        int64_t r_end = r + 16 < J->nrows ? r + 16 : J->nrows;
        for (; r < r_end; ++r) {
            int64_t grow = J->rows ? J->rows[r] : r;
            one_row(J, grow, s, qrow, J->o + r * J->d, J->lse + r);
        }
    }
    free(s);
    free(qrow);
    return NULL;
}

/* Threads used when the caller passes nthreads <= 0: the CPUs this process may run on. */
int attn_oracle_default_threads(void) {
    cpu_set_t set;
    long n = 0;
    if (sched_getaffinity(0, sizeof set, &set) == 0) n = CPU_COUNT(&set);
    if (n < 1) n = sysconf(_SC_NPROCESSORS_ONLN);
    if (n < 1) n = 1;
    if (n > 512) n = 512;
    return (int)n;
}

/*
 * Computes O and LSE for `nrows` query rows.  rows == NULL means every row of
 * [B,H,Nq] in order (nrows must then be B*H*Nq).  nthreads <= 0 uses every online
 * CPU.  Returns 0 on success, a negative value on bad arguments or allocation failure.
 */
int attn_oracle_fwd(const void* q, const void* k, const void* v, int dtype, double* o,
                    double* lse, int64_t B, int64_t H, int64_t Nq, int64_t Nkv, int64_t d,
                    double scale, int causal, const int64_t* rows, int64_t nrows,
                    int nthreads) {
    if (!q || !k || !v || !o || !lse) return -1;
    if (B <= 0 || H <= 0 || Nq <= 0 || Nkv <= 0 || d <= 0) return -2;
    if (dtype != ORC_F64 && dtype != ORC_F16 && dtype != ORC_BF16) return -3;
    if (!rows && nrows != B * H * Nq) return -4;
    if (rows)
        for (int64_t r = 0; r < nrows; ++r)
            if (rows[r] < 0 || rows[r] >= B * H * Nq) return -5;
    if (nthreads <= 0) nthreads = attn_oracle_default_threads();
    if (nthreads > 512) nthreads = 512;

    job_t J = {q, k, v, dtype, o, lse, B, H, Nq, Nkv, d, scale, causal, rows, nrows, 0,
               PTHREAD_MUTEX_INITIALIZER};
    pthread_t th[512];
    int started = 0, rc = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) worker(&J);
    for (int t = 0; t < started; ++t) {
        void* ret = NULL;
        pthread_join(th[t], &ret);
        if (ret) rc = -6;
    }
    return rc;
}

