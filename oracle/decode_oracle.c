/*
 * decode_oracle.c -- fp64 CPU oracle for single-token GQA decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only
 * the test suite, the smoke entry point and the benchmark's CPU-baseline leg
 * may load it.  It shares no code, header, table or constant with the CUDA
 * library; it reads the same raw input bytes (bf16 bit patterns, fp8-e4m3
 * codes, int32 index arrays) and nothing else.
 *
 * What it computes is the plain, untiled definition of attention for one
 * query token per request:
 *
 *   s_j   = sm_scale * sum_i q[b,h,i] * K_b[j, g(h), i]          j in J_b
 *   w_j   = exp(s_j - M) / sum_{j'} exp(s_j' - M),   M = max_j s_j
 *   out_i = sum_j w_j * V_b[j, g(h), i]
 *   lse   = M + ln sum_j exp(s_j - M)                 (natural log)
 *
 * Sources (web pages; section names translated):
 *  - "Forcing Flash Attention onto a TPU" (LLM internals part 5, socker-news),
 *    section "Standard causal attention": scores = q.K^T * scale, softmax over
 *    keys, times V, all in a wide float type.  For decode the single query is
 *    the last position, so the causal mask keeps every cached key.
 *  - "FlashInfer x JAX via jax-tvm-ffi" (upppp.jp), section on the three
 *    kernels: single_decode is GQA attention of one request over its KV cache;
 *    section "Applying it to Gemma 3": local layers attend to a sliding window.
 *  - "Beyond the Memory Wall" (tiptinker), section "2. FlashInfer": paged KV
 *    and FP8 KV caches.
 *  - "FlashDecoding++" explainer (abeam.tech), section "Asynchronous softmax
 *    and unified max value", and "Flashlight" (gist.science), section
 *    "Method", semantic fusion: partial softmax states over disjoint key sets
 *    combine exactly through exp(x - y) = exp(x) / exp(y).  oracle_merge is
 *    that combination written out.
 *
 * Several query tokens per request (speculative or chunked decode, the small-M
 * regime of the "FlashDecoding++" explainer, section "Flat GEMM
 * optimization"): the request's q_len newest cached keys are its query
 * tokens, and token i (position L - q_len + i) sees keys [0, L - q_len + i],
 * the causal mask of "Standard causal attention" restricted to the new rows.
 *
 * Logit soft-capping (named on "FlashInfer x JAX via jax-tvm-ffi", section
 * "Applying it to Gemma 3", as Gemma 2's, and on "Flashlight", section
 * "Results", as the Softcap variant; neither gives the formula): each
 * scaled score s becomes cap * tanh(s / cap), Gemma 2's published form.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - GQA grouping: query head h reads kv head h / (qo_heads / kv_heads).
 *  - window w > 0 keeps exactly the last w keys [L - w, L); w <= 0 keeps all.
 *  - an empty key set gives out = 0 and lse = -inf.
 *  - FP8 is e4m3 "fn" (bias 7, no infinities, S.1111.111 is NaN); a stored
 *    code c of kv head g means decode(c) * scale[g], product taken in fp64.
 *  - INT4 ("Beyond the Memory Wall", section "2. FlashInfer", names INT4
 *    KV quantization without a format): two's-complement 4-bit codes in
 *    [-8, 7], two per byte, the even element of a row in the low nibble; a
 *    code c of kv head g means c * scale[g] (one scale per kv head for K and
 *    one for V, as for FP8).
 *  - paged pool layout [num_pages, page_size, kv_heads, head_dim]; token t of
 *    request b sits in page page_table[b*stride + t/page_size], slot
 *    t % page_size.  Contiguous layout [total_tokens, kv_heads, head_dim];
 *    request b owns rows [kv_indptr[b], kv_indptr[b+1]).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Problem description.  All pointers are host memory owned by the caller. */
typedef struct {
    int32_t batch, qo_heads, kv_heads, head_dim;
    int32_t kv_kind;         /* 0: K/V are bf16 bit patterns; 1: e4m3 codes;
                                2: int4 codes, two per byte                  */
    int32_t paged;           /* 0: contiguous rows; 1: paged pool            */
    int32_t page_size;       /* paged only                                    */
    int32_t page_table_stride;
    int32_t window;          /* <= 0: all keys; > 0: last `window` keys       */
    double sm_scale;
    const uint16_t *q;       /* bf16 bits [batch, qo_heads, head_dim]         */
    const void *k, *v;       /* uint16 (bf16), uint8 (e4m3) or packed int4
                                bytes (head_dim / 2 per row), layout above   */
    const float *k_scale;    /* [kv_heads], fp8 and int4 only                 */
    const float *v_scale;    /* [kv_heads], fp8 and int4 only                 */
    const int32_t *kv_indptr;  /* [batch + 1] token counts, cumulative        */
    const int32_t *page_table; /* [batch, page_table_stride], paged only      */
    int32_t q_len;           /* query tokens per request (0 means 1); q is
                                [batch, q_len, qo_heads, head_dim]            */
    double logit_cap;        /* > 0: each scaled score s becomes
                                cap * tanh(s / cap) before the softmax       */
} oracle_problem;

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_double(uint16_t bits) {
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* e4m3 "fn": 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.
 * Exponent field 0 encodes subnormals m/8 * 2^-6; exponent 15 with mantissa
 * 7 is NaN; there is no infinity, so exponent 15 with mantissa 0..6 is an
 * ordinary normal number (the largest is 1.75 * 2^8 = 448). */
double oracle_e4m3_to_double(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Signed value of the int4 code in the low (high = 0) or high nibble of a
 * byte: two's complement, so 0x8 .. 0xF stand for -8 .. -1. */
int oracle_int4_code(uint8_t byte, int high) {
    int c = high ? (byte >> 4) & 0xF : byte & 0xF;
    return c >= 8 ? c - 16 : c;
}

/* Value of K or V element (token t of request b, kv head g, dim i), as a
 * real number. */
static double kv_element(const oracle_problem *p, const void *base,
                         const float *scale, int b, int t, int g, int i) {
    int64_t row;
    if (p->paged) {
        int32_t page = p->page_table[(int64_t)b * p->page_table_stride + t / p->page_size];
        int32_t slot = t % p->page_size;
        row = (int64_t)page * p->page_size + slot;
    } else {
        row = (int64_t)p->kv_indptr[b] + t;
    }
    int64_t idx = (row * p->kv_heads + g) * p->head_dim + i;
    if (p->kv_kind == 1)
        return oracle_e4m3_to_double(((const uint8_t *)base)[idx]) * (double)scale[g];
    if (p->kv_kind == 2)  /* head_dim is even: element idx is nibble idx & 1 of byte idx / 2 */
        return (double)oracle_int4_code(((const uint8_t *)base)[idx >> 1], (int)(idx & 1)) *
               (double)scale[g];
    return oracle_bf16_to_double(((const uint16_t *)base)[idx]);
}

static int32_t q_len_of(const oracle_problem *p) { return p->q_len > 1 ? p->q_len : 1; }

/* Visible key range [*lo, *hi) of query token i of request b.  The request's
 * q_len newest keys are its query tokens, so token i sits at position
 * L - q_len + i and sees every key up to and including itself (causal), or
 * the last `window` of them.  A token whose position would be negative
 * (L < q_len) sees nothing. */
void oracle_visible_range_q(const oracle_problem *p, int b, int i, int32_t *lo, int32_t *hi) {
    int32_t L = p->kv_indptr[b + 1] - p->kv_indptr[b];
    int32_t end = L - q_len_of(p) + i + 1;
    if (end < 0) end = 0;
    int32_t start = 0;
    if (p->window > 0 && end > p->window) start = end - p->window;
    *lo = start;
    *hi = end;
}

/* Visible key range [*lo, *hi) of request b's last query token (the only
 * one when q_len is 1). */
void oracle_visible_range(const oracle_problem *p, int b, int32_t *lo, int32_t *hi) {
    oracle_visible_range_q(p, b, q_len_of(p) - 1, lo, hi);
}

/* One (request b, query token qi, query head h): writes head_dim outputs and
 * the lse.  Scratch `s` must hold the request's visible key count.  Returns 0. */
static int decode_one(const oracle_problem *p, int b, int qi, int h, double *s,
                      double *out, double *lse) {
    const int d = p->head_dim;
    const int group = p->qo_heads / p->kv_heads;
    const int g = h / group;
    int32_t lo, hi;
    oracle_visible_range_q(p, b, qi, &lo, &hi);
    const int n = hi - lo;
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    if (n <= 0) {
        *lse = -INFINITY;
        return 0;
    }
    const uint16_t *qrow = p->q + (((int64_t)b * q_len_of(p) + qi) * p->qo_heads + h) * d;

    /* scores */
    for (int j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i)
            acc += oracle_bf16_to_double(qrow[i]) *
                   kv_element(p, p->k, p->k_scale, b, lo + j, g, i);
        s[j] = p->sm_scale * acc;
        if (p->logit_cap > 0.0) s[j] = p->logit_cap * tanh(s[j] / p->logit_cap);
    }
    /* stable softmax: max, then normaliser */
    double M = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > M) M = s[j];
    double Z = 0.0;
    for (int j = 0; j < n; ++j) Z += exp(s[j] - M);
    /* weighted sum of values */
    for (int j = 0; j < n; ++j) {
        double w = exp(s[j] - M) / Z;
        for (int i = 0; i < d; ++i)
            out[i] += w * kv_element(p, p->v, p->v_scale, b, lo + j, g, i);
    }
    *lse = M + log(Z);
    return 0;
}

/* Longest visible key range over the batch (scratch sizing). */
static int32_t max_visible(const oracle_problem *p) {
    int32_t m = 0;
    for (int b = 0; b < p->batch; ++b) {
        int32_t lo, hi;
        oracle_visible_range(p, b, &lo, &hi);
        if (hi - lo > m) m = hi - lo;
    }
    return m;
}

/* Selected (request, query token, head) rows:
 * rows[k] = (b * q_len + qi) * qo_heads + h.
 * out: [count, head_dim]; lse: [count].  Returns 0, or -1 on allocation
 * failure. */
int oracle_decode_rows(const oracle_problem *p, const int64_t *rows, int64_t count,
                       double *out, double *lse, int nthreads) {
    int32_t nmax = max_visible(p);
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(nmax > 0 ? nmax : 1));
        if (!s) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < count; ++r) {
                int64_t bq = rows[r] / p->qo_heads;
                int h = (int)(rows[r] % p->qo_heads);
                int b = (int)(bq / q_len_of(p));
                int qi = (int)(bq % q_len_of(p));
                decode_one(p, b, qi, h, s, out + r * p->head_dim, lse + r);
            }
            free(s);
        }
    }
    return failed ? -1 : 0;
}

/* Every (request, query token, head): out [batch, q_len, qo_heads, head_dim];
 * lse [batch, q_len, qo_heads]. */
int oracle_decode_all(const oracle_problem *p, double *out, double *lse, int nthreads) {
    int64_t count = (int64_t)p->batch * q_len_of(p) * p->qo_heads;
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(count > 0 ? count : 1));
    if (!rows) return -1;
    for (int64_t r = 0; r < count; ++r) rows[r] = r;
    int rc = oracle_decode_rows(p, rows, count, out, lse, nthreads);
    free(rows);
    return rc;
}

/* Exact combination of n partial states per (row, head):
 *   lse = M + ln sum_c exp(lse_c - M),   out = sum_c exp(lse_c - lse) * o_c
 * o_parts [n, rows, heads, d], lse_parts [n, rows, heads]; states whose lse is
 * -inf carry no weight; if every state is -inf the result is out = 0,
 * lse = -inf. */
void oracle_merge(const double *o_parts, const double *lse_parts, int32_t n,
                  int32_t rows, int32_t heads, int32_t d, double *out, double *lse) {
    int64_t stride = (int64_t)rows * heads;
    for (int64_t rh = 0; rh < stride; ++rh) {
        double M = -INFINITY;
        for (int c = 0; c < n; ++c)
            if (lse_parts[c * stride + rh] > M) M = lse_parts[c * stride + rh];
        double *o = out + rh * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (M == -INFINITY) {
            lse[rh] = -INFINITY;
            continue;
        }
        double Z = 0.0;
        for (int c = 0; c < n; ++c) Z += exp(lse_parts[c * stride + rh] - M);
        double L = M + log(Z);
        for (int c = 0; c < n; ++c) {
            double w = exp(lse_parts[c * stride + rh] - L);
            const double *oc = o_parts + (c * stride + rh) * d;
            for (int i = 0; i < d; ++i) o[i] += w * oc[i];
        }
        lse[rh] = L;
    }
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
