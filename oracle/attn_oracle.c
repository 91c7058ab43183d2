/*
 * attn_oracle.c -- CPU fp64 reference for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path links, loads or
 * calls this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or helper with the CUDA sources.
 *
 * What it computes is the plain definition of attention, two passes per query row,
 * in double precision from the exactly converted bf16 inputs:
 *
 *   s_ij  = scale * sum_t q[i,t] * k[j,t]            over the keys j that row i may see
 *   m_i   = max_j s_ij,   l_i = sum_j exp(s_ij - m_i)                     (pass 1)
 *   o_i   = sum_j exp(s_ij - m_i) * v[j,:] / l_i                          (pass 2)
 *   lse_i = m_i + ln l_i
 *
 * Sources: the definition softmax(Q K^T / sqrt(d_k)) V of youngju.dev "attention
 * variants" section 1 (cost analysis) and its gqa_attention example in section 2; the
 * masked softmax of the toolsku.com MHA module (masked_fill(mask==0, -inf) before
 * softmax).  Grouped-query sharing follows the same section-2 example: K/V head g is
 * repeated R = Hq/Hkv times with repeat_interleave, so query head h reads K/V head
 * floor(h / R).  Readings where the pages are silent:
 *   - causal with Nq != Nk is bottom-right aligned: row i sees keys j <= i + Nk - Nq;
 *   - decode (one query row per sequence) sees every cached key j < L_b, unmasked;
 *   - lse is the natural log of sum_j exp(s_ij), scale included;
 *   - a row that sees no key (only L_b = 0 in decode) gives o = 0 and lse = -inf;
 *   - sliding window W (youngju.dev section 4: each token looks only at the W most
 *     recent tokens, itself included -- with W = 3, query 5 sees keys 3, 4, 5) is a
 *     lower bound on top of the causal limit: row i sees keys j with
 *     i + Nk - Nq - W < j <= i + Nk - Nq.  It is defined for causal attention only;
 *     W = 0 means no window.
 *
 * Parallelism: OpenMP over independent (batch, head, row) triples; each row is
 * computed start to finish by one thread, so the result does not depend on the
 * thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 is the upper half of an IEEE binary32; the conversion to double is exact. */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Number of keys that query row i may see (keys 0 .. count-1). */
static long visible_keys(long i, long Nq, long Nk, int causal)
{
    if (!causal) return Nk;
    long last = i + (Nk - Nq);          /* bottom-right aligned causal limit */
    if (last >= Nk) last = Nk - 1;
    return last < 0 ? 0 : last + 1;
}

/* First key that query row i may see: the sliding window's lower bound (0 without one).
 * The keys row i sees are first_key(...) .. visible_keys(...) - 1. */
static long first_key(long i, long Nq, long Nk, long window)
{
    if (window <= 0) return 0;
    long first = i + (Nk - Nq) - window + 1;
    return first > 0 ? first : 0;
}

/* One query row against keys [0, nkeys) of one K/V head; writes d outputs and lse. */
static void attend_row(const uint16_t *qrow, const uint16_t *khead, const uint16_t *vhead,
                       long nkeys, long d, double scale,
                       double *qbuf, double *s, double *orow, double *lse)
{
    for (long t = 0; t < d; ++t) qbuf[t] = bf16_bits_to_double(qrow[t]);
    for (long t = 0; t < d; ++t) orow[t] = 0.0;
    if (nkeys <= 0) { *lse = -INFINITY; return; }

    /* scores */
    for (long j = 0; j < nkeys; ++j) {
        const uint16_t *kr = khead + j * d;
        double acc = 0.0;
        for (long t = 0; t < d; ++t) acc += qbuf[t] * bf16_bits_to_double(kr[t]);
        s[j] = scale * acc;
    }
    /* pass 1: row max and normaliser */
    double m = s[0];
    for (long j = 1; j < nkeys; ++j) if (s[j] > m) m = s[j];
    double l = 0.0;
    for (long j = 0; j < nkeys; ++j) l += exp(s[j] - m);
    /* pass 2: normalised weights times V */
    for (long j = 0; j < nkeys; ++j) {
        double p = exp(s[j] - m) / l;
        const uint16_t *vr = vhead + j * d;
        for (long t = 0; t < d; ++t) orow[t] += p * bf16_bits_to_double(vr[t]);
    }
    *lse = m + log(l);
}

/*
 * Prefill / generic forward.
 *   q: (B,Hq,Nq,d) bf16 bits;  k, v: (B,Hkv,Nk,d) bf16 bits.
 *   rows: optional list of nrows query-row indices applied to every (b, h); NULL means
 *         all Nq rows (nrows is then ignored).
 *   o: (B,Hq,R,d) doubles, lse: (B,Hq,R) doubles, R = nrows or Nq.
 *   window: sliding-window width W >= 1 (causal only), or 0 for none.
 * Returns 0, or -1 on an argument error.
 */
int oracle_attn_fwd_window(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           int B, int Hq, int Hkv, int Nq, int Nk, int d,
                           double scale, int causal, int window,
                           const int32_t *rows, int nrows, double *o, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (window < 0 || (window > 0 && !causal)) return -1;
    const long R = Hq / Hkv;
    const long nr = rows ? nrows : Nq;
    const long total = (long)B * Hq * nr;
    int err = 0;
#pragma omp parallel
    {
        double *qbuf = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!qbuf || !s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long idx = 0; idx < total; ++idx) {
                long r = idx % nr;
                long bh = idx / nr;
                long h = bh % Hq;
                long b = bh / Hq;
                long g = h / R;
                long i = rows ? rows[r] : r;
                if (i < 0 || i >= Nq) { continue; }
                const uint16_t *qrow = q + (((long)b * Hq + h) * Nq + i) * d;
                const uint16_t *kh = k + ((long)b * Hkv + g) * (long)Nk * d;
                const uint16_t *vh = v + ((long)b * Hkv + g) * (long)Nk * d;
                long j0 = first_key(i, Nq, Nk, window);
                long j1 = visible_keys(i, Nq, Nk, causal);
                attend_row(qrow, kh + j0 * d, vh + j0 * d, j1 > j0 ? j1 - j0 : 0, d, scale,
                           qbuf, s, o + idx * d, lse + idx);
            }
        }
        free(qbuf);
        free(s);
    }
    return err ? -1 : 0;
}

/* The forward without a sliding window. */
int oracle_attn_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    int B, int Hq, int Hkv, int Nq, int Nk, int d,
                    double scale, int causal, const int32_t *rows, int nrows,
                    double *o, double *lse)
{
    return oracle_attn_fwd_window(q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0,
                                  rows, nrows, o, lse);
}

/*
 * Softmax weights P (B,Hq,Nq,Nk) for tiny problems, by the same two passes; masked
 * entries are exactly 0.  Used only to check that each row of P sums to one.
 */
int oracle_attn_probs_window(const uint16_t *q, const uint16_t *k,
                             int B, int Hq, int Hkv, int Nq, int Nk, int d,
                             double scale, int causal, int window, double *p)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (window < 0 || (window > 0 && !causal)) return -1;
    const long R = Hq / Hkv;
    for (long b = 0; b < B; ++b)
        for (long h = 0; h < Hq; ++h)
            for (long i = 0; i < Nq; ++i) {
                long g = h / R;
                const uint16_t *qrow = q + ((b * Hq + h) * Nq + i) * d;
                const uint16_t *kh = k + (b * Hkv + g) * (long)Nk * d;
                double *prow = p + ((b * Hq + h) * Nq + i) * (long)Nk;
                long j0 = first_key(i, Nq, Nk, window);
                long nk = visible_keys(i, Nq, Nk, causal);
                for (long j = 0; j < Nk; ++j) prow[j] = 0.0;
                if (nk <= j0) continue;
                double m = -INFINITY;
                for (long j = j0; j < nk; ++j) {
                    double acc = 0.0;
                    for (long t = 0; t < d; ++t)
                        acc += bf16_bits_to_double(qrow[t]) * bf16_bits_to_double(kh[j * d + t]);
                    prow[j] = scale * acc;
                    if (prow[j] > m) m = prow[j];
                }
                double l = 0.0;
                for (long j = j0; j < nk; ++j) l += exp(prow[j] - m);
                for (long j = j0; j < nk; ++j) prow[j] = exp(prow[j] - m) / l;
            }
    return 0;
}

/* The weights without a sliding window. */
int oracle_attn_probs(const uint16_t *q, const uint16_t *k,
                      int B, int Hq, int Hkv, int Nq, int Nk, int d,
                      double scale, int causal, double *p)
{
    return oracle_attn_probs_window(q, k, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, p);
}

/*
 * Decode over a KV cache: one query row per (b, h) against cached keys [0, L_b).
 *   q: (B,Hq,d);  kcache, vcache: (B,Hkv,Nmax,d);  seqlens: int32[B] in [0, Nmax].
 *   o: (B,Hq,d) doubles, lse: (B,Hq) doubles.
 */
int oracle_decode(const uint16_t *q, const uint16_t *kcache, const uint16_t *vcache,
                  const int32_t *seqlens, int B, int Hq, int Hkv, int Nmax, int d,
                  double scale, double *o, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nmax <= 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Nmax) return -1;
    const long R = Hq / Hkv;
    const long total = (long)B * Hq;
    int err = 0;
#pragma omp parallel
    {
        double *qbuf = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)Nmax);
        if (!qbuf || !s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long idx = 0; idx < total; ++idx) {
                long h = idx % Hq;
                long b = idx / Hq;
                long g = h / R;
                const uint16_t *kh = kcache + ((long)b * Hkv + g) * (long)Nmax * d;
                const uint16_t *vh = vcache + ((long)b * Hkv + g) * (long)Nmax * d;
                attend_row(q + idx * d, kh, vh, seqlens[b], d, scale, qbuf, s,
                           o + idx * d, lse + idx);
            }
        }
        free(qbuf);
        free(s);
    }
    return err ? -1 : 0;
}

/*
 * Decode over a paged KV cache (youngju.dev "attention variants", section 5: the cache is
 * cut into fixed-size blocks managed like virtual-memory pages).  The page layout is this
 * library's reading, the pages fix none:
 *   kpages, vpages: (num_pages, Hkv, page_size, d) -- a page holds page_size consecutive
 *                   tokens of one sequence, for every K/V head;
 *   block_table:    int32 (B, max_pages): logical page t / page_size of sequence b is
 *                   physical page block_table[b * max_pages + t / page_size], and token t
 *                   is row t % page_size of it.
 * Sequence b attends its first seqlens[b] tokens, exactly as oracle_decode does on a
 * contiguous cache: each (b, K/V head) is first gathered into a contiguous buffer.
 * Returns -1 on an argument error or a block-table entry outside [0, num_pages).
 */
int oracle_decode_paged(const uint16_t *q, const uint16_t *kpages, const uint16_t *vpages,
                        const int32_t *block_table, const int32_t *seqlens,
                        int B, int Hq, int Hkv, int num_pages, int page_size, int max_pages,
                        int d, double scale, double *o, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || num_pages <= 0 || page_size <= 0 || max_pages <= 0 ||
        d <= 0)
        return -1;
    if (Hq % Hkv != 0) return -1;
    const long cap = (long)page_size * max_pages;
    for (int b = 0; b < B; ++b) {
        if (seqlens[b] < 0 || seqlens[b] > cap) return -1;
        for (long t = 0; t < ((long)seqlens[b] + page_size - 1) / page_size; ++t) {
            int32_t pg = block_table[(long)b * max_pages + t];
            if (pg < 0 || pg >= num_pages) return -1;
        }
    }
    const long R = Hq / Hkv;
    int err = 0;
#pragma omp parallel
    {
        double *qbuf = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)cap);
        uint16_t *kg = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)cap * d);
        uint16_t *vg = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)cap * d);
        if (!qbuf || !s || !kg || !vg) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bg = 0; bg < (long)B * Hkv; ++bg) {
                long b = bg / Hkv, g = bg % Hkv;
                long L = seqlens[b];
                for (long t = 0; t < L; ++t) {
                    long page = block_table[b * max_pages + t / page_size];
                    long row = t % page_size;
                    const long src = ((page * Hkv + g) * page_size + row) * d;
                    memcpy(kg + t * d, kpages + src, sizeof(uint16_t) * (size_t)d);
                    memcpy(vg + t * d, vpages + src, sizeof(uint16_t) * (size_t)d);
                }
                for (long h = g * R; h < (g + 1) * R; ++h) {
                    long idx = b * Hq + h;
                    attend_row(q + idx * d, kg, vg, L, d, scale, qbuf, s, o + idx * d, lse + idx);
                }
            }
        }
        free(qbuf);
        free(s);
        free(kg);
        free(vg);
    }
    return err ? -1 : 0;
}

/*
 * OCP FP8 E4M3 (the "e4m3fn" variant): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits.  Exponent field 0 holds the subnormals (m / 8) * 2^-6; exponent 15 with mantissa 7
 * is NaN; there are no infinities, so the largest magnitude is 1.75 * 2^8 = 448.
 */
double oracle_e4m3_to_double(uint8_t x)
{
    int e = (x >> 3) & 15, m = x & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return (x & 0x80) ? -v : v;
}

/* One query row against nkeys dequantized key/value rows (doubles, row-major nkeys x d):
 * the same two passes as attend_row. */
static void attend_row_dq(const uint16_t *qrow, const double *kd, const double *vd, long nkeys,
                          long d, double scale, double *qbuf, double *s, double *orow,
                          double *lse)
{
    for (long t = 0; t < d; ++t) qbuf[t] = bf16_bits_to_double(qrow[t]);
    for (long t = 0; t < d; ++t) orow[t] = 0.0;
    if (nkeys <= 0) { *lse = -INFINITY; return; }
    for (long j = 0; j < nkeys; ++j) {
        double acc = 0.0;
        for (long t = 0; t < d; ++t) acc += qbuf[t] * kd[j * d + t];
        s[j] = scale * acc;
    }
    double mx = s[0];
    for (long j = 1; j < nkeys; ++j) if (s[j] > mx) mx = s[j];
    double sum = 0.0;
    for (long j = 0; j < nkeys; ++j) sum += exp(s[j] - mx);
    for (long j = 0; j < nkeys; ++j) {
        double w = exp(s[j] - mx) / sum;
        for (long t = 0; t < d; ++t) orow[t] += w * vd[j * d + t];
    }
    *lse = mx + log(sum);
}

/*
 * Decode over an FP8 (E4M3) KV cache.  The pages name FP8 KV caches (youngju.dev
 * "attention variants", sections 5 and 7) but fix no scale convention; this library's
 * reading is one dequantization scale per K/V head for K and one for V:
 *   key   j of head g = k_scale[g] * e4m3(kcache[b, g, j, :])
 *   value j of head g = v_scale[g] * e4m3(vcache[b, g, j, :])
 * (a single per-tensor scale is the case of equal entries).  Everything else is
 * oracle_decode: q bf16 (B,Hq,d), caches (B,Hkv,Nmax,d) bytes, seqlens in [0, Nmax].
 */
int oracle_decode_fp8(const uint16_t *q, const uint8_t *kcache, const uint8_t *vcache,
                      const float *k_scale, const float *v_scale, const int32_t *seqlens,
                      int B, int Hq, int Hkv, int Nmax, int d, double scale, double *o,
                      double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nmax <= 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Nmax) return -1;
    const long R = Hq / Hkv;
    int err = 0;
#pragma omp parallel
    {
        double *qbuf = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)Nmax);
        double *kd = (double *)malloc(sizeof(double) * (size_t)Nmax * d);
        double *vd = (double *)malloc(sizeof(double) * (size_t)Nmax * d);
        if (!qbuf || !s || !kd || !vd) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long bg = 0; bg < (long)B * Hkv; ++bg) {
                long b = bg / Hkv, g = bg % Hkv;
                long L = seqlens[b];
                const uint8_t *kh = kcache + bg * (long)Nmax * d;
                const uint8_t *vh = vcache + bg * (long)Nmax * d;
                for (long e = 0; e < L * d; ++e) {
                    kd[e] = (double)k_scale[g] * oracle_e4m3_to_double(kh[e]);
                    vd[e] = (double)v_scale[g] * oracle_e4m3_to_double(vh[e]);
                }
                for (long h = g * R; h < (g + 1) * R; ++h) {
                    long idx = b * Hq + h;
                    attend_row_dq(q + idx * d, kd, vd, L, d, scale, qbuf, s, o + idx * d, lse + idx);
                }
            }
        }
        free(qbuf);
        free(s);
        free(kd);
        free(vd);
    }
    return err ? -1 : 0;
}

/*
 * Prefill over FP8 (E4M3) Q, K and V.  The pages list FP8 among the data types of
 * FlashAttention-3 (toolsku.com, the FlashAttention generations table) without a scale
 * convention; this library's reading is the one of the FP8 KV cache above, extended to Q:
 *   q[b, h, i, :] = q_scale[h] * e4m3(q8[b, h, i, :])        (one scale per query head)
 *   k[b, g, j, :] = k_scale[g] * e4m3(k8[b, g, j, :])        (one per K/V head)
 *   v[b, g, j, :] = v_scale[g] * e4m3(v8[b, g, j, :])
 * and the result is the attention of these dequantized tensors: the same two passes as
 * attend_row, written out over the dequantized values, with the causal and sliding-window
 * rules of oracle_attn_fwd_window.  Layouts as there, with bytes in place of bf16 bits.
 */
static void attend_row_fp8(const uint8_t *qrow, double qs, const uint8_t *khead, double ks,
                           const uint8_t *vhead, double vs, long nkeys, long d, double scale,
                           const double *lut, double *qbuf, double *s, double *orow, double *lse)
{
    for (long t = 0; t < d; ++t) qbuf[t] = qs * lut[qrow[t]];
    for (long t = 0; t < d; ++t) orow[t] = 0.0;
    if (nkeys <= 0) { *lse = -INFINITY; return; }
    for (long j = 0; j < nkeys; ++j) {
        const uint8_t *kr = khead + j * d;
        double acc = 0.0;
        for (long t = 0; t < d; ++t) acc += qbuf[t] * (ks * lut[kr[t]]);
        s[j] = scale * acc;
    }
    double m = s[0];
    for (long j = 1; j < nkeys; ++j) if (s[j] > m) m = s[j];
    double l = 0.0;
    for (long j = 0; j < nkeys; ++j) l += exp(s[j] - m);
    for (long j = 0; j < nkeys; ++j) {
        double p = exp(s[j] - m) / l;
        const uint8_t *vr = vhead + j * d;
        for (long t = 0; t < d; ++t) orow[t] += p * (vs * lut[vr[t]]);
    }
    *lse = m + log(l);
}

int oracle_attn_fwd_fp8(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                        const float *q_scale, const float *k_scale, const float *v_scale,
                        int B, int Hq, int Hkv, int Nq, int Nk, int d, double scale, int causal,
                        int window, const int32_t *rows, int nrows, double *o, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (window < 0 || (window > 0 && !causal)) return -1;
    double lut[256];
    for (int x = 0; x < 256; ++x) lut[x] = oracle_e4m3_to_double((uint8_t)x);
    const long R = Hq / Hkv;
    const long nr = rows ? nrows : Nq;
    const long total = (long)B * Hq * nr;
    int err = 0;
#pragma omp parallel
    {
        double *qbuf = (double *)malloc(sizeof(double) * (size_t)d);
        double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!qbuf || !s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long idx = 0; idx < total; ++idx) {
                long r = idx % nr;
                long bh = idx / nr;
                long h = bh % Hq;
                long b = bh / Hq;
                long g = h / R;
                long i = rows ? rows[r] : r;
                if (i < 0 || i >= Nq) { continue; }
                const uint8_t *qrow = q + (((long)b * Hq + h) * Nq + i) * d;
                const uint8_t *kh = k + ((long)b * Hkv + g) * (long)Nk * d;
                const uint8_t *vh = v + ((long)b * Hkv + g) * (long)Nk * d;
                long j0 = first_key(i, Nq, Nk, window);
                long j1 = visible_keys(i, Nq, Nk, causal);
                attend_row_fp8(qrow, q_scale[h], kh + j0 * d, k_scale[g], vh + j0 * d, v_scale[g],
                               j1 > j0 ? j1 - j0 : 0, d, scale, lut, qbuf, s, o + idx * d, lse + idx);
            }
        }
        free(qbuf);
        free(s);
    }
    return err ? -1 : 0;
}

/* Number of OpenMP threads a parallel region would use (for reporting). */
int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
