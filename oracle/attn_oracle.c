/*
 * attn_oracle.c -- plain, slow fp64 CPU oracle for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference arm of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path and never imports it.
 *
 * What it computes is the plain definition of standard attention, which the
 * tiled method reaches exactly up to rounding order:
 *
 *   "Phase 08 -- Inference Optimization at Depth", Lab 01, Steps (1): standard
 *   attention is the reference; screna.ai interview page, FlashAttention answer:
 *   S = Q K^T and P = softmax(S), with O = P V.  Online-softmax answer on the
 *   same page: softmax exponentiates every score and divides by their sum.
 *
 *   For each batch b and query head h, with key/value head g = h / (Hq/Hkv)
 *   (grouped-query sharing, screna.ai MHA/MQA/GQA answer: heads are grouped and
 *   each group shares one K and V; contiguous groups):
 *     s_ij = scale * sum_c q[b,h,i,c] * k[b,g,j,c] + a_h * (j - i)   for j in V_i
 *     V_i  = { j : j <= i } when causal (Lab 01 step 4), else { 0 .. Nk-1 },
 *            further limited to { j : i - j < W } by a sliding window W > 0
 *   The last two are the Lab 01 "Extensions" (sliding-window attention as in
 *   Mistral, ALiBi bias), which the page only names; read plainly, a window of
 *   W keeps the W most recent keys (i-W < j <= i) and ALiBi adds a per-head
 *   linear bias a_h * (j - i) (slope a_h >= 0 given by the caller) to the
 *   scaled score.  a_h = 0 and W = 0 give plain attention.
 *     m_i  = max_{j in V_i} s_ij
 *     l_i  = sum_{j in V_i} exp(s_ij - m_i)
 *     O_i  = sum_{j in V_i} exp(s_ij - m_i) / l_i * v[b,g,j,:]
 *     L_i  = m_i + ln(l_i)        (the logsumexp "L", Concepts: backward)
 *   An empty V_i (a decode sequence of length 0) gives O_i = 0, L_i = -inf.
 *
 * oracle_attn materialises S for one (b, h) at a time (N x N doubles), takes
 * the row maximum, then exponentials and row sums, then P V -- the "standard
 * attention" of the pages, O(N^2) memory.  oracle_attn_rows evaluates the same
 * definition one requested row at a time, for sampled checks at full size.
 * oracle_decode_paged gathers a sequence's keys and values from the page pool
 * through the block table (Lab 03 step 4: pages reached through an
 * indirection table), then evaluates the same definition for its one query.
 * oracle_decode_paged_q8 is the same over 8-bit pages (E4M3 or INT8) with one
 * scale per (page, kv head): each element is dequantised to fp64 first.
 * oracle_prefill_paged evaluates a chunk of queries at the end of each
 * sequence against its paged keys (chunked prefill, causal from the end).
 * oracle_attn_bwd (and its sampled forms _dq_rows, _dkv_rows) evaluates the
 * gradients of the same definition with respect to Q, K and V.
 *
 * Inputs are float (the exact values the GPU sees: fp32, or bf16 upcast) or,
 * for the page pool, raw bf16 bit patterns; arithmetic is double throughout.
 * Return value: 0 on success, -1 on a bad argument, -2 on allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_double(uint16_t bits)
{
    /* A bf16 value is the top half of an IEEE binary32 pattern. */
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Softmax-weighted sum of the rows of v for one query, given its scores.
 * s has n entries and is overwritten with the unnormalised weights. */
static void softmax_row_times_v(double *s, int n, const double *v, int d,
                                double *o_row, double *lse)
{
    int j, c;
    double m, l;
    for (c = 0; c < d; ++c) o_row[c] = 0.0;
    if (n == 0) { *lse = -INFINITY; return; }
    m = s[0];
    for (j = 1; j < n; ++j) if (s[j] > m) m = s[j];
    l = 0.0;
    for (j = 0; j < n; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
    for (j = 0; j < n; ++j) {
        double p = s[j] / l;
        const double *vj = v + (size_t)j * d;
        for (c = 0; c < d; ++c) o_row[c] += p * vj[c];
    }
    *lse = m + log(l);
}

static int check_dims(int B, int Hq, int Hkv, int Nq, int Nk, int d)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    return 0;
}

/* Visible key range [*lo, *hi) of query i. */
static void visible_range(int i, int Nk, int causal, int window, int *lo, int *hi)
{
    *hi = causal ? ((i + 1 < Nk) ? i + 1 : Nk) : Nk;
    *lo = (window > 0 && i - window + 1 > 0) ? i - window + 1 : 0;
    if (*lo > *hi) *lo = *hi;
}

/* Full evaluation: q [B,Hq,Nq,d], k,v [B,Hkv,Nk,d] (float), o [B,Hq,Nq,d],
 * lse [B,Hq,Nq] (double).  Causal means key j is visible to query i iff j <= i;
 * window W > 0 additionally requires i - j < W; slopes (Hq values, or NULL)
 * add the ALiBi bias slopes[h] * (j - i). */
int oracle_attn(const float *q, const float *k, const float *v,
                double *o, double *lse,
                int B, int Hq, int Hkv, int Nq, int Nk, int d,
                double scale, int causal, int window, const double *slopes,
                int nthreads)
{
    int b, h, G;
    double *S, *Kd, *Vd, *Qd;
    if (check_dims(B, Hq, Hkv, Nq, Nk, d) || window < 0) return -1;
    if (!q || !k || !v || !o || !lse) return -1;
    G = Hq / Hkv;
    if (nthreads <= 0) nthreads = 1;
    S = (double *)malloc(sizeof(double) * ((size_t)Nq * Nk + 1));
    Kd = (double *)malloc(sizeof(double) * ((size_t)Nk * d + 1));
    Vd = (double *)malloc(sizeof(double) * ((size_t)Nk * d + 1));
    Qd = (double *)malloc(sizeof(double) * ((size_t)Nq * d + 1));
    if (!S || !Kd || !Vd || !Qd) { free(S); free(Kd); free(Vd); free(Qd); return -2; }

    for (b = 0; b < B; ++b) {
        for (h = 0; h < Hq; ++h) {
            int g = h / G;
            const float *qh = q + ((size_t)b * Hq + h) * (size_t)Nq * d;
            const float *kh = k + ((size_t)b * Hkv + g) * (size_t)Nk * d;
            const float *vh = v + ((size_t)b * Hkv + g) * (size_t)Nk * d;
            double *oh = o + ((size_t)b * Hq + h) * (size_t)Nq * d;
            double *lh = lse + ((size_t)b * Hq + h) * (size_t)Nq;
            long i;
            for (i = 0; i < (long)Nq * d; ++i) Qd[i] = (double)qh[i];
            for (i = 0; i < (long)Nk * d; ++i) { Kd[i] = (double)kh[i]; Vd[i] = (double)vh[i]; }

            /* S = scale * Q K^T (+ ALiBi bias), the whole Nq x Nk matrix of this head. */
            #pragma omp parallel for num_threads(nthreads) schedule(static)
            for (i = 0; i < Nq; ++i) {
                int j, c;
                for (j = 0; j < Nk; ++j) {
                    double acc = 0.0;
                    for (c = 0; c < d; ++c) acc += Qd[(size_t)i * d + c] * Kd[(size_t)j * d + c];
                    S[(size_t)i * Nk + j] = scale * acc;
                    if (slopes) S[(size_t)i * Nk + j] += slopes[h] * (double)(j - i);
                }
            }
            /* Row-wise softmax over the visible keys, then P V and L. */
            #pragma omp parallel for num_threads(nthreads) schedule(static)
            for (i = 0; i < Nq; ++i) {
                int lo, hi;
                visible_range((int)i, Nk, causal, window, &lo, &hi);
                softmax_row_times_v(S + (size_t)i * Nk + lo, hi - lo, Vd + (size_t)lo * d, d,
                                    oh + (size_t)i * d, lh + i);
            }
        }
    }
    free(S); free(Kd); free(Vd); free(Qd);
    return 0;
}

/* Selected rows only.  rows[r] = (b*Hq + h)*Nq + i.  o_rows [nrows,d],
 * lse_rows [nrows].  Same definition, one row at a time. */
int oracle_attn_rows(const float *q, const float *k, const float *v,
                     double *o_rows, double *lse_rows,
                     int B, int Hq, int Hkv, int Nq, int Nk, int d,
                     double scale, int causal, int window, const double *slopes,
                     const int64_t *rows, int nrows, int nthreads)
{
    int G, r, bad = 0;
    if (check_dims(B, Hq, Hkv, Nq, Nk, d) || window < 0) return -1;
    if (!q || !k || !v || !o_rows || !lse_rows || (!rows && nrows > 0) || nrows < 0) return -1;
    for (r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * Hq * Nq) return -1;
    G = Hq / Hkv;
    if (nthreads <= 0) nthreads = 1;

    #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1) reduction(|:bad)
    for (r = 0; r < nrows; ++r) {
        int64_t id = rows[r];
        int i = (int)(id % Nq);
        int bh = (int)(id / Nq);
        int h = bh % Hq, b = bh / Hq, g = h / G;
        int lo, hi, n;
        const float *qi = q + (((size_t)b * Hq + h) * Nq + i) * (size_t)d;
        const float *kh = k + ((size_t)b * Hkv + g) * (size_t)Nk * d;
        const float *vh = v + ((size_t)b * Hkv + g) * (size_t)Nk * d;
        double *s, *vd;
        int j, c;
        visible_range(i, Nk, causal, window, &lo, &hi);
        n = hi - lo;
        s = (double *)malloc(sizeof(double) * ((size_t)n + 1));
        vd = (double *)malloc(sizeof(double) * ((size_t)n * d + 1));
        if (!s || !vd) { free(s); free(vd); bad = 1; continue; }
        for (j = lo; j < hi; ++j) {
            double acc = 0.0;
            for (c = 0; c < d; ++c) acc += (double)qi[c] * (double)kh[(size_t)j * d + c];
            s[j - lo] = scale * acc + (slopes ? slopes[h] * (double)(j - i) : 0.0);
            for (c = 0; c < d; ++c) vd[(size_t)(j - lo) * d + c] = (double)vh[(size_t)j * d + c];
        }
        softmax_row_times_v(s, n, vd, d, o_rows + (size_t)r * d, lse_rows + r);
        free(s); free(vd);
    }
    return bad ? -2 : 0;
}

/* Single-token decode over a paged KV cache, for the sequences listed in
 * seq_ids.  q [S,Hq,d] float; k_pages, v_pages [num_pages,Hkv,page_size,d] as
 * bf16 bit patterns; block_table [S,max_blocks]; seq_lens [S].
 * Token t of sequence s lives in page block_table[s, t / page_size], slot
 * t % page_size.  o [nseq,Hq,d], lse [nseq,Hq].  Returns -1 if a page id the
 * sequence needs is outside [0, num_pages) or a length is out of range. */
int oracle_decode_paged(const float *q, const uint16_t *k_pages, const uint16_t *v_pages,
                        const int32_t *block_table, const int32_t *seq_lens,
                        double *o, double *lse,
                        int S, int Hq, int Hkv, int d, int page_size, int max_blocks,
                        int num_pages, double scale,
                        const int32_t *seq_ids, int nseq, int nthreads)
{
    int G, r, bad = 0;
    if (S <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || page_size <= 0 || max_blocks <= 0 ||
        num_pages <= 0 || Hq % Hkv != 0 || nseq < 0) return -1;
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || !lse ||
        (!seq_ids && nseq > 0)) return -1;
    G = Hq / Hkv;
    for (r = 0; r < nseq; ++r) {
        int s = seq_ids[r], t, len;
        if (s < 0 || s >= S) return -1;
        len = seq_lens[s];
        if (len < 0 || len > max_blocks * page_size) return -1;
        for (t = 0; t < len; t += page_size) {
            int32_t p = block_table[(size_t)s * max_blocks + t / page_size];
            if (p < 0 || p >= num_pages) return -1;
        }
    }
    if (nthreads <= 0) nthreads = 1;

    #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1) reduction(|:bad)
    for (r = 0; r < nseq * Hkv; ++r) {
        int s = seq_ids[r / Hkv], g = r % Hkv;
        int len = seq_lens[s];
        int t, c, hh;
        double *kd = (double *)malloc(sizeof(double) * ((size_t)len * d + 1));
        double *vd = (double *)malloc(sizeof(double) * ((size_t)len * d + 1));
        double *sc = (double *)malloc(sizeof(double) * ((size_t)len + 1));
        if (!kd || !vd || !sc) { free(kd); free(vd); free(sc); bad = 1; continue; }
        /* Gather: follow the block table to contiguous [len, d] keys/values. */
        for (t = 0; t < len; ++t) {
            int32_t p = block_table[(size_t)s * max_blocks + t / page_size];
            size_t base = (((size_t)p * Hkv + g) * page_size + (t % page_size)) * (size_t)d;
            for (c = 0; c < d; ++c) {
                kd[(size_t)t * d + c] = bf16_bits_to_double(k_pages[base + c]);
                vd[(size_t)t * d + c] = bf16_bits_to_double(v_pages[base + c]);
            }
        }
        for (hh = 0; hh < G; ++hh) {
            int h = g * G + hh;
            const float *qs = q + ((size_t)s * Hq + h) * (size_t)d;
            for (t = 0; t < len; ++t) {
                double acc = 0.0;
                for (c = 0; c < d; ++c) acc += (double)qs[c] * kd[(size_t)t * d + c];
                sc[t] = scale * acc;
            }
            softmax_row_times_v(sc, len, vd, d,
                                o + ((size_t)(r / Hkv) * Hq + h) * (size_t)d,
                                lse + (size_t)(r / Hkv) * Hq + h);
        }
        free(kd); free(vd); free(sc);
    }
    return bad ? -2 : 0;
}

/* An OCP FP8 E4M3 ("e4m3fn") byte: 1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there
 * is no infinity.  Written from the format's definition. */
static double e4m3_to_double(uint8_t b)
{
    int sign = (b >> 7) & 1, e = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Chunked prefill over the paged cache ("Phase 08" page, Concepts: chunked
 * prefill splits a long prompt over several steps; Lab 03 Extensions: add
 * chunked prefill; paged attention as above).  Read plainly: sequence s holds
 * seq_lens[s] tokens in its pages, of which the last qlen_s = cu_q[s+1] - cu_q[s]
 * are the current chunk's queries (their K/V already written to the cache).
 * Query t of the chunk sits at position ctx_s + t, ctx_s = seq_lens[s] - qlen_s,
 * and sees keys 0 .. ctx_s + t (causal, aligned to the end of the keys).
 * q [T,Hq,d] float (T = cu_q[S], token-major), o [T,Hq,d], lse [T,Hq] double. */
int oracle_prefill_paged(const float *q, const uint16_t *k_pages, const uint16_t *v_pages,
                         const int32_t *block_table, const int32_t *seq_lens,
                         const int32_t *cu_q, double *o, double *lse,
                         int S, int Hq, int Hkv, int d, int page_size, int max_blocks,
                         int num_pages, double scale, int nthreads)
{
    int G, s, bad = 0, T;
    if (S <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || page_size <= 0 || max_blocks <= 0 ||
        num_pages <= 0 || Hq % Hkv != 0) return -1;
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !cu_q || !o || !lse) return -1;
    if (cu_q[0] != 0) return -1;
    for (s = 0; s < S; ++s) {
        int len = seq_lens[s], ql = cu_q[s + 1] - cu_q[s], t;
        if (ql < 0 || len < ql || len > max_blocks * page_size) return -1;
        for (t = 0; t < len; t += page_size) {
            int32_t p = block_table[(size_t)s * max_blocks + t / page_size];
            if (p < 0 || p >= num_pages) return -1;
        }
    }
    G = Hq / Hkv;
    T = cu_q[S];
    if (nthreads <= 0) nthreads = 1;
    (void)T;

    #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1) reduction(|:bad)
    for (s = 0; s < S * Hkv; ++s) {
        int seq = s / Hkv, g = s % Hkv;
        int len = seq_lens[seq], q0 = cu_q[seq], ql = cu_q[seq + 1] - cu_q[seq];
        int ctx = len - ql, t, c, hh;
        double *kd = (double *)malloc(sizeof(double) * ((size_t)len * d + 1));
        double *vd = (double *)malloc(sizeof(double) * ((size_t)len * d + 1));
        double *sc = (double *)malloc(sizeof(double) * ((size_t)len + 1));
        if (!kd || !vd || !sc) { free(kd); free(vd); free(sc); bad = 1; continue; }
        for (t = 0; t < len; ++t) {
            int32_t p = block_table[(size_t)seq * max_blocks + t / page_size];
            size_t base = (((size_t)p * Hkv + g) * page_size + (t % page_size)) * (size_t)d;
            for (c = 0; c < d; ++c) {
                kd[(size_t)t * d + c] = bf16_bits_to_double(k_pages[base + c]);
                vd[(size_t)t * d + c] = bf16_bits_to_double(v_pages[base + c]);
            }
        }
        for (hh = 0; hh < G; ++hh) {
            int h = g * G + hh;
            for (t = 0; t < ql; ++t) {
                const float *qt = q + ((size_t)(q0 + t) * Hq + h) * (size_t)d;
                int nvis = ctx + t + 1, j;
                for (j = 0; j < nvis; ++j) {
                    double acc = 0.0;
                    for (c = 0; c < d; ++c) acc += (double)qt[c] * kd[(size_t)j * d + c];
                    sc[j] = scale * acc;
                }
                softmax_row_times_v(sc, nvis, vd, d, o + ((size_t)(q0 + t) * Hq + h) * (size_t)d,
                                    lse + (size_t)(q0 + t) * Hq + h);
            }
        }
        free(kd); free(vd); free(sc);
    }
    return bad ? -2 : 0;
}

/* ------------------------------------------------------------------ backward
 *
 * The gradients of the attention of one head with respect to its inputs, given
 * the output gradient dO ("Phase 08" page, Concepts: FlashAttention backward;
 * Lab 01 step 6: a backward pass that keeps only O and L; quiz question on
 * recomputation).  They follow from the chain rule on the definition above:
 *   P_ij  = exp(s_ij - L_i) for j in V_i, 0 elsewhere
 *   dV_j  = sum_i P_ij dO_i                       (O = P V)
 *   dP_ij = dO_i . v_j
 *   D_i   = sum_j P_ij dP_ij                      (= dO_i . O_i)
 *   dS_ij = P_ij (dP_ij - D_i)                    (softmax Jacobian)
 *   dQ_i  = scale * sum_j dS_ij k_j,   dK_j = scale * sum_i dS_ij q_i
 * The ALiBi bias does not depend on Q or K and drops out of the chain.  With
 * grouped heads, dK and dV of a K/V head sum the contributions of every query
 * head of its group.  Nq = Nk = N (self-attention prefill).
 */

/* Scores of query i (q row qi) against keys [lo, hi) into s[j - lo]; returns
 * the row's logsumexp. */
static double score_row(const double *qi, const double *Kd, int lo, int hi, int d, double scale,
                        double slope, int i, double *s)
{
    int j, c;
    double m = -INFINITY, l = 0.0;
    for (j = lo; j < hi; ++j) {
        double acc = 0.0;
        for (c = 0; c < d; ++c) acc += qi[c] * Kd[(size_t)j * d + c];
        s[j - lo] = scale * acc + slope * (double)(j - i);
        if (s[j - lo] > m) m = s[j - lo];
    }
    if (hi <= lo) return -INFINITY;
    for (j = lo; j < hi; ++j) l += exp(s[j - lo] - m);
    return m + log(l);
}

/* Full backward: q, dout [B,Hq,N,d], k, v [B,Hkv,N,d] (float); dq [B,Hq,N,d],
 * dk, dv [B,Hkv,N,d] (double, written).  Materialises P and dS of one head at a
 * time (N x N doubles each). */
int oracle_attn_bwd(const float *q, const float *k, const float *v, const float *dout,
                    double *dq, double *dk, double *dv,
                    int B, int Hq, int Hkv, int N, int d,
                    double scale, int causal, int window, const double *slopes,
                    int nthreads)
{
    int b, h, G;
    double *P, *dS, *Qd, *Kd, *Vd, *dOd;
    if (check_dims(B, Hq, Hkv, N, N, d) || window < 0) return -1;
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    G = Hq / Hkv;
    if (nthreads <= 0) nthreads = 1;
    P = (double *)malloc(sizeof(double) * ((size_t)N * N + 1));
    dS = (double *)malloc(sizeof(double) * ((size_t)N * N + 1));
    Qd = (double *)malloc(sizeof(double) * ((size_t)N * d + 1));
    Kd = (double *)malloc(sizeof(double) * ((size_t)N * d + 1));
    Vd = (double *)malloc(sizeof(double) * ((size_t)N * d + 1));
    dOd = (double *)malloc(sizeof(double) * ((size_t)N * d + 1));
    if (!P || !dS || !Qd || !Kd || !Vd || !dOd) {
        free(P); free(dS); free(Qd); free(Kd); free(Vd); free(dOd);
        return -2;
    }
    memset(dk, 0, sizeof(double) * (size_t)B * Hkv * N * d);
    memset(dv, 0, sizeof(double) * (size_t)B * Hkv * N * d);

    for (b = 0; b < B; ++b) {
        for (h = 0; h < Hq; ++h) {
            int g = h / G;
            const size_t qoff = ((size_t)b * Hq + h) * (size_t)N * d;
            const size_t koff = ((size_t)b * Hkv + g) * (size_t)N * d;
            const double slope = slopes ? slopes[h] : 0.0;
            long i;
            for (i = 0; i < (long)N * d; ++i) {
                Qd[i] = (double)q[qoff + i];
                dOd[i] = (double)dout[qoff + i];
                Kd[i] = (double)k[koff + i];
                Vd[i] = (double)v[koff + i];
            }
            /* Rows: P, dS and dQ. */
            #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 4)
            for (i = 0; i < N; ++i) {
                int j, c, lo, hi;
                double L, D = 0.0;
                double *Pi = P + (size_t)i * N, *dSi = dS + (size_t)i * N;
                double *dqi = dq + qoff + (size_t)i * d;
                visible_range((int)i, N, causal, window, &lo, &hi);
                for (j = 0; j < N; ++j) { Pi[j] = 0.0; dSi[j] = 0.0; }
                L = score_row(Qd + (size_t)i * d, Kd, lo, hi, d, scale, slope, (int)i, Pi + lo);
                for (j = lo; j < hi; ++j) Pi[j] = exp(Pi[j] - L);
                for (j = lo; j < hi; ++j) {
                    double dp = 0.0;
                    for (c = 0; c < d; ++c) dp += dOd[(size_t)i * d + c] * Vd[(size_t)j * d + c];
                    dSi[j] = dp;                     /* dP for now */
                    D += Pi[j] * dp;
                }
                for (j = lo; j < hi; ++j) dSi[j] = Pi[j] * (dSi[j] - D);
                for (c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (j = lo; j < hi; ++j) acc += dSi[j] * Kd[(size_t)j * d + c];
                    dqi[c] = scale * acc;
                }
            }
            /* Columns: dK and dV of the K/V head, summed over its query heads. */
            #pragma omp parallel for num_threads(nthreads) schedule(static)
            for (i = 0; i < N; ++i) {      /* i is the key index here */
                int r, c;
                double *dkj = dk + koff + (size_t)i * d, *dvj = dv + koff + (size_t)i * d;
                for (c = 0; c < d; ++c) {
                    double ak = 0.0, av = 0.0;
                    for (r = 0; r < N; ++r) {
                        ak += dS[(size_t)r * N + i] * Qd[(size_t)r * d + c];
                        av += P[(size_t)r * N + i] * dOd[(size_t)r * d + c];
                    }
                    dkj[c] += scale * ak;
                    dvj[c] += av;
                }
            }
        }
    }
    free(P); free(dS); free(Qd); free(Kd); free(Vd); free(dOd);
    return 0;
}

/* dQ for selected rows (rows[r] = (b*Hq + h)*N + i), one row at a time. */
int oracle_attn_bwd_dq_rows(const float *q, const float *k, const float *v, const float *dout,
                            double *dq_rows, int B, int Hq, int Hkv, int N, int d,
                            double scale, int causal, int window, const double *slopes,
                            const int64_t *rows, int nrows, int nthreads)
{
    int r, G, bad = 0;
    if (check_dims(B, Hq, Hkv, N, N, d) || window < 0 || nrows < 0) return -1;
    if (!q || !k || !v || !dout || !dq_rows || (!rows && nrows > 0)) return -1;
    for (r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * Hq * N) return -1;
    G = Hq / Hkv;
    if (nthreads <= 0) nthreads = 1;
    #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1) reduction(|:bad)
    for (r = 0; r < nrows; ++r) {
        int64_t bh = rows[r] / N;
        int i = (int)(rows[r] % N), b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
        int j, c, lo, hi;
        const float *qi = q + (size_t)rows[r] * d, *doi = dout + (size_t)rows[r] * d;
        const float *kh = k + ((size_t)b * Hkv + g) * (size_t)N * d;
        const float *vh = v + ((size_t)b * Hkv + g) * (size_t)N * d;
        double *Kd = (double *)malloc(sizeof(double) * ((size_t)N * d + 1));
        double *s = (double *)malloc(sizeof(double) * ((size_t)N + 1));
        double *dp = (double *)malloc(sizeof(double) * ((size_t)N + 1));
        double qd[512], L, D = 0.0;
        if (!Kd || !s || !dp || d > 512) { free(Kd); free(s); free(dp); bad = 1; continue; }
        for (c = 0; c < d; ++c) qd[c] = (double)qi[c];
        visible_range(i, N, causal, window, &lo, &hi);
        for (j = lo; j < hi; ++j)
            for (c = 0; c < d; ++c) Kd[(size_t)j * d + c] = (double)kh[(size_t)j * d + c];
        L = score_row(qd, Kd, lo, hi, d, scale, slopes ? slopes[h] : 0.0, i, s);
        for (j = lo; j < hi; ++j) {
            double acc = 0.0;
            s[j - lo] = exp(s[j - lo] - L);
            for (c = 0; c < d; ++c) acc += (double)doi[c] * (double)vh[(size_t)j * d + c];
            dp[j - lo] = acc;
            D += s[j - lo] * acc;
        }
        for (c = 0; c < d; ++c) {
            double acc = 0.0;
            for (j = lo; j < hi; ++j) acc += s[j - lo] * (dp[j - lo] - D) * Kd[(size_t)j * d + c];
            dq_rows[(size_t)r * d + c] = scale * acc;
        }
        free(Kd); free(s); free(dp);
    }
    return bad ? -2 : 0;
}

/* dK and dV for selected keys (keys[r] = (b*Hkv + g)*N + j).  Every query row
 * of the K/V head's group needs its L_i and D_i, computed here from their
 * definitions for each (b, g) the request touches. */
int oracle_attn_bwd_dkv_rows(const float *q, const float *k, const float *v, const float *dout,
                             double *dk_rows, double *dv_rows, int B, int Hq, int Hkv, int N,
                             int d, double scale, int causal, int window, const double *slopes,
                             const int64_t *keys, int nkeys, int nthreads)
{
    int r, G, bg;
    double *L, *D;
    if (check_dims(B, Hq, Hkv, N, N, d) || window < 0 || nkeys < 0) return -1;
    if (!q || !k || !v || !dout || !dk_rows || !dv_rows || (!keys && nkeys > 0)) return -1;
    for (r = 0; r < nkeys; ++r)
        if (keys[r] < 0 || keys[r] >= (int64_t)B * Hkv * N) return -1;
    G = Hq / Hkv;
    if (nthreads <= 0) nthreads = 1;
    L = (double *)malloc(sizeof(double) * ((size_t)G * N + 1));
    D = (double *)malloc(sizeof(double) * ((size_t)G * N + 1));
    if (!L || !D) { free(L); free(D); return -2; }
    for (bg = 0; bg < B * Hkv; ++bg) {
        int b = bg / Hkv, g = bg % Hkv, need = 0, bad = 0;
        long t;
        const float *kh = k + (size_t)bg * N * d, *vh = v + (size_t)bg * N * d;
        for (r = 0; r < nkeys; ++r) if (keys[r] / N == bg) need = 1;
        if (!need) continue;
        /* L_i and D_i of every row of the group's query heads. */
        #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 8) reduction(|:bad)
        for (t = 0; t < (long)G * N; ++t) {
            int hh = (int)(t / N), i = (int)(t % N), h = g * G + hh, j, c, lo, hi;
            const float *qi = q + (((size_t)b * Hq + h) * N + i) * d;
            const float *doi = dout + (((size_t)b * Hq + h) * N + i) * d;
            double *s = (double *)malloc(sizeof(double) * ((size_t)N + 1));
            double m = -INFINITY, l = 0.0, acc;
            if (!s) { bad = 1; continue; }
            visible_range(i, N, causal, window, &lo, &hi);
            for (j = lo; j < hi; ++j) {
                acc = 0.0;
                for (c = 0; c < d; ++c) acc += (double)qi[c] * (double)kh[(size_t)j * d + c];
                s[j - lo] = scale * acc + (slopes ? slopes[h] : 0.0) * (double)(j - i);
                if (s[j - lo] > m) m = s[j - lo];
            }
            for (j = lo; j < hi; ++j) l += exp(s[j - lo] - m);
            L[t] = (hi > lo) ? m + log(l) : -INFINITY;
            D[t] = 0.0;
            for (j = lo; j < hi; ++j) {
                acc = 0.0;
                for (c = 0; c < d; ++c) acc += (double)doi[c] * (double)vh[(size_t)j * d + c];
                D[t] += exp(s[j - lo] - L[t]) * acc;
            }
            free(s);
        }
        if (bad) { free(L); free(D); return -2; }
        #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
        for (r = 0; r < nkeys; ++r) {
            int j, hh, i, c;
            double kj[512], vj[512], ak[512], av[512];
            if (keys[r] / N != bg || d > 512) continue;
            j = (int)(keys[r] % N);
            for (c = 0; c < d; ++c) {
                kj[c] = (double)kh[(size_t)j * d + c];
                vj[c] = (double)vh[(size_t)j * d + c];
                ak[c] = 0.0; av[c] = 0.0;
            }
            for (hh = 0; hh < G; ++hh) {
                int h = g * G + hh;
                for (i = 0; i < N; ++i) {
                    int lo, hi;
                    const float *qi = q + (((size_t)b * Hq + h) * N + i) * d;
                    const float *doi = dout + (((size_t)b * Hq + h) * N + i) * d;
                    double sc = 0.0, dp = 0.0, p;
                    visible_range(i, N, causal, window, &lo, &hi);
                    if (j < lo || j >= hi) continue;
                    for (c = 0; c < d; ++c) {
                        sc += (double)qi[c] * kj[c];
                        dp += (double)doi[c] * vj[c];
                    }
                    p = exp(scale * sc + (slopes ? slopes[h] : 0.0) * (double)(j - i) - L[(size_t)hh * N + i]);
                    for (c = 0; c < d; ++c) {
                        ak[c] += p * (dp - D[(size_t)hh * N + i]) * (double)qi[c];
                        av[c] += p * (double)doi[c];
                    }
                }
            }
            for (c = 0; c < d; ++c) {
                dk_rows[(size_t)r * d + c] = scale * ak[c];
                dv_rows[(size_t)r * d + c] = av[c];
            }
        }
    }
    free(L); free(D);
    return 0;
}

/* One 8-bit cache element: fmt 0 = FP8 E4M3, fmt 1 = INT8 (two's complement). */
static double q8_to_double(uint8_t b, int fmt)
{
    return fmt == 0 ? e4m3_to_double(b) : (double)(int8_t)b;
}

/* Decode over an 8-bit paged KV cache: the KV-cache quantisation answer of the
 * screna.ai page (8-bit storage halves the cache against 16-bit; INT8 is the
 * safe default, NVIDIA's FP8 the hardware format; group-wise scales keep
 * accuracy).  Read plainly: each (page, kv head) slice of K and of V is one
 * group with one fp32 scale, k = k_scales[p*Hkv+g] * q8(byte), likewise v;
 * the bytes are E4M3 (fmt 0) or INT8 (fmt 1).  Everything else is exactly
 * oracle_decode_paged. */
int oracle_decode_paged_q8(const float *q, const uint8_t *k_pages, const uint8_t *v_pages,
                           const float *k_scales, const float *v_scales,
                           const int32_t *block_table, const int32_t *seq_lens,
                           double *o, double *lse,
                           int S, int Hq, int Hkv, int d, int page_size, int max_blocks,
                           int num_pages, double scale, int fmt,
                           const int32_t *seq_ids, int nseq, int nthreads)
{
    int G, r, bad = 0;
    if (S <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || page_size <= 0 || max_blocks <= 0 ||
        num_pages <= 0 || Hq % Hkv != 0 || nseq < 0 || (fmt != 0 && fmt != 1)) return -1;
    if (!q || !k_pages || !v_pages || !k_scales || !v_scales || !block_table || !seq_lens ||
        !o || !lse || (!seq_ids && nseq > 0)) return -1;
    G = Hq / Hkv;
    for (r = 0; r < nseq; ++r) {
        int s = seq_ids[r], t, len;
        if (s < 0 || s >= S) return -1;
        len = seq_lens[s];
        if (len < 0 || len > max_blocks * page_size) return -1;
        for (t = 0; t < len; t += page_size) {
            int32_t p = block_table[(size_t)s * max_blocks + t / page_size];
            if (p < 0 || p >= num_pages) return -1;
        }
    }
    if (nthreads <= 0) nthreads = 1;

    #pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1) reduction(|:bad)
    for (r = 0; r < nseq * Hkv; ++r) {
        int s = seq_ids[r / Hkv], g = r % Hkv;
        int len = seq_lens[s];
        int t, c, hh;
        double *kd = (double *)malloc(sizeof(double) * ((size_t)len * d + 1));
        double *vd = (double *)malloc(sizeof(double) * ((size_t)len * d + 1));
        double *sc = (double *)malloc(sizeof(double) * ((size_t)len + 1));
        if (!kd || !vd || !sc) { free(kd); free(vd); free(sc); bad = 1; continue; }
        for (t = 0; t < len; ++t) {
            int32_t p = block_table[(size_t)s * max_blocks + t / page_size];
            size_t base = (((size_t)p * Hkv + g) * page_size + (t % page_size)) * (size_t)d;
            double ks = (double)k_scales[(size_t)p * Hkv + g];
            double vs = (double)v_scales[(size_t)p * Hkv + g];
            for (c = 0; c < d; ++c) {
                kd[(size_t)t * d + c] = ks * q8_to_double(k_pages[base + c], fmt);
                vd[(size_t)t * d + c] = vs * q8_to_double(v_pages[base + c], fmt);
            }
        }
        for (hh = 0; hh < G; ++hh) {
            int h = g * G + hh;
            const float *qs = q + ((size_t)s * Hq + h) * (size_t)d;
            for (t = 0; t < len; ++t) {
                double acc = 0.0;
                for (c = 0; c < d; ++c) acc += (double)qs[c] * kd[(size_t)t * d + c];
                sc[t] = scale * acc;
            }
            softmax_row_times_v(sc, len, vd, d,
                                o + ((size_t)(r / Hkv) * Hq + h) * (size_t)d,
                                lse + (size_t)(r / Hkv) * Hq + h);
        }
        free(kd); free(vd); free(sc);
    }
    return bad ? -2 : 0;
}

/* Exposed for the pins: the e4m3 decode of one byte. */
double oracle_e4m3_to_double(int byte) { return e4m3_to_double((uint8_t)byte); }

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
