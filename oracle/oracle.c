/*
 * CPU oracle for exact scaled-dot-product attention.  TEST INFRASTRUCTURE ONLY:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * this code.  It shares nothing with the CUDA library.
 *
 * What it computes (plain definition, fp64 throughout):
 *
 *   O = softmax(scale * Q K^T [+ causal mask]) V,   lse = log(sum_j e^{s_j})
 *
 * following the standard three-step statement of attention (Gemini 3 Flash
 * kernel-fusion post, "traditional attention": S = QK^T, P = softmax(S),
 * O = PV; GPU-optimisation tag page, "algorithm principle": S = Q K^T / sqrt(d))
 * and the three-sweep softmax of the FlashAttention optimisation article
 * (section 2.2: one sweep for the row max, one for exp(x - max) and its sum,
 * one to normalise).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - causal masking is aligned bottom-right: key j is visible to query i iff
 *    j <= i + (Nkv - Nq); with Nq == Nkv that is the usual j <= i;
 *  - a row with no visible key returns O = 0 and lse = -inf;
 *  - lse is the natural log of the scaled scores' normaliser: m + ln(l);
 *  - query head hq reads KV head hq / (Hq / Hkv) (consecutive heads share one
 *    KV head, GPU-optimisation tag page, GQA section);
 *  - the paged cache is [num_pages_total, Hkv, page_size, d]; logical token t
 *    of sequence s lives at page block_table[s][t / page_size], row
 *    t % page_size (paged-gather article, section 2.1/2.3: a per-sequence list
 *    of physical blocks); table entries beyond the sequence are never read;
 *  - FP8 attention (the FP8 tensor-core variant named in the LLM-inference
 *    page's Flash Attention V3 section) takes E4M3 codes with one descale
 *    factor per tensor; its result here is the exact attention of the
 *    dequantised values.  Rounding P to FP8 for a tensor-core P.V product is
 *    part of a kernel's error, not of the definition.
 *
 * All bf16 inputs are passed as uint16 bit patterns and widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_TABLE 4
#define ORACLE_ERR_NOMEM 6

static double bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * One query row against n keys/values (rows of length d, row stride d).
 * s is scratch of length n.  Writes o[0..d) and *lse.
 * visible = number of leading keys the query may see (keys >= visible are
 * masked to -inf explicitly before the softmax).
 */
static void attend_row(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       int n, int d, double scale, int visible,
                       double *s, double *o, double *lse)
{
    /* scores, with the mask written out explicitly */
    for (int j = 0; j < n; ++j) {
        if (j >= visible) {
            s[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        const uint16_t *kj = k + (size_t)j * d;
        for (int t = 0; t < d; ++t)
            acc += bf16_to_f64(q[t]) * bf16_to_f64(kj[t]);
        s[j] = scale * acc;
    }
    /* sweep 1: row maximum */
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > m)
            m = s[j];
    for (int t = 0; t < d; ++t)
        o[t] = 0.0;
    if (m == -INFINITY) {       /* no visible key */
        *lse = -INFINITY;
        return;
    }
    /* sweep 2: normaliser */
    double l = 0.0;
    for (int j = 0; j < n; ++j)
        if (s[j] != -INFINITY)
            l += exp(s[j] - m);
    /* sweep 3: normalised weights times V */
    for (int j = 0; j < n; ++j) {
        if (s[j] == -INFINITY)
            continue;
        double p = exp(s[j] - m) / l;
        const uint16_t *vj = v + (size_t)j * d;
        for (int t = 0; t < d; ++t)
            o[t] += p * bf16_to_f64(vj[t]);
    }
    *lse = m + log(l);
}

static int visible_keys(int i, int Nq, int Nkv, int causal)
{
    if (!causal)
        return Nkv;
    long lim = (long)i + (long)(Nkv - Nq) + 1;
    if (lim < 0)
        lim = 0;
    if (lim > Nkv)
        lim = Nkv;
    return (int)lim;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Contiguous attention.  q [B,Hq,Nq,d], k/v [B,Hkv,Nkv,d] (bf16 bits).
 * rows: optional list of flat row ids r = (b*Hq + hq)*Nq + i to evaluate;
 * if rows == NULL every row is evaluated in order.  o is [nrows, d] fp64,
 * lse is [nrows] fp64 (may be NULL).
 */
int oracle_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                double scale, int causal, const int64_t *rows, int64_t nrows,
                double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nkv < 0 || d <= 0 || Hq % Hkv)
        return ORACLE_ERR_ARG;
    const int64_t total = (int64_t)B * Hq * Nq;
    if (!rows)
        nrows = total;
    const int G = Hq / Hkv;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Nkv > 0 ? Nkv : 1));
        if (!s) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!s)
                continue;
            int64_t id = rows ? rows[r] : r;
            if (id < 0 || id >= total) {
#pragma omp atomic write
                err = ORACLE_ERR_ARG;
                continue;
            }
            int i = (int)(id % Nq);
            int64_t bh = id / Nq;
            int hq = (int)(bh % Hq);
            int b = (int)(bh / Hq);
            int hkv = hq / G;
            const uint16_t *qi = q + (size_t)id * d;
            const uint16_t *kb = k + ((size_t)b * Hkv + hkv) * (size_t)Nkv * d;
            const uint16_t *vb = v + ((size_t)b * Hkv + hkv) * (size_t)Nkv * d;
            double l;
            attend_row(qi, kb, vb, Nkv, d, scale, visible_keys(i, Nq, Nkv, causal),
                       s, o + (size_t)r * d, &l);
            if (lse)
                lse[r] = l;
        }
        free(s);
    }
    return err;
}

/*
 * FP8 inputs.  A code is an OCP 8-bit float in the E4M3 form ("e4m3fn"):
 * sign bit, 4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0
 * holds the subnormals m/8 * 2^-6; there is no infinity, and S.1111.111 is NaN,
 * so the largest finite magnitude is 1.75 * 2^8 = 448.
 */
static double e4m3_to_f64(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);          /* (m / 8) * 2^(1 - 7) */
    else
        v = ldexp(8.0 + m, e - 10);        /* (1 + m / 8) * 2^(e - 7) */
    return (b & 0x80) ? -v : v;
}

void oracle_e4m3_decode(const uint8_t *codes, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = e4m3_to_f64(codes[i]);
}

/*
 * One query row of FP8 attention: the same three sweeps as attend_row, on the
 * dequantised values dq * e4m3(q), dk * e4m3(k), dv * e4m3(v).
 */
static void attend_row_fp8(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                           double dq, double dk, double dv, int n, int d, double scale,
                           int visible, double *s, double *o, double *lse)
{
    for (int j = 0; j < n; ++j) {
        if (j >= visible) {
            s[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        const uint8_t *kj = k + (size_t)j * d;
        for (int t = 0; t < d; ++t)
            acc += (dq * e4m3_to_f64(q[t])) * (dk * e4m3_to_f64(kj[t]));
        s[j] = scale * acc;
    }
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > m)
            m = s[j];
    for (int t = 0; t < d; ++t)
        o[t] = 0.0;
    if (m == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j)
        if (s[j] != -INFINITY)
            l += exp(s[j] - m);
    for (int j = 0; j < n; ++j) {
        if (s[j] == -INFINITY)
            continue;
        double p = exp(s[j] - m) / l;
        const uint8_t *vj = v + (size_t)j * d;
        for (int t = 0; t < d; ++t)
            o[t] += p * (dv * e4m3_to_f64(vj[t]));
    }
    *lse = m + log(l);
}

/*
 * Contiguous FP8 attention: q [B,Hq,Nq,d], k/v [B,Hkv,Nkv,d] as E4M3 codes,
 * one descale factor per tensor (the real inputs are q_descale * e4m3(q) and
 * so on).  The exact attention of the dequantised inputs; rows, masking, head
 * mapping and outputs as oracle_attn.
 */
int oracle_attn_fp8(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                    double q_descale, double k_descale, double v_descale,
                    int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                    double scale, int causal, const int64_t *rows, int64_t nrows,
                    double *o, double *lse)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nkv < 0 || d <= 0 || Hq % Hkv)
        return ORACLE_ERR_ARG;
    const int64_t total = (int64_t)B * Hq * Nq;
    if (!rows)
        nrows = total;
    const int G = Hq / Hkv;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Nkv > 0 ? Nkv : 1));
        if (!s) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!s)
                continue;
            int64_t id = rows ? rows[r] : r;
            if (id < 0 || id >= total) {
#pragma omp atomic write
                err = ORACLE_ERR_ARG;
                continue;
            }
            int i = (int)(id % Nq);
            int64_t bh = id / Nq;
            int hq = (int)(bh % Hq);
            int b = (int)(bh / Hq);
            int hkv = hq / G;
            const uint8_t *qi = q + (size_t)id * d;
            const uint8_t *kb = k + ((size_t)b * Hkv + hkv) * (size_t)Nkv * d;
            const uint8_t *vb = v + ((size_t)b * Hkv + hkv) * (size_t)Nkv * d;
            double l;
            attend_row_fp8(qi, kb, vb, q_descale, k_descale, v_descale, Nkv, d, scale,
                           visible_keys(i, Nq, Nkv, causal), s, o + (size_t)r * d, &l);
            if (lse)
                lse[r] = l;
        }
        free(s);
    }
    return err;
}

/*
 * Explicit gather of one sequence's logical K and V rows for KV head hkv:
 * k_out/v_out [seq_len, d] (bf16 bits) = cache[block_table[seq][t/ps], hkv, t%ps, :].
 * Returns ORACLE_ERR_TABLE if a needed table entry is outside [0, num_pages_total)
 * or the length does not fit in max_pages pages.
 */
int oracle_paged_gather(const uint16_t *k_cache, const uint16_t *v_cache,
                        const int32_t *block_table, const int32_t *seq_lens,
                        int seq, int hkv, int page_size, int Hkv, int d,
                        int max_pages, int64_t num_pages_total,
                        uint16_t *k_out, uint16_t *v_out)
{
    if (page_size <= 0 || Hkv <= 0 || d <= 0 || hkv < 0 || hkv >= Hkv || seq < 0)
        return ORACLE_ERR_ARG;
    int len = seq_lens[seq];
    if (len < 0 || (int64_t)len > (int64_t)max_pages * page_size)
        return ORACLE_ERR_TABLE;
    for (int t = 0; t < len; ++t) {
        int32_t page = block_table[(size_t)seq * max_pages + t / page_size];
        if (page < 0 || page >= num_pages_total)
            return ORACLE_ERR_TABLE;
        size_t src = (((size_t)page * Hkv + hkv) * page_size + (size_t)(t % page_size)) * d;
        memcpy(k_out + (size_t)t * d, k_cache + src, sizeof(uint16_t) * (size_t)d);
        memcpy(v_out + (size_t)t * d, v_cache + src, sizeof(uint16_t) * (size_t)d);
    }
    return ORACLE_OK;
}

/*
 * Paged decode: one query token per sequence attends all seq_lens[s] keys of
 * its sequence (no mask).  q/o [num_seqs, Hq, d], lse [num_seqs, Hq].
 * seqs: optional list of sequences to evaluate (o/lse rows follow that list).
 */
int oracle_paged_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                        const int32_t *block_table, const int32_t *seq_lens,
                        int page_size, int num_seqs, int Hq, int Hkv, int d,
                        int max_pages, int64_t num_pages_total, double scale,
                        const int32_t *seqs, int nseqs, double *o, double *lse)
{
    if (num_seqs < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv || page_size <= 0)
        return ORACLE_ERR_ARG;
    if (!seqs)
        nseqs = num_seqs;
    const int G = Hq / Hkv;
    int err = ORACLE_OK;
    const int64_t items = (int64_t)nseqs * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t it = 0; it < items; ++it) {
        int si = (int)(it / Hkv), hkv = (int)(it % Hkv);
        int s = seqs ? seqs[si] : si;
        if (s < 0 || s >= num_seqs) {
#pragma omp atomic write
            err = ORACLE_ERR_ARG;
            continue;
        }
        int len = seq_lens[s];
        if (len < 0)
            len = 0;
        size_t n = (size_t)(len > 0 ? len : 1);
        uint16_t *kg = (uint16_t *)malloc(sizeof(uint16_t) * n * d);
        uint16_t *vg = (uint16_t *)malloc(sizeof(uint16_t) * n * d);
        double *sc = (double *)malloc(sizeof(double) * n);
        if (!kg || !vg || !sc) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
            int e = oracle_paged_gather(k_cache, v_cache, block_table, seq_lens, s, hkv,
                                        page_size, Hkv, d, max_pages, num_pages_total, kg, vg);
            if (e) {
#pragma omp atomic write
                err = e;
            } else {
                for (int g = 0; g < G; ++g) {
                    int hq = hkv * G + g;
                    size_t row = (size_t)si * Hq + hq;
                    double l;
                    attend_row(q + ((size_t)s * Hq + hq) * d, kg, vg, len, d, scale, len,
                               sc, o + row * d, &l);
                    if (lse)
                        lse[row] = l;
                }
            }
        }
        free(kg);
        free(vg);
        free(sc);
    }
    return err;
}

/*
 * Varlen (chunked) prefill against the paged cache: several sequences' new
 * query rows, packed, each attending over its sequence's keys in the pool
 * (the new tokens' K/V already appended).  The page structure is the paged
 * decode's (paged-gather article, sections 2.1-2.4; GPU-optimisation tag
 * page, PagedAttention); chunked prefill joins it to the prefill
 * (LLM-inference article, section 3.2).
 *
 * Sequence s owns query rows [cu_seqlens[s], cu_seqlens[s+1]) of q
 * [total_q, Hq, d] and seq_lens[s] keys.  Its logical K/V rows are gathered
 * explicitly (oracle_paged_gather), then every query row follows the
 * definition of oracle_attn with Nq = q_len and Nkv = seq_len: under the
 * bottom-right causal alignment query i sits at position seq_len - q_len + i.
 * seqs: optional subset of sequences (NULL = all).  o [total_q, Hq, d] and
 * lse [total_q, Hq] (fp64) are written for the listed sequences' rows only.
 */
int oracle_paged_prefill(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                         const int32_t *block_table, const int32_t *cu_seqlens, const int32_t *seq_lens,
                         int page_size, int num_seqs, int64_t total_q, int Hq, int Hkv, int d,
                         int max_pages, int64_t num_pages_total, double scale, int causal,
                         const int32_t *seqs, int nseqs, double *o, double *lse)
{
    if (num_seqs < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv || page_size <= 0 || total_q < 0)
        return ORACLE_ERR_ARG;
    if (!seqs)
        nseqs = num_seqs;
    const int G = Hq / Hkv;
    int err = ORACLE_OK;
    const int64_t items = (int64_t)nseqs * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t it = 0; it < items; ++it) {
        int si = (int)(it / Hkv), hkv = (int)(it % Hkv);
        int s = seqs ? seqs[si] : si;
        if (s < 0 || s >= num_seqs || cu_seqlens[s] < 0 || cu_seqlens[s + 1] < cu_seqlens[s] ||
            cu_seqlens[s + 1] > total_q) {
#pragma omp atomic write
            err = ORACLE_ERR_ARG;
            continue;
        }
        int q0 = cu_seqlens[s], q_len = cu_seqlens[s + 1] - cu_seqlens[s];
        int len = seq_lens[s] > 0 ? seq_lens[s] : 0;
        size_t n = (size_t)(len > 0 ? len : 1);
        uint16_t *kg = (uint16_t *)malloc(sizeof(uint16_t) * n * d);
        uint16_t *vg = (uint16_t *)malloc(sizeof(uint16_t) * n * d);
        double *sc = (double *)malloc(sizeof(double) * n);
        if (!kg || !vg || !sc) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
            int e = oracle_paged_gather(k_cache, v_cache, block_table, seq_lens, s, hkv,
                                        page_size, Hkv, d, max_pages, num_pages_total, kg, vg);
            if (e) {
#pragma omp atomic write
                err = e;
            } else {
                for (int g = 0; g < G; ++g) {
                    int hq = hkv * G + g;
                    for (int i = 0; i < q_len; ++i) {
                        size_t row = (size_t)(q0 + i) * Hq + hq;
                        double l;
                        attend_row(q + row * d, kg, vg, len, d, scale, visible_keys(i, q_len, len, causal),
                                   sc, o + row * d, &l);
                        if (lse)
                            lse[row] = l;
                    }
                }
            }
        }
        free(kg);
        free(vg);
        free(sc);
    }
    return err;
}

/*
 * Gradients of attention (the backward pass), plain chain rule in fp64.
 *
 * The kernel-fusion post (section 4, recomputation) fixes the strategy of the
 * backward pass -- keep only each row's max and normaliser, recompute the
 * Q K^T blocks, stream the gradients -- but prints no formulas, so this is
 * the derivative of the definition above, written out:
 *
 *   S = scale Q K^T (+ mask),  P = softmax_rows(S),  O = P V,  loss gradient dO
 *   dV = P^T dO
 *   dP = dO V^T
 *   dS_ij = P_ij (dP_ij - sum_t P_it dP_it)          (softmax Jacobian)
 *   dQ = scale dS K,   dK = scale dS^T Q
 *
 * With grouped heads a KV head's dK and dV sum the contributions of every
 * query head that reads it.  Masked entries have P = 0 and contribute
 * nothing; a row with no visible key contributes nothing.
 *
 * Evaluation order (plain loops, parallel over independent outputs):
 *   sweep 1, per query row i: scores, the three-sweep softmax, dP_i., the
 *            Jacobian row term r_i = sum_t P_it dP_it, and dQ_i; keeps the
 *            row's max m_i and normaliser l_i;
 *   sweep 2, per key j: P_ij = exp(s_ij - m_i) / l_i and dP_ij recomputed for
 *            every row i that sees j, then dV_j and dK_j.
 *
 * groups: optional list of flat KV-head ids g = b*Hkv + hkv to evaluate (each
 * with all rows of its query heads); NULL = all.  dq [B,Hq,Nq,d] and
 * dk/dv [B,Hkv,Nkv,d] (fp64) are written for the listed groups only and must
 * be zero-initialised by the caller.
 */
static double dot_bf16(const uint16_t *a, const uint16_t *b, int d)
{
    double acc = 0.0;
    for (int t = 0; t < d; ++t)
        acc += bf16_to_f64(a[t]) * bf16_to_f64(b[t]);
    return acc;
}

int oracle_attn_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                    int B, int Hq, int Hkv, int Nq, int Nkv, int d, double scale, int causal,
                    const int64_t *groups, int64_t ngroups, double *dq, double *dk, double *dv)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nkv < 0 || d <= 0 || Hq % Hkv)
        return ORACLE_ERR_ARG;
    const int64_t total = (int64_t)B * Hkv;
    if (!groups)
        ngroups = total;
    for (int64_t gi = 0; gi < ngroups; ++gi)
        if (groups && (groups[gi] < 0 || groups[gi] >= total))
            return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const int64_t rows_per_group = (int64_t)G * Nq;
    /* per row of the listed groups: softmax max, normaliser, Jacobian row term */
    double *rm = (double *)malloc(sizeof(double) * (size_t)(ngroups * rows_per_group + 1));
    double *rl = (double *)malloc(sizeof(double) * (size_t)(ngroups * rows_per_group + 1));
    double *rr = (double *)malloc(sizeof(double) * (size_t)(ngroups * rows_per_group + 1));
    if (!rm || !rl || !rr) {
        free(rm);
        free(rl);
        free(rr);
        return ORACLE_ERR_NOMEM;
    }
    int err = ORACLE_OK;

    /* sweep 1: one query row at a time */
#pragma omp parallel
    {
        size_t n = (size_t)(Nkv > 0 ? Nkv : 1);
        double *s = (double *)malloc(sizeof(double) * n);
        double *p = (double *)malloc(sizeof(double) * n);
        double *dp = (double *)malloc(sizeof(double) * n);
        if (!s || !p || !dp) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t x = 0; x < ngroups * rows_per_group; ++x) {
            if (!s || !p || !dp)
                continue;
            int64_t gid = groups ? groups[x / rows_per_group] : x / rows_per_group;
            int b = (int)(gid / Hkv), hkv = (int)(gid % Hkv);
            int hq = hkv * G + (int)((x % rows_per_group) / Nq);
            int i = (int)(x % Nq);
            size_t row = ((size_t)b * Hq + hq) * (size_t)Nq + i;
            const uint16_t *qi = q + row * d, *doi = dout + row * d;
            const uint16_t *kb = k + ((size_t)b * Hkv + hkv) * (size_t)Nkv * d;
            const uint16_t *vb = v + ((size_t)b * Hkv + hkv) * (size_t)Nkv * d;
            int visible = visible_keys(i, Nq, Nkv, causal);
            rm[x] = -INFINITY;
            rl[x] = 0.0;
            rr[x] = 0.0;
            if (visible == 0)
                continue;
            double m = -INFINITY;
            for (int j = 0; j < visible; ++j) {
                s[j] = scale * dot_bf16(qi, kb + (size_t)j * d, d);
                if (s[j] > m)
                    m = s[j];
            }
            double l = 0.0;
            for (int j = 0; j < visible; ++j)
                l += exp(s[j] - m);
            double rowterm = 0.0;
            for (int j = 0; j < visible; ++j) {
                p[j] = exp(s[j] - m) / l;
                dp[j] = dot_bf16(doi, vb + (size_t)j * d, d);
                rowterm += p[j] * dp[j];
            }
            double *dqi = dq + row * d;
            for (int j = 0; j < visible; ++j) {
                double ds = p[j] * (dp[j] - rowterm);
                for (int t = 0; t < d; ++t)
                    dqi[t] += scale * ds * bf16_to_f64(kb[(size_t)j * d + t]);
            }
            rm[x] = m;
            rl[x] = l;
            rr[x] = rowterm;
        }
        free(s);
        free(p);
        free(dp);
    }

    /* sweep 2: one key at a time, over every row of the group that sees it */
#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t y = 0; y < ngroups * (int64_t)Nkv; ++y) {
        int64_t gi = y / Nkv;
        int64_t gid = groups ? groups[gi] : gi;
        int b = (int)(gid / Hkv), hkv = (int)(gid % Hkv);
        int j = (int)(y % Nkv);
        const uint16_t *kj = k + (((size_t)b * Hkv + hkv) * (size_t)Nkv + j) * d;
        const uint16_t *vj = v + (((size_t)b * Hkv + hkv) * (size_t)Nkv + j) * d;
        double *dkj = dk + (((size_t)b * Hkv + hkv) * (size_t)Nkv + j) * d;
        double *dvj = dv + (((size_t)b * Hkv + hkv) * (size_t)Nkv + j) * d;
        for (int hq = hkv * G; hq < (hkv + 1) * G; ++hq) {
            for (int i = 0; i < Nq; ++i) {
                if (j >= visible_keys(i, Nq, Nkv, causal))
                    continue;
                int64_t x = gi * rows_per_group + (int64_t)(hq - hkv * G) * Nq + i;
                size_t row = ((size_t)b * Hq + hq) * (size_t)Nq + i;
                const uint16_t *qi = q + row * d, *doi = dout + row * d;
                double p = exp(scale * dot_bf16(qi, kj, d) - rm[x]) / rl[x];
                double ds = p * (dot_bf16(doi, vj, d) - rr[x]);
                for (int t = 0; t < d; ++t) {
                    dkj[t] += scale * ds * bf16_to_f64(qi[t]);
                    dvj[t] += p * bf16_to_f64(doi[t]);
                }
            }
        }
    }
    free(rm);
    free(rl);
    free(rr);
    return err;
}
