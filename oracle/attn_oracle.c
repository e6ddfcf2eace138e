/*
 * attn_oracle.c -- the CPU oracle for fused attention.  TEST INFRASTRUCTURE
 * ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg are the
 * only callers.  It shares no code, header, table or helper with the CUDA
 * library, and the library never calls it.
 *
 * What it computes is the plain definition that FlashAttention-style tiling
 * reaches up to rounding order:
 *   - "Real-time inference optimisation: making large models respond fast"
 *     (llmapi-app.pages.dev), section "Flash Attention optimisation": scores
 *     q.k^T times a scale, a softmax over the keys (kept there as a running
 *     max / running sum, which is algebraically the same softmax), then the
 *     probability-weighted sum of the values, divided by the softmax sum.
 *   - "FlashRT-HF-kernels" (zingnex.cn), section "Attention optimisation":
 *     causal masking for autoregressive generation and MQA/GQA head sharing;
 *     section "Attention operators": paged KV cache.
 *   - same page 5, method `paged_attention`: pages of 16 tokens.  That sketch
 *     adds per-page normalised outputs, which is not softmax attention; the
 *     oracle instead gathers the pages and applies the one definition, and the
 *     partial-result merge is the log-sum-exp weighting that the online
 *     softmax update of the same page implies.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   scale is passed in (the sketch's 1/sqrt of an ambiguous "K" read as
 *   1/sqrt(D)); natural exp and natural-log LSE, scale included; causal mask is
 *   bottom-right aligned: key j is visible to query i iff j <= i + (Skv - Sq);
 *   query head h reads KV head h / (Hq/Hkv); the paged cache is
 *   [num_pages][Hkv][page_size][D] with token t of sequence b in physical page
 *   block_table[b][t / page_size], slot t % page_size; a row with no visible
 *   key has o = 0 and lse = -inf.
 *
 * Arithmetic is fp64 throughout.  Inputs are bf16 bit patterns (uint16), which
 * widen exactly to fp64.  Each (batch, head) materialises its full score
 * matrix (rows i0..i1 of it when sampling) and applies an explicit softmax.
 * OpenMP only spreads independent (batch, head) or row work over threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_MEM 2

static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Attention for query rows i0..i1-1 of one (query head, batch):
 *   qh : [Sq][D]  this head's queries      kh, vh : [Skv][D]  its KV head
 *   oh : [i1-i0][D]  output rows (fp64)    lseh   : [i1-i0]   log-sum-exp
 * The (i1-i0) x Skv score matrix is materialised in `s` (caller-provided).
 */
static void attend_rows(const uint16_t *qh, const uint16_t *kh, const uint16_t *vh,
                        double *oh, double *lseh, int Sq, int Skv, int D,
                        int causal, double scale, int i0, int i1, double *s)
{
    const long long offset = (long long)Skv - (long long)Sq;   /* bottom-right alignment */

    /* 1. scores s_ij = scale * sum_d q_id k_jd, masked ones set to -inf */
    for (int i = i0; i < i1; ++i) {
        double *srow = s + (size_t)(i - i0) * Skv;
        for (int j = 0; j < Skv; ++j) {
            int visible = !causal || ((long long)j <= (long long)i + offset);
            if (!visible) {
                srow[j] = -INFINITY;
                continue;
            }
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += widen_bf16(qh[(size_t)i * D + d]) * widen_bf16(kh[(size_t)j * D + d]);
            srow[j] = scale * dot;
        }
    }

    /* 2. explicit softmax per row, 3. probability-weighted sum of values */
    for (int i = i0; i < i1; ++i) {
        double *srow = s + (size_t)(i - i0) * Skv;
        double *orow = oh + (size_t)(i - i0) * D;
        double m = -INFINITY;
        for (int j = 0; j < Skv; ++j)
            if (srow[j] > m) m = srow[j];
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        if (m == -INFINITY) {           /* no visible key */
            lseh[i - i0] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int j = 0; j < Skv; ++j) {
            double p = (srow[j] == -INFINITY) ? 0.0 : exp(srow[j] - m);
            srow[j] = p;
            l += p;
        }
        for (int j = 0; j < Skv; ++j) {
            double w = srow[j] / l;
            if (w == 0.0) continue;     /* masked key: contributes exactly nothing */
            for (int d = 0; d < D; ++d)
                orow[d] += w * widen_bf16(vh[(size_t)j * D + d]);
        }
        lseh[i - i0] = m + log(l);
    }
}

static int check_shape(int B, int Hq, int Hkv, int Sq, int Skv, int D, double scale)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Sq < 0 || Skv < 0 || D <= 0) return ORACLE_ERR_ARG;
    if (Hq % Hkv != 0) return ORACLE_ERR_ARG;
    if (!(scale > 0.0) || !isfinite(scale)) return ORACLE_ERR_ARG;
    return ORACLE_OK;
}

/*
 * Full attention.  q [B][Hq][Sq][D], k and v [B][Hkv][Skv][D] (bf16 bits,
 * contiguous); o [B][Hq][Sq][D] and lse [B][Hq][Sq] in fp64.
 */
int oracle_attn_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    double *o, double *lse, int B, int Hq, int Hkv, int Sq, int Skv,
                    int D, int causal, double scale)
{
    int rc = check_shape(B, Hq, Hkv, Sq, Skv, D, scale);
    if (rc) return rc;
    const int g = Hq / Hkv;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (long long bh = 0; bh < (long long)B * Hq; ++bh) {
        const int b = (int)(bh / Hq), h = (int)(bh % Hq), kvh = h / g;
        double *s = (double *)malloc(sizeof(double) * ((size_t)Sq * Skv + 1));
        if (!s) { failed |= 1; continue; }
        attend_rows(q + ((size_t)b * Hq + h) * Sq * D,
                    k + ((size_t)b * Hkv + kvh) * Skv * D,
                    v + ((size_t)b * Hkv + kvh) * Skv * D,
                    o + ((size_t)b * Hq + h) * Sq * D,
                    lse + ((size_t)b * Hq + h) * Sq,
                    Sq, Skv, D, causal, scale, 0, Sq, s);
        free(s);
    }
    return failed ? ORACLE_ERR_MEM : ORACLE_OK;
}

/*
 * Sampled attention: the same definition for n_rows chosen rows.  rows[r] is
 * the flat index (b*Hq + h)*Sq + i of row r; o_rows [n_rows][D], lse_rows
 * [n_rows].  Used where the full problem is too large for the oracle.
 */
int oracle_attn_fwd_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         int B, int Hq, int Hkv, int Sq, int Skv, int D, int causal,
                         double scale, int n_rows, const int64_t *rows,
                         double *o_rows, double *lse_rows)
{
    int rc = check_shape(B, Hq, Hkv, Sq, Skv, D, scale);
    if (rc) return rc;
    const int g = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * Sq;
    for (int r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return ORACLE_ERR_ARG;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int r = 0; r < n_rows; ++r) {
        const int64_t flat = rows[r];
        const int i = (int)(flat % Sq);
        const int h = (int)((flat / Sq) % Hq);
        const int b = (int)(flat / ((int64_t)Sq * Hq));
        const int kvh = h / g;
        double *s = (double *)malloc(sizeof(double) * ((size_t)Skv + 1));
        if (!s) { failed |= 1; continue; }
        attend_rows(q + ((size_t)b * Hq + h) * Sq * D,
                    k + ((size_t)b * Hkv + kvh) * Skv * D,
                    v + ((size_t)b * Hkv + kvh) * Skv * D,
                    o_rows + (size_t)r * D, lse_rows + r, Sq, Skv, D, causal, scale,
                    i, i + 1, s);
        free(s);
    }
    return failed ? ORACLE_ERR_MEM : ORACLE_OK;
}

/*
 * Decode (one query token per sequence) over a paged KV cache.
 *   q           [B][Hq][D]                         bf16 bits
 *   k_pages     [num_pages][Hkv][page_size][D]     bf16 bits (v_pages likewise)
 *   block_table [B][max_pages]                     physical page of each logical page
 *   seq_lens    [B]                                tokens in each sequence
 *   o [B][Hq][D], lse [B][Hq]                      fp64
 * Each sequence's cache is first gathered into contiguous [Hkv][len][D] arrays
 * through the block table with plain integer indexing; the same definition as
 * oracle_attn_fwd then applies with Sq = 1, Skv = len, no mask.
 * heads_mask, if not NULL, is [B*Hq]: rows with 0 are skipped (left as is).
 */
int oracle_attn_decode_paged(const uint16_t *q, const uint16_t *k_pages,
                             const uint16_t *v_pages, const int32_t *block_table,
                             int max_pages, const int32_t *seq_lens, int page_size,
                             int num_pages, double *o, double *lse, int B, int Hq,
                             int Hkv, int D, double scale, const uint8_t *heads_mask)
{
    int rc = check_shape(B, Hq, Hkv, 1, 0, D, scale);
    if (rc) return rc;
    if (page_size <= 0 || num_pages < 0 || max_pages < 0) return ORACLE_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        long long len = seq_lens[b];
        if (len < 0 || (len + page_size - 1) / page_size > max_pages) return ORACLE_ERR_ARG;
        for (long long p = 0; p < (len + page_size - 1) / page_size; ++p) {
            int32_t phys = block_table[(size_t)b * max_pages + p];
            if (phys < 0 || phys >= num_pages) return ORACLE_ERR_ARG;
        }
    }
    const int g = Hq / Hkv;
    for (int b = 0; b < B; ++b) {
        const int len = seq_lens[b];
        const size_t per_head = (size_t)len * D;
        uint16_t *kc = (uint16_t *)malloc(sizeof(uint16_t) * (per_head * Hkv + 1));
        uint16_t *vc = (uint16_t *)malloc(sizeof(uint16_t) * (per_head * Hkv + 1));
        if (!kc || !vc) { free(kc); free(vc); return ORACLE_ERR_MEM; }
        /* gather: token t -> page block_table[b][t / page_size], slot t % page_size */
        for (int kvh = 0; kvh < Hkv; ++kvh)
            for (int t = 0; t < len; ++t) {
                const int32_t phys = block_table[(size_t)b * max_pages + t / page_size];
                const int slot = t % page_size;
                const size_t src = (((size_t)phys * Hkv + kvh) * page_size + slot) * D;
                const size_t dst = (size_t)kvh * per_head + (size_t)t * D;
                memcpy(kc + dst, k_pages + src, sizeof(uint16_t) * D);
                memcpy(vc + dst, v_pages + src, sizeof(uint16_t) * D);
            }
        int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
        for (int h = 0; h < Hq; ++h) {
            if (heads_mask && !heads_mask[(size_t)b * Hq + h]) continue;
            const int kvh = h / g;
            double *s = (double *)malloc(sizeof(double) * ((size_t)len + 1));
            if (!s) { failed |= 1; continue; }
            attend_rows(q + ((size_t)b * Hq + h) * D, kc + (size_t)kvh * per_head,
                        vc + (size_t)kvh * per_head, o + ((size_t)b * Hq + h) * D,
                        lse + (size_t)b * Hq + h, 1, len, D, 0, scale, 0, 1, s);
            free(s);
        }
        free(kc);
        free(vc);
        if (failed) return ORACLE_ERR_MEM;
    }
    return ORACLE_OK;
}

/*
 * Chunked prefill over a paged KV cache: sequence b holds seq_lens[b] cached
 * tokens (the new chunk included) in the paged layout of
 * oracle_attn_decode_paged, and its last q_lens[b] tokens are the queries.
 *   q [B][Hq][max_q][D] bf16 bits (rows i >= q_lens[b] are padding)
 *   o [B][Hq][max_q][D], lse [B][Hq][max_q] fp64; padding rows get o = 0,
 *   lse = -inf.
 * The cache is gathered through the block table exactly as for decode, then
 * the definition applies with Sq = q_lens[b], Skv = seq_lens[b] and the
 * bottom-right causal mask (query i sees keys j <= i + Skv - Sq) when causal.
 */
int oracle_attn_prefill_paged(const uint16_t *q, const uint16_t *k_pages,
                              const uint16_t *v_pages, const int32_t *block_table,
                              int max_pages, const int32_t *seq_lens, const int32_t *q_lens,
                              int page_size, int num_pages, double *o, double *lse, int B,
                              int Hq, int Hkv, int max_q, int D, int causal, double scale)
{
    int rc = check_shape(B, Hq, Hkv, max_q, 0, D, scale);
    if (rc) return rc;
    if (page_size <= 0 || num_pages < 0 || max_pages < 0) return ORACLE_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        long long len = seq_lens[b];
        if (len < 0 || (len + page_size - 1) / page_size > max_pages) return ORACLE_ERR_ARG;
        if (q_lens[b] < 0 || q_lens[b] > max_q) return ORACLE_ERR_ARG;
        for (long long p = 0; p < (len + page_size - 1) / page_size; ++p) {
            int32_t phys = block_table[(size_t)b * max_pages + p];
            if (phys < 0 || phys >= num_pages) return ORACLE_ERR_ARG;
        }
    }
    const int g = Hq / Hkv;
    for (size_t i = 0; i < (size_t)B * Hq * max_q * D; ++i) o[i] = 0.0;
    for (size_t i = 0; i < (size_t)B * Hq * max_q; ++i) lse[i] = -INFINITY;
    for (int b = 0; b < B; ++b) {
        const int len = seq_lens[b], ql = q_lens[b];
        const size_t per_head = (size_t)len * D;
        uint16_t *kc = (uint16_t *)malloc(sizeof(uint16_t) * (per_head * Hkv + 1));
        uint16_t *vc = (uint16_t *)malloc(sizeof(uint16_t) * (per_head * Hkv + 1));
        if (!kc || !vc) { free(kc); free(vc); return ORACLE_ERR_MEM; }
        for (int kvh = 0; kvh < Hkv; ++kvh)
            for (int t = 0; t < len; ++t) {
                const int32_t phys = block_table[(size_t)b * max_pages + t / page_size];
                const size_t src = (((size_t)phys * Hkv + kvh) * page_size + t % page_size) * D;
                const size_t dst = (size_t)kvh * per_head + (size_t)t * D;
                memcpy(kc + dst, k_pages + src, sizeof(uint16_t) * D);
                memcpy(vc + dst, v_pages + src, sizeof(uint16_t) * D);
            }
        int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
        for (int h = 0; h < Hq; ++h) {
            const int kvh = h / g;
            double *s = (double *)malloc(sizeof(double) * ((size_t)ql * len + 1));
            if (!s) { failed |= 1; continue; }
            attend_rows(q + ((size_t)b * Hq + h) * max_q * D, kc + (size_t)kvh * per_head,
                        vc + (size_t)kvh * per_head, o + ((size_t)b * Hq + h) * max_q * D,
                        lse + ((size_t)b * Hq + h) * max_q, ql, len, D, causal, scale, 0, ql, s);
            free(s);
        }
        free(kc);
        free(vc);
        if (failed) return ORACLE_ERR_MEM;
    }
    return ORACLE_OK;
}

/*
 * FP8 e4m3 (the "fn" variant: no infinities) to fp64, from its bit fields:
 * sign s (bit 7), exponent e (bits 6-3, bias 7), mantissa m (bits 2-0).
 *   e = 0           : (-1)^s * m/8 * 2^(1-7)       (subnormal, zero)
 *   e = 15, m = 7   : NaN
 *   otherwise       : (-1)^s * (1 + m/8) * 2^(e-7)
 * Exported so that the tests can compare it code by code with torch's
 * float8_e4m3fn.
 */
double oracle_e4m3_to_f64(uint8_t code)
{
    const int sgn = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m / 8.0, 1 - 7) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return sgn ? -mag : mag;
}

/* One decode row over fp64 keys and values: scores scale * q.k_j, explicit
 * softmax, probability-weighted sum of the values (the definition). */
static void attend_decode_row(const uint16_t *qh, const double *kh, const double *vh, int len,
                              int D, double scale, double *orow, double *lse, double *s)
{
    for (int d = 0; d < D; ++d) orow[d] = 0.0;
    if (len == 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int j = 0; j < len; ++j) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += widen_bf16(qh[d]) * kh[(size_t)j * D + d];
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int j = 0; j < len; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int j = 0; j < len; ++j) {
        const double w = s[j] / l;
        for (int d = 0; d < D; ++d) orow[d] += w * vh[(size_t)j * D + d];
    }
    *lse = m + log(l);
}

/*
 * Paged decode over an FP8 KV cache.  The FasterTransformer read-through
 * (pptc.cn), section 3.3, stores the KV cache quantised (int8) and
 * dequantises it before use; section 4.2 enables FP8 on H100 and later.
 * Reading: K and V pages hold e4m3 codes in the layout of
 * oracle_attn_decode_paged ([num_pages][Hkv][page_size][D], one byte per
 * element) and KV head h's value is code * k_scale[h] (resp. v_scale[h]).
 * The cache is gathered through the block table and dequantised exactly to
 * fp64, then the same definition applies (Sq = 1, no mask).
 */
int oracle_attn_decode_paged_fp8(const uint16_t *q, const uint8_t *k_pages, const uint8_t *v_pages,
                                 const float *k_scale, const float *v_scale,
                                 const int32_t *block_table, int max_pages,
                                 const int32_t *seq_lens, int page_size, int num_pages,
                                 double *o, double *lse, int B, int Hq, int Hkv, int D,
                                 double scale, const uint8_t *heads_mask)
{
    int rc = check_shape(B, Hq, Hkv, 1, 0, D, scale);
    if (rc) return rc;
    if (page_size <= 0 || num_pages < 0 || max_pages < 0) return ORACLE_ERR_ARG;
    for (int h = 0; h < Hkv; ++h)
        if (!isfinite(k_scale[h]) || !isfinite(v_scale[h])) return ORACLE_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        long long len = seq_lens[b];
        if (len < 0 || (len + page_size - 1) / page_size > max_pages) return ORACLE_ERR_ARG;
        for (long long p = 0; p < (len + page_size - 1) / page_size; ++p) {
            int32_t phys = block_table[(size_t)b * max_pages + p];
            if (phys < 0 || phys >= num_pages) return ORACLE_ERR_ARG;
        }
    }
    const int g = Hq / Hkv;
    for (int b = 0; b < B; ++b) {
        const int len = seq_lens[b];
        const size_t per_head = (size_t)len * D;
        double *kc = (double *)malloc(sizeof(double) * (per_head * Hkv + 1));
        double *vc = (double *)malloc(sizeof(double) * (per_head * Hkv + 1));
        if (!kc || !vc) { free(kc); free(vc); return ORACLE_ERR_MEM; }
        for (int kvh = 0; kvh < Hkv; ++kvh)
            for (int t = 0; t < len; ++t) {
                const int32_t phys = block_table[(size_t)b * max_pages + t / page_size];
                const size_t src = (((size_t)phys * Hkv + kvh) * page_size + t % page_size) * D;
                const size_t dst = (size_t)kvh * per_head + (size_t)t * D;
                for (int d = 0; d < D; ++d) {
                    kc[dst + d] = oracle_e4m3_to_f64(k_pages[src + d]) * (double)k_scale[kvh];
                    vc[dst + d] = oracle_e4m3_to_f64(v_pages[src + d]) * (double)v_scale[kvh];
                }
            }
        int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
        for (int h = 0; h < Hq; ++h) {
            if (heads_mask && !heads_mask[(size_t)b * Hq + h]) continue;
            const int kvh = h / g;
            double *s = (double *)malloc(sizeof(double) * ((size_t)len + 1));
            if (!s) { failed |= 1; continue; }
            attend_decode_row(q + ((size_t)b * Hq + h) * D, kc + (size_t)kvh * per_head,
                              vc + (size_t)kvh * per_head, len, D, scale,
                              o + ((size_t)b * Hq + h) * D, lse + (size_t)b * Hq + h, s);
            free(s);
        }
        free(kc);
        free(vc);
        if (failed) return ORACLE_ERR_MEM;
    }
    return ORACLE_OK;
}

/*
 * Merge of partial attention results over disjoint key sets by their
 * log-sum-exp.  If part s attended keys K_s with lse_s = log sum_{j in K_s}
 * exp(s_j) and o_s = sum_{j in K_s} exp(s_j - lse_s) v_j, then over the union
 *   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) o_s.
 * (the max is subtracted before exponentiating, which changes nothing
 * mathematically).  Parts with lse_s = -inf (no keys) contribute nothing; if
 * every part is empty the row is o = 0, lse = -inf.
 *   o_parts [S][n_rows][D], lse_parts [S][n_rows]  ->  o [n_rows][D], lse [n_rows]
 */
int oracle_merge_lse(const double *o_parts, const double *lse_parts, int S, int n_rows,
                     int D, double *o, double *lse)
{
    if (S <= 0 || n_rows < 0 || D <= 0) return ORACLE_ERR_ARG;
    for (int r = 0; r < n_rows; ++r) {
        double m = -INFINITY;
        for (int s = 0; s < S; ++s)
            if (lse_parts[(size_t)s * n_rows + r] > m) m = lse_parts[(size_t)s * n_rows + r];
        double *orow = o + (size_t)r * D;
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double total = 0.0;
        for (int s = 0; s < S; ++s) {
            double ls = lse_parts[(size_t)s * n_rows + r];
            if (ls == -INFINITY) continue;
            total += exp(ls - m);
        }
        const double lse_r = m + log(total);
        for (int s = 0; s < S; ++s) {
            double ls = lse_parts[(size_t)s * n_rows + r];
            if (ls == -INFINITY) continue;
            const double w = exp(ls - lse_r);
            const double *op = o_parts + ((size_t)s * n_rows + r) * D;
            for (int d = 0; d < D; ++d) orow[d] += w * op[d];
        }
        lse[r] = lse_r;
    }
    return ORACLE_OK;
}
