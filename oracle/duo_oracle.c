/*
 * Plain fp64 CPU oracle for mixed-head (DuoAttention) attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this file's library. It shares no code, header, table
 * or helper with the CUDA path in mixed_head_kv_b200/.
 *
 * What it computes (DuoAttention abstract, "read the original abstract" on the
 * pith.science review page; restated on the sourcepulse project card, "How It
 * Works"): every attention head is either
 *   - a retrieval head, which keeps a full KV cache and attends to every
 *     previous token, or
 *   - a streaming head, which keeps a constant-length cache holding the
 *     attention-sink tokens and the most recent tokens, and attends only to
 *     those.
 * For GQA models the head type belongs to the KV head and every query head of
 * its group inherits it.
 *
 * Readings of points the pages leave open:
 *   - key set of a streaming head for a query at absolute position p:
 *       K(p) = { j <= p : j < sink  or  p - j < recent }
 *     ("recent" counts the query's own token; the union counts a key once);
 *   - retrieval head: K(p) = { 0 .. p } (causal);
 *   - scores s_j = scale * <q_p, k_j>, weights a_j = exp(s_j - max) / sum,
 *     output o_p = sum_j a_j v_j, everything in double precision from bf16
 *     inputs widened exactly;
 *   - streaming cache slots: slot p for a sink position p < sink, ring slot
 *     sink + (p - sink) mod recent otherwise (a fixed sink region plus a ring).
 *
 * All loops are the definitions written out: no blocking, no online softmax,
 * no reordering beyond summation order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bit pattern -> double (exact: bf16 is the top half of an IEEE binary32). */
static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Membership of key position j in the key set of a query at position p.
 * Retrieval head: every previous token. Streaming head: attention sinks plus
 * the recent window (DuoAttention abstract: a streaming head keeps only the
 * sink tokens and the latest tokens, in a cache of fixed size). */
int duo_oracle_key_allowed(int is_retrieval, int64_t p, int64_t j, int64_t sink, int64_t recent) {
    if (j < 0 || j > p) return 0;
    if (is_retrieval) return 1;
    return (j < sink) || (p - j < recent);
}

/* Softmax attention of one query row over the key/value rows listed in idx:
 * row idx[i] of keys/vals (D bf16 each). out[D] receives sum_i a_i v_i and
 * *wsum receives sum_i a_i (1 up to rounding). Returns 0, or -1 when the list
 * is empty or allocation fails. */
static int attend_indexed(const uint16_t* q, const uint16_t* keys, const uint16_t* vals, const int64_t* idx,
                          int64_t n, int D, double scale, double* out, double* wsum) {
    if (n <= 0) return -1;
    double* s = (double*)malloc(sizeof(double) * (size_t)n);
    if (!s) return -1;
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        const uint16_t* kr = keys + idx[i] * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16_to_double(q[d]) * bf16_to_double(kr[d]);
        s[i] = scale * dot;
        if (s[i] > m) m = s[i];
    }
    double denom = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        s[i] = exp(s[i] - m);
        denom += s[i];
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    double total = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        const uint16_t* vr = vals + idx[i] * D;
        double a = s[i] / denom;
        total += a;
        for (int d = 0; d < D; ++d) out[d] += a * bf16_to_double(vr[d]);
    }
    if (wsum) *wsum = total;
    free(s);
    return 0;
}

/* Attention of one query row over an explicit list of n key/value rows
 * (row i at keys + i*D). */
int duo_oracle_attend_rows(const uint16_t* q, const uint16_t* keys, const uint16_t* vals,
                           int64_t n, int D, double scale, double* out, double* wsum) {
    if (n <= 0) return -1;
    int64_t* idx = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
    if (!idx) return -1;
    for (int64_t i = 0; i < n; ++i) idx[i] = i;
    int rc = attend_indexed(q, keys, vals, idx, n, D, scale, out, wsum);
    free(idx);
    return rc;
}

/* Attention of one query at absolute position p of one head over the full
 * key/value history of its KV head (k_hist/v_hist: T rows, row j = position j),
 * restricted to the key set K(p) of that head's type. */
static int attend_masked(const uint16_t* q, const uint16_t* k_hist, const uint16_t* v_hist,
                         int64_t T, int D, int64_t p, int is_retrieval, int64_t sink,
                         int64_t recent, double scale, double* out, double* wsum) {
    int64_t last = p < T - 1 ? p : T - 1;
    int64_t n = 0;
    for (int64_t j = 0; j <= last; ++j) n += duo_oracle_key_allowed(is_retrieval, p, j, sink, recent);
    if (n == 0) return -1;
    int64_t* idx = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
    if (!idx) return -1;
    int64_t c = 0;
    for (int64_t j = 0; j <= last; ++j)
        if (duo_oracle_key_allowed(is_retrieval, p, j, sink, recent)) idx[c++] = j;
    int rc = attend_indexed(q, k_hist, v_hist, idx, n, D, scale, out, wsum);
    free(idx);
    return rc;
}

/* Mixed-head attention for a batch of queries.
 *   q      [B][Hq][NQ][D]   bf16 bits; query i of every head sits at position qpos[i]
 *   k, v   [B][Hkv][T][D]   bf16 bits; row j is the token at position j
 *   is_retrieval [Hkv]      1 = retrieval KV head, 0 = streaming KV head
 *   out    [B][Hq][NQ][D]   double
 *   wsum   [B][Hq][NQ]      double, optional: sum of the softmax weights
 * Query head h reads KV head h / (Hq / Hkv). Returns the number of rows that
 * failed (empty key set), 0 on success. Threads: OpenMP over (b, h, i). */
int64_t duo_oracle_attention(const uint16_t* q, const int64_t* qpos, const uint16_t* k,
                             const uint16_t* v, const uint8_t* is_retrieval, int B, int Hq,
                             int Hkv, int64_t NQ, int64_t T, int D, int64_t sink, int64_t recent,
                             double scale, double* out, double* wsum) {
    int G = Hq / Hkv;
    int64_t total = (int64_t)B * Hq * NQ;
    int64_t failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : failed)
    for (int64_t idx = 0; idx < total; ++idx) {
        int64_t i = idx % NQ;
        int h = (int)((idx / NQ) % Hq);
        int b = (int)(idx / (NQ * Hq));
        int g = h / G;
        const uint16_t* qr = q + (((int64_t)b * Hq + h) * NQ + i) * D;
        const uint16_t* kh = k + ((int64_t)b * Hkv + g) * T * D;
        const uint16_t* vh = v + ((int64_t)b * Hkv + g) * T * D;
        double ws = 0.0;
        int rc = attend_masked(qr, kh, vh, T, D, qpos[i], is_retrieval[g], sink, recent, scale,
                               out + idx * D, &ws);
        if (wsum) wsum[idx] = ws;
        if (rc != 0) failed += 1;
    }
    return failed;
}

/* Cache slot model: which absolute position each slot of one head's cache
 * holds after `len` tokens were appended (closed form), -1 for an empty slot.
 *   retrieval head: slot j holds position j for j < len;
 *   streaming head (nslots = sink + recent): slot s < sink holds position s;
 *     slot sink + r holds the latest position p < len with p >= sink and
 *     (p - sink) mod recent == r. */
void duo_oracle_slot_positions(int is_retrieval, int64_t sink, int64_t recent, int64_t len,
                               int64_t nslots, int64_t* pos) {
    for (int64_t s = 0; s < nslots; ++s) {
        pos[s] = -1;
        if (is_retrieval || s < sink) {
            if (s < len) pos[s] = s;
            continue;
        }
        int64_t r = s - sink;
        if (r >= recent) continue;
        int64_t best = -1;
        for (int64_t p = sink + r; p < len; p += recent) best = p; /* latest writer wins */
        pos[s] = best;
    }
}

/* Threads the OpenMP runtime will use for duo_oracle_attention. */
int duo_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------
 * FP8 E4M3 retrieval caches (a next step of this library: the pages reach
 * their longest contexts only together with KV quantization). Reading: each
 * retrieval-head element x (bf16) is stored as the E4M3 code of x * inv_scale,
 * the product taken in fp32 (inv_scale = the fp32 reciprocal of a per-head
 * scale), rounded to nearest with ties to even and saturated to +-448; it is
 * read back as value(code) * scale.
 *
 * E4M3 (the "fn" variant of the OCP 8-bit floating-point formats): 1 sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the
 * subnormals m * 2^-9; exponent field 15 with mantissa 7 is NaN (no infinity);
 * the largest finite magnitude is 1.75 * 2^8 = 448.
 * ---------------------------------------------------------------------- */

/* Value of an E4M3 code (NaN for 0x7F and 0xFF). */
double duo_oracle_e4m3_value(uint8_t c) {
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* E4M3 code of x: round to nearest, ties to even; magnitudes above 448
 * (infinity included) saturate to 448; NaN gives 0x7F. */
uint8_t duo_oracle_e4m3_code(double x) {
    if (isnan(x)) return 0x7F;
    const uint8_t s = signbit(x) ? 0x80 : 0x00;
    const double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(s | 0x7E);
    int e = (int)floor(log2(a > 0.0 ? a : 1.0));
    if (a == 0.0) return s;
    if (e < -6) { /* subnormal: units of 2^-9 */
        const double m = nearbyint(ldexp(a, 9)); /* default rounding mode: to nearest, ties to even */
        return (uint8_t)(s | (int)m);           /* m == 8 is the smallest normal, code 0x08 */
    }
    /* guard against log2 rounding at exact powers of two */
    if (ldexp(1.0, e) > a) --e;
    if (ldexp(1.0, e + 1) <= a) ++e;
    double m = nearbyint((ldexp(a, -e) - 1.0) * 8.0);
    if (m == 8.0) { m = 0.0; ++e; }
    if (e > 8 || (e == 8 && m > 6.0)) return (uint8_t)(s | 0x7E); /* rounded past 448 */
    return (uint8_t)(s | ((e + 7) << 3) | (int)m);
}

/* Codes of n bf16 values times inv_scale, the product rounded to fp32 first. */
void duo_oracle_e4m3_quantize(const uint16_t* x, int64_t n, float inv_scale, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        const float prod = (float)bf16_to_double(x[i]) * inv_scale;
        out[i] = duo_oracle_e4m3_code((double)prod);
    }
}

/* Attention of one query row (bf16) over n key/value rows held as E4M3 codes
 * of a quantized retrieval cache: key element = value(code) * k_scale, value
 * element = value(code) * v_scale; otherwise the same definition as
 * duo_oracle_attend_rows. */
int duo_oracle_attend_rows_e4m3(const uint16_t* q, const uint8_t* k_codes, const uint8_t* v_codes, int64_t n, int D,
                                double k_scale, double v_scale, double scale, double* out, double* wsum) {
    if (n <= 0) return -1;
    double* s = (double*)malloc(sizeof(double) * (size_t)n);
    if (!s) return -1;
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_to_double(q[d]) * (duo_oracle_e4m3_value(k_codes[i * D + d]) * k_scale);
        s[i] = scale * dot;
        if (s[i] > m) m = s[i];
    }
    double denom = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        s[i] = exp(s[i] - m);
        denom += s[i];
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    double total = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        const double a = s[i] / denom;
        total += a;
        for (int d = 0; d < D; ++d) out[d] += a * (duo_oracle_e4m3_value(v_codes[i * D + d]) * v_scale);
    }
    if (wsum) *wsum = total;
    free(s);
    return 0;
}
