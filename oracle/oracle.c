/*
 * Float64 CPU oracle for grouped-query scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, written out, no blocking, no online
 * softmax).  For batch b, query head h, query row s, with group size
 * g = Hq / Hkv and K/V head kvh = h / g:
 *
 *     pos   = q_offset + s
 *     T     = { t in [0, Skv) : !causal  or  t <= pos }
 *     z_t   = scale * sum_d Q[b,s,h,d] * K[b,t,kvh,d]
 *     m     = max_{t in T} z_t
 *     l     = sum_{t in T} exp(z_t - m)
 *     O[b,s,h,:] = sum_{t in T} exp(z_t - m) / l * V[b,t,kvh,:]
 *     LSE[b,h,s] = m + ln(l)                      (natural log, scaled logits)
 *
 * Sources on the pages:
 *   - grouped-query heads sharing one K/V head: "ggml-org/llama.cpp PR #28507",
 *     Setup ("GQA 8") and the FLASH_ATTN_EXT test case list (nr23 broadcast
 *     ratio, mask=1), read as the contiguous-group broadcast kvh = h / g;
 *   - the scale applied to Q.K: "AstrAI commit log, gqa_prefill_attn_mma.cuh",
 *     the pre-scaled Q item (here the scale multiplies the exact fp64 dot
 *     product, which is the same quantity without a rounding step);
 *   - per-row (max, rowsum) metadata and the merge of split tiles:
 *     "Anbeeld/beellama.cpp PR #149", Overview (ub>64 fix: every block
 *     publishes its (max, rowsum)) and the review's note on the combine
 *     kernel for parallel_blocks > 1.
 *
 * Readings where the pages are silent:
 *   - layout: Q, O are [B, Sq, Hq, D]; K, V are [B, Skv, Hkv, D];
 *     LSE is [B, Hq, Sq]; all contiguous, row-major;
 *   - causal alignment: key t is visible to row s iff t <= q_offset + s;
 *   - split sigma of num_splits covers keys [sigma*c, min((sigma+1)*c, Skv)),
 *     c = ceil(Skv / num_splits); a split with no visible key for a row
 *     publishes lse = -inf and O = 0 for that row, and the merge gives it
 *     weight zero.
 *
 * Every input is a double array; callers widen bf16 values exactly.
 *
 * Optional terms of the logit (the *_ex functions; all off by default), from
 * the parameters of the FLASH_ATTN_EXT operator ("ggml-org/llama.cpp PR
 * #28507", Crash 1: sinks, max_bias, logit_softcap), read as follows:
 *   softcap c > 0:      z_t = c * tanh(z_t / c)            (on the scaled logit)
 *   ALiBi max_bias > 0: z_t += slope_h * (t - pos), slopes geometric per head:
 *                       n2 = largest power of two <= Hq, m0 = 2^(-max_bias/n2),
 *                       m1 = 2^(-max_bias/(2 n2)); slope_h = m0^(h+1) for
 *                       h < n2, else m1^(2(h-n2)+1)
 *   sink logit s_h:     one more term exp(s_h) in the softmax denominator
 *                       (and in the LSE), with no value row
 *   window w > 0:       key t is visible only if pos - w < t (with causal,
 *                       each row sees its w most recent keys)
 *   additive mask M:    z_t += M[b, s, t] (the `mask` parameter of the same
 *                       test case; -inf removes the key), after softcap and
 *                       ALiBi; a row whose every logit is -inf, with no
 *                       sink, has O = 0 and LSE = -inf
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static int64_t q_index(int64_t b, int64_t s, int64_t h, int64_t Sq, int64_t Hq, int64_t D) {
    return ((b * Sq + s) * Hq + h) * D;
}

static int64_t kv_index(int64_t b, int64_t t, int64_t kvh, int64_t Skv, int64_t Hkv, int64_t D) {
    return ((b * Skv + t) * Hkv + kvh) * D;
}

typedef struct {
    double softcap;         /* 0: off */
    double alibi_max_bias;  /* 0: off */
    const double* sinks;    /* NULL: off; else [Hq] sink logits */
    int64_t window;         /* 0: off */
    const double* mask;     /* NULL: off; else additive mask, element (b, s, t) at */
    int64_t mask_sb;        /*   mask[b * mask_sb + s * mask_ss + t] (mask_sb = 0: */
    int64_t mask_ss;        /*   one mask for every sequence) */
} oracle_opts;

/* ALiBi slope of head h out of Hq (see the header comment). */
double oracle_alibi_slope(int64_t h, int64_t Hq, double max_bias) {
    int64_t n2 = 1;
    while (n2 * 2 <= Hq) n2 *= 2;
    const double m0 = pow(2.0, -max_bias / (double)n2);
    const double m1 = pow(2.0, -max_bias / 2.0 / (double)n2);
    return h < n2 ? pow(m0, (double)(h + 1)) : pow(m1, (double)(2 * (h - n2) + 1));
}

/* One output row restricted to keys [t_lo, t_hi).  z is scratch of length
 * >= t_hi - t_lo.  Returns the LSE (or -inf when no key is visible and there
 * is no sink, in which case o_row is all zeros).  opt may be NULL. */
static double attend_row(const double* q, const double* k, const double* v,
                         int64_t b, int64_t h, int64_t s,
                         int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                         int64_t q_offset, int causal, double scale,
                         int64_t t_lo, int64_t t_hi, double* z, double* o_row,
                         const oracle_opts* opt) {
    const int64_t g = Hq / Hkv;
    const int64_t kvh = h / g;
    const int64_t pos = q_offset + s;
    const double* qr = q + q_index(b, s, h, Sq, Hq, D);
    const double softcap = opt ? opt->softcap : 0.0;
    const double slope = (opt && opt->alibi_max_bias > 0.0) ? oracle_alibi_slope(h, Hq, opt->alibi_max_bias) : 0.0;
    const int has_sink = opt && opt->sinks;

    int64_t first = t_lo;                      /* inclusive lower bound of T */
    if (opt && opt->window > 0 && pos - opt->window + 1 > first) first = pos - opt->window + 1;
    int64_t last = t_hi;                       /* exclusive upper bound of T */
    if (causal && pos + 1 < last) last = pos + 1;
    for (int64_t d = 0; d < D; ++d) o_row[d] = 0.0;
    if (last <= first && !has_sink) return -INFINITY;

    /* pass 1: logits and their maximum (the sink logit takes part) */
    double m = has_sink ? opt->sinks[h] : -INFINITY;
    for (int64_t t = first; t < last; ++t) {
        const double* kr = k + kv_index(b, t, kvh, Skv, Hkv, D);
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += qr[d] * kr[d];
        const double zt = scale * acc;
        const double zc = softcap > 0.0 ? softcap * tanh(zt / softcap) : zt;
        z[t - t_lo] = zc + slope * (double)(t - pos);
        if (opt && opt->mask) z[t - t_lo] += opt->mask[b * opt->mask_sb + s * opt->mask_ss + t];
        if (z[t - t_lo] > m) m = z[t - t_lo];
    }
    /* every visible logit masked to -inf and no sink: no key takes part */
    if (m == -INFINITY) return -INFINITY;
    /* pass 2: exponentials, their sum, and the weighted sum of V rows */
    double l = has_sink ? exp(opt->sinks[h] - m) : 0.0;
    for (int64_t t = first; t < last; ++t) {
        const double p = exp(z[t - t_lo] - m);
        z[t - t_lo] = p;
        l += p;
    }
    for (int64_t t = first; t < last; ++t) {
        const double w = z[t - t_lo] / l;
        const double* vr = v + kv_index(b, t, kvh, Skv, Hkv, D);
        for (int64_t d = 0; d < D; ++d) o_row[d] += w * vr[d];
    }
    return m + log(l);
}

/* Full attention: out [B,Sq,Hq,D], lse [B,Hq,Sq]; opt may be NULL. */
static void attention_impl(const double* q, const double* k, const double* v,
                           double* out, double* lse,
                           int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                           int64_t q_offset, int causal, double scale, const oracle_opts* opt) {
    const int64_t rows = B * Hq * Sq;
#pragma omp parallel
    {
        double* z = (double*)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t b = r / (Hq * Sq);
            const int64_t h = (r / Sq) % Hq;
            const int64_t s = r % Sq;
            double* o_row = out + q_index(b, s, h, Sq, Hq, D);
            lse[(b * Hq + h) * Sq + s] =
                attend_row(q, k, v, b, h, s, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale,
                           0, Skv, z, o_row, opt);
        }
        free(z);
    }
}

/* Selected rows only: rows is n triples (b, h, s); out_rows [n, D]; lse_rows [n]. */
static void attention_rows_impl(const double* q, const double* k, const double* v,
                                const int64_t* rows, int64_t n, double* out_rows, double* lse_rows,
                                int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                                int64_t q_offset, int causal, double scale, const oracle_opts* opt) {
    (void)B;
#pragma omp parallel
    {
        double* z = (double*)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n; ++i) {
            const int64_t b = rows[3 * i], h = rows[3 * i + 1], s = rows[3 * i + 2];
            lse_rows[i] = attend_row(q, k, v, b, h, s, Hq, Hkv, Sq, Skv, D, q_offset, causal,
                                     scale, 0, Skv, z, out_rows + i * D, opt);
        }
        free(z);
    }
}

/* The normalised attention weights of one row, written to p[0..Skv); masked keys get 0. */
void oracle_probs(const double* q, const double* k,
                  int64_t b, int64_t h, int64_t s, double* p,
                  int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                  int64_t q_offset, int causal, double scale) {
    const int64_t g = Hq / Hkv;
    const int64_t kvh = h / g;
    const int64_t pos = q_offset + s;
    const double* qr = q + q_index(b, s, h, Sq, Hq, D);
    double m = -INFINITY;
    for (int64_t t = 0; t < Skv; ++t) {
        if (causal && t > pos) { p[t] = -INFINITY; continue; }
        const double* kr = k + kv_index(b, t, kvh, Skv, Hkv, D);
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += qr[d] * kr[d];
        p[t] = scale * acc;
        if (p[t] > m) m = p[t];
    }
    double l = 0.0;
    for (int64_t t = 0; t < Skv; ++t) {
        p[t] = (p[t] == -INFINITY) ? 0.0 : exp(p[t] - m);
        l += p[t];
    }
    for (int64_t t = 0; t < Skv; ++t) p[t] /= l;
}

/* Split-KV partials: pout [S,B,Sq,Hq,D] (each split normalised on its own keys),
 * plse [S,B,Hq,Sq].  Sinks never enter a partial (the merge adds them once). */
static void split_impl(const double* q, const double* k, const double* v,
                       double* pout, double* plse,
                       int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                       int64_t q_offset, int causal, double scale, int64_t num_splits,
                       const oracle_opts* opt) {
    const int64_t chunk = (Skv + num_splits - 1) / num_splits;
    const int64_t rows = B * Hq * Sq;
    const int64_t total = num_splits * rows;
#pragma omp parallel
    {
        double* z = (double*)malloc(sizeof(double) * (size_t)(chunk > 0 ? chunk : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = 0; i < total; ++i) {
            const int64_t sigma = i / rows;
            const int64_t r = i % rows;
            const int64_t b = r / (Hq * Sq);
            const int64_t h = (r / Sq) % Hq;
            const int64_t s = r % Sq;
            int64_t lo = sigma * chunk, hi = lo + chunk;
            if (lo > Skv) lo = Skv;
            if (hi > Skv) hi = Skv;
            double* o_row = pout + sigma * (B * Sq * Hq * D) + q_index(b, s, h, Sq, Hq, D);
            plse[sigma * rows + (b * Hq + h) * Sq + s] =
                attend_row(q, k, v, b, h, s, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale,
                           lo, hi, z, o_row, opt);
        }
        free(z);
    }
}

/* Merge of split partials by their log-sum-exp:
 *   M = max_sigma lse_sigma,  w_sigma = exp(lse_sigma - M),
 *   O = sum w_sigma O_sigma / sum w_sigma,  lse = M + ln(sum w_sigma).
 * A split with lse = -inf has weight 0; if every split is -inf the row is
 * O = 0, lse = -inf.  A sink logit s_h (sinks != NULL) joins M and adds
 * exp(s_h - M) to the denominator only. */
static void merge_impl(const double* pout, const double* plse, double* out, double* lse,
                       int64_t B, int64_t Hq, int64_t Sq, int64_t D, int64_t num_splits,
                       const double* sinks) {
    const int64_t rows = B * Hq * Sq;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t b = r / (Hq * Sq);
        const int64_t h = (r / Sq) % Hq;
        const int64_t s = r % Sq;
        double* o_row = out + q_index(b, s, h, Sq, Hq, D);
        double M = sinks ? sinks[h] : -INFINITY;
        for (int64_t sg = 0; sg < num_splits; ++sg) {
            const double x = plse[sg * rows + r];
            if (x > M) M = x;
        }
        for (int64_t d = 0; d < D; ++d) o_row[d] = 0.0;
        if (M == -INFINITY) { lse[r] = -INFINITY; continue; }
        double wsum = sinks ? exp(sinks[h] - M) : 0.0;
        for (int64_t sg = 0; sg < num_splits; ++sg) {
            const double x = plse[sg * rows + r];
            if (x == -INFINITY) continue;
            const double w = exp(x - M);
            wsum += w;
            const double* pr = pout + sg * (B * Sq * Hq * D) + q_index(b, s, h, Sq, Hq, D);
            for (int64_t d = 0; d < D; ++d) o_row[d] += w * pr[d];
        }
        for (int64_t d = 0; d < D; ++d) o_row[d] /= wsum;
        lse[r] = M + log(wsum);
    }
}

/* ---- public entry points: the plain definition, and the *_ex variants with
 * the optional logit terms (softcap, ALiBi, sinks, window) ---- */
void oracle_attention(const double* q, const double* k, const double* v, double* out, double* lse,
                      int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                      int64_t q_offset, int causal, double scale) {
    attention_impl(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale, NULL);
}

void oracle_attention_rows(const double* q, const double* k, const double* v,
                           const int64_t* rows, int64_t n, double* out_rows, double* lse_rows,
                           int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                           int64_t q_offset, int causal, double scale) {
    attention_rows_impl(q, k, v, rows, n, out_rows, lse_rows, B, Hq, Hkv, Sq, Skv, D, q_offset, causal,
                        scale, NULL);
}

void oracle_split(const double* q, const double* k, const double* v, double* pout, double* plse,
                  int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                  int64_t q_offset, int causal, double scale, int64_t num_splits) {
    split_impl(q, k, v, pout, plse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale, num_splits, NULL);
}

void oracle_merge(const double* pout, const double* plse, double* out, double* lse,
                  int64_t B, int64_t Hq, int64_t Sq, int64_t D, int64_t num_splits) {
    merge_impl(pout, plse, out, lse, B, Hq, Sq, D, num_splits, NULL);
}

static oracle_opts make_opts(double softcap, double alibi_max_bias, const double* sinks, int64_t window,
                             const double* mask, int64_t mask_sb, int64_t mask_ss) {
    oracle_opts o;
    o.softcap = softcap;
    o.alibi_max_bias = alibi_max_bias;
    o.sinks = sinks;
    o.window = window;
    o.mask = mask;
    o.mask_sb = mask_sb;
    o.mask_ss = mask_ss;
    return o;
}

void oracle_attention_ex(const double* q, const double* k, const double* v, double* out, double* lse,
                         int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                         int64_t q_offset, int causal, double scale,
                         double softcap, double alibi_max_bias, const double* sinks, int64_t window,
                         const double* mask, int64_t mask_sb, int64_t mask_ss) {
    const oracle_opts o = make_opts(softcap, alibi_max_bias, sinks, window, mask, mask_sb, mask_ss);
    attention_impl(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale, &o);
}

void oracle_attention_rows_ex(const double* q, const double* k, const double* v,
                              const int64_t* rows, int64_t n, double* out_rows, double* lse_rows,
                              int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                              int64_t q_offset, int causal, double scale,
                              double softcap, double alibi_max_bias, const double* sinks, int64_t window,
                              const double* mask, int64_t mask_sb, int64_t mask_ss) {
    const oracle_opts o = make_opts(softcap, alibi_max_bias, sinks, window, mask, mask_sb, mask_ss);
    attention_rows_impl(q, k, v, rows, n, out_rows, lse_rows, B, Hq, Hkv, Sq, Skv, D, q_offset, causal,
                        scale, &o);
}

void oracle_split_ex(const double* q, const double* k, const double* v, double* pout, double* plse,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                     int64_t q_offset, int causal, double scale, int64_t num_splits,
                     double softcap, double alibi_max_bias, int64_t window,
                     const double* mask, int64_t mask_sb, int64_t mask_ss) {
    const oracle_opts o = make_opts(softcap, alibi_max_bias, NULL, window, mask, mask_sb, mask_ss);
    split_impl(q, k, v, pout, plse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale, num_splits, &o);
}

void oracle_merge_ex(const double* pout, const double* plse, double* out, double* lse,
                     int64_t B, int64_t Hq, int64_t Sq, int64_t D, int64_t num_splits, const double* sinks) {
    merge_impl(pout, plse, out, lse, B, Hq, Sq, D, num_splits, sinks);
}

/* Value of an fp8 e4m3 code: 1 sign bit, 4 exponent bits with bias 7 and 3
 * mantissa bits.  Exponent 0 is subnormal (m/8 * 2^-6); codes 0x7f and 0xff
 * are NaN; the format has no infinity ("ggml-org/llama.cpp PR #28507",
 * Setup: the q8_0 K cache; "Anbeeld/beellama.cpp PR #149", Overview: a
 * quantised K/V cache read by the attention kernel). */
double oracle_e4m3_value(int code) {
    const int sign = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Attention over an fp8 e4m3 K/V cache with one scale per K/V head:
 * K = e4m3(k_codes) * k_scale[kvh], V = e4m3(v_codes) * v_scale[kvh], then
 * the extended attention above (codes [B, Skv, Hkv, D], one byte each). */
void oracle_attention_fp8(const double* q, const unsigned char* k_codes, const unsigned char* v_codes,
                          const double* k_scale, const double* v_scale, double* out, double* lse,
                          int64_t B, int64_t Hq, int64_t Hkv, int64_t Sq, int64_t Skv, int64_t D,
                          int64_t q_offset, int causal, double scale,
                          double softcap, double alibi_max_bias, const double* sinks, int64_t window,
                          const double* mask, int64_t mask_sb, int64_t mask_ss) {
    const int64_t n = B * Skv * Hkv * D;
    double* k = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double* v = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        const int64_t kvh = (i / D) % Hkv;
        k[i] = oracle_e4m3_value(k_codes[i]) * k_scale[kvh];
        v[i] = oracle_e4m3_value(v_codes[i]) * v_scale[kvh];
    }
    const oracle_opts o = make_opts(softcap, alibi_max_bias, sinks, window, mask, mask_sb, mask_ss);
    attention_impl(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, q_offset, causal, scale, &o);
    free(k);
    free(v);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
