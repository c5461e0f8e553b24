/*
 * oracle.c -- plain, slow, fp64 CPU reference of the hybrid compressed
 * attention hot path (CSA + HCA).  TEST INFRASTRUCTURE ONLY: it is loaded by
 * the tests, by the package's smoke check and by the benchmark's CPU-baseline
 * leg, never by the product path.  It shares no code with the CUDA library.
 *
 * Every routine is a literal transcription of the definition it cites, in
 * fp64, with no blocking, fusion or reordering.  Inputs are bf16 bit patterns
 * (uint16) and fp32 parameters, widened exactly to double.
 *
 * Sources (web pages, cited by title and section):
 *  [F]  "Frontier Techniques: NTK RoPE, CSA+HCA, QAT, MTP", section 2
 *       "CSA + HCA -- sparse attention at 1M tokens" (2.1 CSA: compress m=4,
 *       top-1024 by the Lightning Indexer, 128-token raw sliding window;
 *       2.2 HCA: compress m'=128, dense attention over all entries).
 *  [V4] "DeepSeek V4 comprimeix el context: aixi funcionen CSA i HCA",
 *       sections "DeepSeek comprimeix la dimensio temporal" (shared 512-d KV,
 *       softmax-weighted sum with a separate weight per channel),
 *       "Finestres solapades per evitar fronteres artificials" (overlapping
 *       windows, weights recomputed inside each window, incomplete block kept
 *       raw), "CSA: buscar primer i atendre despres" (a light indexer scores
 *       the compressed entries and keeps the best; attention over the chosen
 *       entries plus the local window), "HCA: un resum global 128 vegades mes
 *       curt" (dense attention over every 128-token summary).
 *
 * Readings where the pages leave a step open (each stated where used):
 *  R1 window geometry: CSA entry j covers tokens [m*j - m, m*j + m) clipped at
 *     0 (a window of 2m, so consecutive windows overlap by m tokens); HCA entry
 *     j covers [m'*j, m'*j + m').  An entry exists once its last token exists:
 *     m*(j+1) <= L.
 *  R2 per-offset bias: the logit of token t in entry j's window is
 *     logit_t[c] + bias[t - start_j][c], start_j the UNCLIPPED window start.
 *  R3 indexer score s_j = sum_h w_h * relu(q^I_h . K^I_j), no scale; indexer
 *     keys are compressed with the softmax weights of channels 0..d_I-1.
 *  R4 top-k order: score descending, ties to the lower entry index; fewer
 *     than k candidates selects all, the rest of the list is -1.
 *  R5 a query at visible length L sees raw tokens [0, L): CSA entries
 *     j < floor(L/m), HCA entries j < floor(L/m'), window [max(0,L-W), L).
 *  R6 K = V = the stored bf16 vector (MQA over the shared latent); scale
 *     1/sqrt(d); the CSA and HCA partials are merged by log-sum-exp.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- bf16 <-> double (the oracle's own conversions) -------------------- */

static double bf16_to_double(uint16_t h) {
    union { uint32_t u; float f; } c;
    c.u = (uint32_t)h << 16;
    return (double)c.f;
}

/* Round-to-nearest-even of a finite double to bf16.  Done by scaling to the
 * bf16 grid of the value's binade and rounding with rint (ties to even under
 * the default rounding mode).  Subnormal bf16 results are produced exactly
 * the same way on the subnormal grid. */
static uint16_t double_to_bf16(double v) {
    if (v != v) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1): binade exponent e-1 */
    int be = e - 1;               /* a in [2^be, 2^(be+1)) */
    if (be < -126) be = -126;     /* subnormal grid */
    double ulp = ldexp(1.0, be - 7);
    double r = rint(a / ulp) * ulp; /* exact: a/ulp is exact (power-of-two scale) */
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
    union { uint32_t u; float f; } c;
    c.f = (float)r;               /* exact: r has at most 8 significant bits */
    return (uint16_t)(sign | (uint16_t)((c.u >> 16) & 0x7FFF));
}

void oracle_round_bf16(const double* in, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(in[i]);
}

void oracle_bf16_to_double(const uint16_t* in, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_double(in[i]);
}

/* ---- a1 / a2: the token-axis compressor -------------------------------- */
/*
 * [V4] "DeepSeek comprimeix la dimensio temporal": an entry is a softmax-
 * weighted sum of the tokens it summarises, with a separate weight for every
 * channel; "Finestres solapades ...": windows overlap and the weights are
 * recomputed inside each window.  [F] 2.1 / 2.2: m = 4 (CSA), m' = 128 (HCA).
 *
 * For each entry j in js[0..n): window start s = m*j - (win - m) (R1; win = 2m
 * gives the overlapping CSA window, win = m the HCA block), tokens
 * t in [max(0, s), m*j + m).  Per channel c:
 *   z_t   = logit_t[c] + bias[t - s][c]                      (R2)
 *   w_t   = exp(z_t) / sum_t' exp(z_t')                      (softmax over the window)
 *   E[c]  = sum_t w_t * x_t[c]
 *   KI[c] = sum_t w_t * kI_t[c]   for c < d_I                (R3)
 * x, logit: [L, d]; kI: [L, d_I] or NULL; bias: [win, d].
 * Outputs (unrounded fp64): E [n, d]; KI [n, d_I] when kI and KI are given.
 * Returns 0, or -1 if some j is not yet complete (m*(j+1) > L) or negative.
 */
int oracle_compress(const uint16_t* x, const uint16_t* logit, const float* bias, const uint16_t* kI,
                    int64_t L, int d, int d_I, int m, int win, const int64_t* js, int64_t n,
                    double* E, double* KI) {
    if (win != m && win != 2 * m) return -2;
    double* z = (double*)malloc(sizeof(double) * (size_t)win);
    double* w = (double*)malloc(sizeof(double) * (size_t)win);
    if (!z || !w) { free(z); free(w); return -3; }
    int rc = 0;
    for (int64_t e = 0; e < n; ++e) {
        int64_t j = js[e];
        if (j < 0 || (int64_t)m * (j + 1) > L) { rc = -1; break; }
        int64_t s = (int64_t)m * j - (win - m);
        int64_t t0 = s < 0 ? 0 : s;
        int64_t t1 = (int64_t)m * j + m;
        int cnt = (int)(t1 - t0);
        for (int c = 0; c < d; ++c) {
            double zmax = -INFINITY;
            for (int i = 0; i < cnt; ++i) {
                int64_t t = t0 + i;
                z[i] = bf16_to_double(logit[t * d + c]) + (double)bias[(t - s) * d + c];
                if (z[i] > zmax) zmax = z[i];
            }
            double den = 0.0;
            for (int i = 0; i < cnt; ++i) { w[i] = exp(z[i] - zmax); den += w[i]; }
            for (int i = 0; i < cnt; ++i) w[i] /= den;
            double acc = 0.0;
            for (int i = 0; i < cnt; ++i) acc += w[i] * bf16_to_double(x[(t0 + i) * d + c]);
            E[e * d + c] = acc;
            if (kI && KI && c < d_I) {
                double acck = 0.0;
                for (int i = 0; i < cnt; ++i) acck += w[i] * bf16_to_double(kI[(t0 + i) * d_I + c]);
                KI[e * d_I + c] = acck;
            }
        }
    }
    free(z);
    free(w);
    return rc;
}

/* The softmax weights themselves, for the invariant tests: W [n, cnt_max=win, d],
 * zero where the window is clipped. */
int oracle_compress_weights(const uint16_t* logit, const float* bias, int64_t L, int d, int m, int win,
                            const int64_t* js, int64_t n, double* Wout) {
    for (int64_t e = 0; e < n; ++e) {
        int64_t j = js[e];
        if (j < 0 || (int64_t)m * (j + 1) > L) return -1;
        int64_t s = (int64_t)m * j - (win - m);
        for (int c = 0; c < d; ++c) {
            double zmax = -INFINITY;
            for (int o = 0; o < win; ++o) {
                int64_t t = s + o;
                if (t < 0) continue;
                double zz = bf16_to_double(logit[t * d + c]) + (double)bias[o * d + c];
                if (zz > zmax) zmax = zz;
            }
            double den = 0.0;
            for (int o = 0; o < win; ++o) {
                int64_t t = s + o;
                if (t < 0) continue;
                den += exp(bf16_to_double(logit[t * d + c]) + (double)bias[o * d + c] - zmax);
            }
            for (int o = 0; o < win; ++o) {
                int64_t t = s + o;
                double v = 0.0;
                if (t >= 0) v = exp(bf16_to_double(logit[t * d + c]) + (double)bias[o * d + c] - zmax) / den;
                Wout[(e * win + o) * d + c] = v;
            }
        }
    }
    return 0;
}

/* ---- a3: Lightning-Indexer scores --------------------------------------- */
/*
 * [V4] "CSA: buscar primer i atendre despres": a lightweight indexer scores
 * every compressed entry.  [F] 2.1: the Lightning Indexer.  Score (R3):
 *   s_j = sum_h w_h * relu( sum_c qI[h][c] * KI_j[c] ),  j in [0, n_entries).
 */
void oracle_index_scores(const uint16_t* qI, const float* w, int H_I, int d_I, const uint16_t* KI,
                         int64_t n_entries, double* s) {
    for (int64_t j = 0; j < n_entries; ++j) {
        double acc = 0.0;
        for (int h = 0; h < H_I; ++h) {
            double dot = 0.0;
            for (int c = 0; c < d_I; ++c) dot += bf16_to_double(qI[h * d_I + c]) * bf16_to_double(KI[j * d_I + c]);
            acc += (double)w[h] * (dot > 0.0 ? dot : 0.0);
        }
        s[j] = acc;
    }
}

/* ---- a4: top-k selection ------------------------------------------------- */

typedef struct { double s; int64_t j; } scored_t;

static int by_score_desc_index_asc(const void* pa, const void* pb) {
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int by_index_asc(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/* [F] 2.1: keep the top-k entries (k = 1024).  R4: order by score descending
 * with ties to the lower index (a full sort, then truncation); the kept
 * indices are written in ascending order, the rest of idx[0..k) is -1. */
int oracle_topk(const double* s, int64_t n, int k, int32_t* idx) {
    scored_t* v = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    if (!v) return -3;
    for (int64_t j = 0; j < n; ++j) { v[j].s = s[j]; v[j].j = j; }
    qsort(v, (size_t)n, sizeof(scored_t), by_score_desc_index_asc);
    int64_t keep = n < k ? n : k;
    for (int64_t i = 0; i < keep; ++i) idx[i] = (int32_t)v[i].j;
    qsort(idx, (size_t)keep, sizeof(int32_t), by_index_asc);
    for (int64_t i = keep; i < k; ++i) idx[i] = -1;
    free(v);
    return 0;
}

/* ---- a5 / a6: softmax attention over an explicit key list --------------- */
/*
 * One query vector per head q_h [d]; keys = values = the listed bf16 rows
 * (R6, MQA over the shared latent).  For each head:
 *   l_i = scale * q_h . key_i,   lse = log sum_i exp(l_i),
 *   O_h = sum_i exp(l_i - lse) * key_i.
 * An empty list gives lse = -inf and O = 0.
 */
static void attend_rows(const uint16_t* q, int H, int d, const uint16_t* const* rows, int64_t n, double scale,
                        double* O, double* lse) {
    double* l = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int h = 0; h < H; ++h) {
        double* o = O + (int64_t)h * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (n == 0) { lse[h] = -INFINITY; continue; }
        double lmax = -INFINITY;
        for (int64_t i = 0; i < n; ++i) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += bf16_to_double(q[h * d + c]) * bf16_to_double(rows[i][c]);
            l[i] = scale * dot;
            if (l[i] > lmax) lmax = l[i];
        }
        double den = 0.0;
        for (int64_t i = 0; i < n; ++i) den += exp(l[i] - lmax);
        for (int64_t i = 0; i < n; ++i) {
            double p = exp(l[i] - lmax) / den;
            for (int c = 0; c < d; ++c) o[c] += p * bf16_to_double(rows[i][c]);
        }
        lse[h] = lmax + log(den);
    }
    free(l);
}

/*
 * a5, CSA partial.  [V4] "CSA: buscar primer i atendre despres": attention
 * runs over the chosen compressed entries and the local window.  [F] 2.1:
 * the window is the last 128 raw tokens.  Keys: entries[idx[i]] for every
 * idx[i] >= 0, then raw tokens t in [max(0, L-W), L) (R5).
 * entries: [*, d] (the sequence's CSA cache), raw: [L, d] (the sequence's raw
 * latents).  Returns -5 if an index is not a causal entry (>= floor(L/m)).
 */
int oracle_csa_attn(const uint16_t* q, int H, int d, const uint16_t* entries, const int32_t* idx, int k, int m,
                    const uint16_t* raw, int64_t L, int W, double scale, double* O, double* lse) {
    int64_t n_causal = L / m;
    int64_t w0 = L - W > 0 ? L - W : 0;
    int64_t nmax = (int64_t)k + (L - w0);
    const uint16_t** rows = (const uint16_t**)malloc(sizeof(uint16_t*) * (size_t)(nmax > 0 ? nmax : 1));
    int64_t n = 0;
    for (int i = 0; i < k; ++i) {
        if (idx[i] < 0) continue;
        if (idx[i] >= n_causal) { free(rows); return -5; }
        rows[n++] = entries + (int64_t)idx[i] * d;
    }
    for (int64_t t = w0; t < L; ++t) rows[n++] = raw + t * d;
    attend_rows(q, H, d, rows, n, scale, O, lse);
    free(rows);
    return 0;
}

/*
 * a6, HCA partial.  [F] 2.2 and [V4] "HCA: un resum global ...": dense
 * attention over every visible HCA entry, j < floor(L/m') (R5), plus,
 * when W > 0, the raw window [max(0, L-W), L) (used only when HCA is called
 * on its own; the hybrid call passes W = 0 so the window is counted once).
 */
int oracle_hca_attn(const uint16_t* q, int H, int d, const uint16_t* hca, int m_hca, const uint16_t* raw,
                    int64_t L, int W, double scale, double* O, double* lse) {
    int64_t n_vis = L / m_hca;
    int64_t w0 = L - W > 0 ? L - W : 0;
    int64_t nmax = n_vis + (W > 0 ? (L - w0) : 0);
    const uint16_t** rows = (const uint16_t**)malloc(sizeof(uint16_t*) * (size_t)(nmax > 0 ? nmax : 1));
    int64_t n = 0;
    for (int64_t j = 0; j < n_vis; ++j) rows[n++] = hca + j * d;
    if (W > 0)
        for (int64_t t = w0; t < L; ++t) rows[n++] = raw + t * d;
    attend_rows(q, H, d, rows, n, scale, O, lse);
    free(rows);
    return 0;
}

/*
 * a7: log-sum-exp merge of two partials over disjoint key sets (R6):
 *   lse = log(exp(lse1) + exp(lse2)),  O = exp(lse1 - lse) O1 + exp(lse2 - lse) O2.
 * A partial with lse = -inf contributes nothing.
 */
void oracle_lse_merge(const double* O1, const double* lse1, const double* O2, const double* lse2, int H, int d,
                      double* O, double* lse) {
    for (int h = 0; h < H; ++h) {
        double a = lse1[h], b = lse2[h];
        double mx = a > b ? a : b;
        if (mx == -INFINITY) {
            lse[h] = -INFINITY;
            for (int c = 0; c < d; ++c) O[h * d + c] = 0.0;
            continue;
        }
        double l = mx + log(exp(a - mx) + exp(b - mx));
        double wa = exp(a - l), wb = exp(b - l);
        for (int c = 0; c < d; ++c) O[h * d + c] = wa * O1[h * d + c] + wb * O2[h * d + c];
        lse[h] = l;
    }
}

/* ---- f1: 8-bit block-scaled indexer keys --------------------------------- */
/*
 * "Frontier Techniques: NTK RoPE, CSA+HCA, QAT, MTP", section 3 (DeepSeek V4 quantizes the
 * indexer's QK path to a 4-bit block-scaled format) and "Compressed attention . CSA / HCA va hai
 * truc nen", sections 3 and 4 (quantized caches carry block scales; the scale bytes count).  The
 * pages fix neither the element format nor the block, so this is a reading in the same family
 * (MX-style, 8-bit elements): the indexer keys of an entry are cut into blocks of 32 consecutive
 * channels; a block shares one power-of-two scale 2^e, stored as the byte e + 127; its elements
 * are FP8 E4M3 numbers (exponent bias 7, largest 448, subnormal step 2^-9).  e is the smallest
 * integer with amax <= 448 * 2^e (amax = the block's largest magnitude; a zero block takes
 * e = -127), and each element is x / 2^e rounded to the nearest E4M3 value, ties to even.  Only the
 * keys are quantized; the indexer queries stay bf16, and the score is the plain score of the
 * dequantized keys, element = 2^e * E4M3 value.
 */

/* Round |v| <= 448 to the nearest E4M3 value (ties to even). */
static double e4m3_round(double v) {
    double a = fabs(v);
    if (a == 0.0) return v;
    double q;
    if (a < ldexp(1.0, -6)) {               /* subnormal grid: steps of 2^-9 */
        q = rint(a / ldexp(1.0, -9)) * ldexp(1.0, -9);
    } else {
        int y;
        frexp(a, &y);                        /* a in [2^(y-1), 2^y) */
        double step = ldexp(1.0, y - 1 - 3); /* 3 mantissa bits */
        q = rint(a / step) * step;
    }
    return v < 0 ? -q : q;
}

/* The E4M3 bit pattern of a value on the E4M3 grid (|v| <= 448). */
static uint8_t e4m3_bits(double v) {
    uint8_t s = signbit(v) ? 0x80 : 0;
    double a = fabs(v);
    if (a == 0.0) return s;
    if (a < ldexp(1.0, -6)) return (uint8_t)(s | (uint8_t)(a / ldexp(1.0, -9)));
    int y;
    double g = frexp(a, &y);                 /* a = g 2^y, g in [0.5, 1) */
    int E = y - 1 + 7;
    int m = (int)((2.0 * g - 1.0) * 8.0);
    return (uint8_t)(s | (E << 3) | m);
}

static double e4m3_value(uint8_t b) {
    int E = (b >> 3) & 15, m = b & 7;
    double a = E == 0 ? m * ldexp(1.0, -9) : ldexp(1.0 + m / 8.0, E - 7);
    return (b & 0x80) ? -a : a;
}

void oracle_e4m3_round(const double* in, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_bits(e4m3_round(in[i]));
}

void oracle_e4m3_value(const uint8_t* in, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(in[i]);
}

/* Quantize n bf16 key rows [n, d_I] (d_I a multiple of 32) to Kq [n, d_I] E4M3 bytes and
 * scales [n, d_I / 32] biased exponents. */
int oracle_quantize_keys_mx8(const uint16_t* K, int64_t n, int d_I, uint8_t* Kq, uint8_t* scales) {
    if (d_I % 32) return -2;
    int nb = d_I / 32;
    for (int64_t j = 0; j < n; ++j) {
        for (int b = 0; b < nb; ++b) {
            const uint16_t* x = K + j * d_I + 32 * b;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs(bf16_to_double(x[i]));
                if (a > amax) amax = a;
            }
            int e = -127;
            if (amax > 0.0) {
                int y;
                frexp(amax, &y);
                e = y - 9;                                    /* a start near the answer (amax < 2^y) */
                while (amax > ldexp(448.0, e)) ++e;           /* smallest e with amax <= 448 * 2^e */
                while (e > -127 && amax <= ldexp(448.0, e - 1)) --e;
            }
            scales[j * nb + b] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; ++i)
                Kq[j * d_I + 32 * b + i] = e4m3_bits(e4m3_round(ldexp(bf16_to_double(x[i]), -e)));
        }
    }
    return 0;
}

/* a3 with 8-bit keys: s_j = sum_h w_h * relu(qI_h . K_j) with K_j the dequantized key
 * (element 2^e * E4M3 value), everything in double. */
void oracle_index_scores_mx8(const uint16_t* qI, const float* w, int H_I, int d_I, const uint8_t* Kq,
                             const uint8_t* scales, int64_t n_entries, double* s) {
    int nb = d_I / 32;
    for (int64_t j = 0; j < n_entries; ++j) {
        double acc = 0.0;
        for (int h = 0; h < H_I; ++h) {
            double dot = 0.0;
            for (int c = 0; c < d_I; ++c) {
                double k = ldexp(e4m3_value(Kq[j * d_I + c]), (int)scales[j * nb + c / 32] - 127);
                dot += bf16_to_double(qI[h * d_I + c]) * k;
            }
            acc += (double)w[h] * (dot > 0.0 ? dot : 0.0);
        }
        s[j] = acc;
    }
}

/* ---- f3: query / compressed-entry normalization ---------------------------- */
/*
 * "DeepSeek V4 comprimeix el context", section "CSA: buscar primer i atendre despres", last
 * paragraph: the design normalizes the queries and the compressed entries to stabilize the logits.
 * Reading (the page names no formula): RMS normalization with a learned gain, applied to each query
 * head's d-wide vector and to each compressed entry (CSA and HCA) as it is produced:
 *   out[c] = x[c] / sqrt(mean_c' x[c']^2 + eps) * gain[c].
 * rows of d doubles in, rows of d doubles out.
 */
void oracle_rms_norm(const double* x, int64_t rows, int d, const float* gain, double eps, double* out) {
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int c = 0; c < d; ++c) ss += x[r * d + c] * x[r * d + c];
        double inv = 1.0 / sqrt(ss / d + eps);
        for (int c = 0; c < d; ++c) out[r * d + c] = x[r * d + c] * inv * (double)gain[c];
    }
}

/* ---- f4: FP4 compressed entries with block scales --------------------------- */
/*
 * "Compressed attention · CSA / HCA va hai truc nen", section 3 (Giai phap): the V4.1 FP4 KV cache
 * carries block scales and a packing overhead.  Reading R15 (the page gives no format): the same
 * block-scaled family as the 8-bit indexer keys (R11), with 4-bit elements: every stored entry row
 * (CSA and HCA; the raw window tokens stay bf16) is cut into blocks of 32 channels; block scale 2^e
 * with e the smallest integer such that amax <= 6 * 2^e (e >= -127; a zero block takes e = -127),
 * stored as the byte e + 127; elements E2M1 (sign, two exponent bits with bias 1, one mantissa
 * bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), x / 2^e rounded to the nearest magnitude, a tie to
 * the one whose mantissa bit is 0; two elements per byte, the even channel in the low nibble.  The
 * attention uses the dequantized entries (code value * 2^e) as keys and values.
 */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* The 4-bit code of the E2M1 value nearest to v (ties to the even code), magnitudes above 6 to 6;
   bit 3 is the sign (kept for negative values that round to zero). */
static uint8_t e2m1_code(double v) {
    double a = fabs(v);
    int m = 7;
    if (a < 6.0) {
        int i = 0;
        while (!(a < kE2M1[i + 1])) ++i;             /* kE2M1[i] <= a < kE2M1[i + 1] */
        double dl = a - kE2M1[i], dh = kE2M1[i + 1] - a;
        m = dl < dh ? i : dh < dl ? i + 1 : ((i & 1) == 0 ? i : i + 1);
    }
    return (uint8_t)(((v < 0.0 || (v == 0.0 && signbit(v))) ? 8 : 0) | m);
}

static double e2m1_value(uint8_t code) {
    double a = kE2M1[code & 7];
    return (code & 8) ? -a : a;
}

void oracle_e2m1_round(const double* in, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e2m1_code(in[i]);
}

/* bf16 entry rows [n, d] -> packed codes [n, d / 2] and scale bytes [n, d / 32].  Returns -2 if d is
   not a multiple of 32. */
int oracle_quantize_entries_mx4(const uint16_t* E, int64_t n, int d, uint8_t* Eq, uint8_t* scales) {
    if (d % 32) return -2;
    int nb = d / 32;
    for (int64_t j = 0; j < n; ++j) {
        for (int b = 0; b < nb; ++b) {
            const uint16_t* x = E + j * d + 32 * b;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs(bf16_to_double(x[i]));
                if (a > amax) amax = a;
            }
            int e = -127;
            if (amax > 0.0) {
                int y;
                frexp(amax, &y);
                e = y - 3;                                     /* a start near the answer */
                while (amax > ldexp(6.0, e)) ++e;              /* smallest e with amax <= 6 * 2^e */
                while (e > -127 && amax <= ldexp(6.0, e - 1)) --e;
            }
            scales[j * nb + b] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; i += 2) {
                uint8_t lo = e2m1_code(ldexp(bf16_to_double(x[i]), -e));
                uint8_t hi = e2m1_code(ldexp(bf16_to_double(x[i + 1]), -e));
                Eq[j * (d / 2) + 16 * b + i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return 0;
}

/* packed codes + scale bytes -> the dequantized values [n, d] (fp64). */
void oracle_dequantize_entries_mx4(const uint8_t* Eq, const uint8_t* scales, int64_t n, int d, double* out) {
    int nb = d / 32;
    for (int64_t j = 0; j < n; ++j)
        for (int c = 0; c < d; ++c) {
            uint8_t byte = Eq[j * (d / 2) + c / 2];
            uint8_t code = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
            out[j * d + c] = ldexp(e2m1_value(code), (int)scales[j * nb + c / 32] - 127);
        }
}
