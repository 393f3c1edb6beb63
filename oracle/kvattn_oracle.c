/*
 * kvattn_oracle.c -- plain fp64 CPU oracle for single-token decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no source, header, table or helper with the CUDA library.
 *
 * What it computes is the plain definition of softmax attention for one query
 * token, written out with naive loops and three passes (max, sum, weighted sum):
 *
 *   GQA / MQA / MHA  ("Attention variants: MQA, GQA, and MLA", sections
 *   "MQA: one KV head for everyone" and "GQA: interpolating with groups";
 *   "Grouped-Query Attention: Fewer KV Heads, Same Quality", section
 *   "Writing the formula explicitly" and "The Unified View"):
 *       head_i = softmax(q_i . K_j^T / sqrt(d)) V_j,  j = the group of head i.
 *   The pages number heads and groups from 1 and write j = ceil(i * n_kv / n_q);
 *   with 0-based indices that is j = h / (n_q / n_kv) (consecutive groups, the
 *   same order as repeat_interleave).  The caller passes the scale explicitly.
 *
 *   Absorbed MLA  ("Attention variants: MQA, GQA, and MLA", section "MLA: cache
 *   a latent, not the keys and values"): W_UK is folded into the query, so head h
 *   scores  q_lat[h] . c_t + q_rope[h] . r_t  against the cached latent c_t and
 *   the decoupled RoPE key r_t, and its output is the softmax-weighted sum of the
 *   latents c_t (W_UV is applied downstream).  Keys and values are the same
 *   latent vector; the RoPE part enters the score only.
 *
 * Readings where the pages are silent:
 *   - decode attends to every cached position t < seq_lens[b]; no mask;
 *   - lse is the natural log of sum_t exp(s_t) with s_t already scaled;
 *   - an empty sequence (seq_lens[b] == 0) gives out = 0 and lse = -inf;
 *   - inputs arrive as fp64 arrays (the bf16 values are converted exactly by the
 *     caller before the call).
 *
 * Build:  gcc -O2 -fopenmp -shared -fPIC kvattn_oracle.c -o libkvattn_oracle.so -lm
 * The optional -DKVO_MUTANT=n plants one deliberate mistake (used only by the
 * test that proves the pins catch such mistakes); the default build has none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifndef KVO_MUTANT
#define KVO_MUTANT 0
#endif

/* Returns the version of the oracle's interface. */
int kvo_version(void) { return 1; }

/* Returns the planted-mistake id this build carries (0 for the real oracle). */
int kvo_mutant(void) { return KVO_MUTANT; }

/* Index of the KV head that query head h reads: consecutive groups of n_q/n_kv. */
static int kv_head_of(int h, int n_q, int n_kv) {
#if KVO_MUTANT == 1
    (void)n_q;
    return h % n_kv;                  /* planted mistake: strided groups */
#else
    return h / (n_q / n_kv);
#endif
}

/*
 * GQA / MQA / MHA decode.
 *   q    [B, n_q, d]
 *   k, v [B, n_kv, T_max, d]
 *   seq_lens [B]   (positions t < seq_lens[b] are attended; values are clamped to [0, T_max])
 *   out  [B, n_q, d],  lse [B, n_q]
 * Returns 0 on success, -1 on bad arguments, -2 if scratch memory is unavailable.
 */
int kvo_gqa_decode(const double *q, const double *k, const double *v,
                   const int32_t *seq_lens, int B, int n_q, int n_kv, int d,
                   int T_max, double scale, double *out, double *lse) {
    if (B < 0 || n_q <= 0 || n_kv <= 0 || d <= 0 || T_max < 0 || n_q % n_kv != 0)
        return -1;
    int failed = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < n_q; ++h) {
            int T = seq_lens[b];
            if (T < 0) T = 0;
            if (T > T_max) T = T_max;
#if KVO_MUTANT == 6
            if (T > 1) T -= 1;                /* planted mistake: last position dropped */
#endif
            const int j = kv_head_of(h, n_q, n_kv);
            const double *qh = q + ((size_t)b * n_q + h) * d;
            const double *kb = k + ((size_t)b * n_kv + j) * (size_t)T_max * d;
#if KVO_MUTANT == 5
            const double *vb = k + ((size_t)b * n_kv + j) * (size_t)T_max * d; /* planted mistake: values read from K */
#else
            const double *vb = v + ((size_t)b * n_kv + j) * (size_t)T_max * d;
#endif
            double *oh = out + ((size_t)b * n_q + h) * d;
            for (int i = 0; i < d; ++i) oh[i] = 0.0;
            if (T == 0) {
                lse[(size_t)b * n_q + h] = -INFINITY;
                continue;
            }
            double *s = (double *)malloc(sizeof(double) * (size_t)T);
            if (!s) {
#pragma omp atomic write
                failed = 1;
                continue;
            }
            /* scores */
            for (int t = 0; t < T; ++t) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i) acc += qh[i] * kb[(size_t)t * d + i];
#if KVO_MUTANT == 2
                s[t] = acc;                    /* planted mistake: scale dropped */
#else
                s[t] = scale * acc;
#endif
            }
            /* pass 1: max */
            double m = s[0];
            for (int t = 1; t < T; ++t) if (s[t] > m) m = s[t];
            /* pass 2: normaliser */
            double l = 0.0;
            for (int t = 0; t < T; ++t) l += exp(s[t] - m);
            /* pass 3: weighted sum of values */
            for (int t = 0; t < T; ++t) {
                const double w = exp(s[t] - m) / l;
                for (int i = 0; i < d; ++i) oh[i] += w * vb[(size_t)t * d + i];
            }
#if KVO_MUTANT == 3
            lse[(size_t)b * n_q + h] = m + log2(l);   /* planted mistake: base-2 log */
#else
            lse[(size_t)b * n_q + h] = m + log(l);
#endif
            free(s);
        }
    }
    return failed ? -2 : 0;
}

/*
 * Several new tokens per sequence (multi-token decode, e.g. verifying drafted tokens),
 * optionally with a sliding window.
 *   q    [B, L, n_q, d]     the L newest tokens' queries, oldest first
 *   k, v [B, n_kv, T_max, d] the cache, which already holds those L tokens at positions
 *                           seq_lens[b] - L .. seq_lens[b] - 1
 *   out  [B, L, n_q, d],  lse [B, L, n_q]
 * Query i sits at position p = seq_lens[b] - L + i and attends to the cached positions
 * t <= p (the causal mask of "Attention variants: MQA, GQA, and MLA", section
 * "Implementation, twice": a query never sees later tokens) and, when window > 0, only
 * to the last `window` of them, p - window < t (the sliding window named in
 * "Grouped-Query Attention: Fewer KV Heads, Same Quality", section on modern
 * architectures, Mistral 7B).  A query with no visible position (p < 0) gets out = 0,
 * lse = -inf.  Each query is the plain softmax of the single-token routine over its
 * visible positions, in the same three passes.
 */
int kvo_gqa_decode_multi(const double *q, const double *k, const double *v, const int32_t *seq_lens,
                         int B, int L, int n_q, int n_kv, int d, int T_max, double scale, int window,
                         double *out, double *lse) {
    if (B < 0 || L <= 0 || n_q <= 0 || n_kv <= 0 || d <= 0 || T_max < 0 || n_q % n_kv != 0 || window < 0)
        return -1;
    int failed = 0;
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < L; ++i) {
            for (int h = 0; h < n_q; ++h) {
                int T = seq_lens[b];
                if (T < 0) T = 0;
                if (T > T_max) T = T_max;
                const int pos = T - L + i;
#if KVO_MUTANT == 9
                const int hi = pos;                 /* planted mistake: the query's own position hidden */
#else
                const int hi = pos + 1;             /* visible: t < hi */
#endif
#if KVO_MUTANT == 10
                const int lo = window > 0 ? (hi - window - 1 > 0 ? hi - window - 1 : 0) : 0;  /* planted: window + 1 */
#else
                const int lo = window > 0 ? (hi - window > 0 ? hi - window : 0) : 0;
#endif
                const int j = kv_head_of(h, n_q, n_kv);
                const double *qh = q + (((size_t)b * L + i) * n_q + h) * d;
                const double *kb = k + ((size_t)b * n_kv + j) * (size_t)T_max * d;
                const double *vb = v + ((size_t)b * n_kv + j) * (size_t)T_max * d;
                double *oh = out + (((size_t)b * L + i) * n_q + h) * d;
                double *lh = lse + ((size_t)b * L + i) * n_q + h;
                for (int e = 0; e < d; ++e) oh[e] = 0.0;
                if (hi <= lo) {
                    *lh = -INFINITY;
                    continue;
                }
                const int n = hi - lo;
                double *s = (double *)malloc(sizeof(double) * (size_t)n);
                if (!s) {
#pragma omp atomic write
                    failed = 1;
                    continue;
                }
                for (int t = 0; t < n; ++t) {
                    double acc = 0.0;
                    for (int e = 0; e < d; ++e) acc += qh[e] * kb[(size_t)(lo + t) * d + e];
                    s[t] = scale * acc;
                }
                double m = s[0];
                for (int t = 1; t < n; ++t) if (s[t] > m) m = s[t];
                double l = 0.0;
                for (int t = 0; t < n; ++t) l += exp(s[t] - m);
                for (int t = 0; t < n; ++t) {
                    const double w = exp(s[t] - m) / l;
                    for (int e = 0; e < d; ++e) oh[e] += w * vb[(size_t)(lo + t) * d + e];
                }
                *lh = m + log(l);
                free(s);
            }
        }
    }
    return failed ? -2 : 0;
}

/*
 * Absorbed MLA decode.
 *   q_lat  [B, H, d_c]      query already multiplied by W_UK (latent space)
 *   q_rope [B, H, d_r]      rotated decoupled-RoPE query part
 *   lat    [B, T_max, d_c]  cached latents c_t (one per token, shared by all heads)
 *   rope   [B, T_max, d_r]  cached rotated RoPE keys r_t
 *   out    [B, H, d_c],  lse [B, H]
 * d_r may be 0 (then q_rope / rope are not read).
 */
int kvo_mla_decode(const double *q_lat, const double *q_rope, const double *lat,
                   const double *rope, const int32_t *seq_lens, int B, int H,
                   int d_c, int d_r, int T_max, double scale, double *out,
                   double *lse) {
    if (B < 0 || H <= 0 || d_c <= 0 || d_r < 0 || T_max < 0) return -1;
    int failed = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            int T = seq_lens[b];
            if (T < 0) T = 0;
            if (T > T_max) T = T_max;
            const double *ql = q_lat + ((size_t)b * H + h) * d_c;
            const double *qr = d_r ? q_rope + ((size_t)b * H + h) * d_r : 0;
            const double *cb = lat + (size_t)b * T_max * d_c;
            const double *rb = d_r ? rope + (size_t)b * T_max * d_r : 0;
            double *oh = out + ((size_t)b * H + h) * d_c;
            for (int i = 0; i < d_c; ++i) oh[i] = 0.0;
            if (T == 0) {
                lse[(size_t)b * H + h] = -INFINITY;
                continue;
            }
            double *s = (double *)malloc(sizeof(double) * (size_t)T);
            if (!s) {
#pragma omp atomic write
                failed = 1;
                continue;
            }
            for (int t = 0; t < T; ++t) {
                double acc = 0.0;
                for (int i = 0; i < d_c; ++i) acc += ql[i] * cb[(size_t)t * d_c + i];
#if KVO_MUTANT != 4
                for (int i = 0; i < d_r; ++i) acc += qr[i] * rb[(size_t)t * d_r + i];
#endif                                         /* mutant 4: RoPE term dropped */
                s[t] = scale * acc;
            }
            double m = s[0];
            for (int t = 1; t < T; ++t) if (s[t] > m) m = s[t];
            double l = 0.0;
            for (int t = 0; t < T; ++t) l += exp(s[t] - m);
            for (int t = 0; t < T; ++t) {
                const double w = exp(s[t] - m) / l;
                for (int i = 0; i < d_c; ++i) oh[i] += w * cb[(size_t)t * d_c + i];
            }
            lse[(size_t)b * H + h] = m + log(l);
            free(s);
        }
    }
    return failed ? -2 : 0;
}

/*
 * Rotary position embedding of vectors (the new token's query and key before they
 * meet the cache).  The pages name RoPE -- applied to queries and keys upstream of the
 * attention ("Attention variants: MQA, GQA, and MLA", section "MLA: cache a latent, not
 * the keys and values": the decoupled rotary key cached alongside the latent) -- but do
 * not write its formula, so this is the textbook rotation of feature pairs: for a
 * vector x of even length d at position p, pair i (i = 0 .. d/2 - 1) turns by the angle
 *     theta_i = p * base^(-2i / d)
 *     x'_a = x_a cos(theta_i) - x_b sin(theta_i)
 *     x'_b = x_a sin(theta_i) + x_b cos(theta_i)
 * with (a, b) = (2i, 2i + 1) for interleaved pairs and (i, i + d/2) for split halves.
 * n vectors of length d in x (row r at position pos[r]); out may alias x.
 */
int kvo_rope(const double *x, int n, int d, const int32_t *pos, double base, int interleaved,
             double *out) {
    if (d <= 0 || (d & 1) || base <= 0.0) return 1;
    const int half = d / 2;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < n; ++r) {
        const double *xr = x + (size_t)r * d;
        double *yr = out + (size_t)r * d;
        for (int i = 0; i < half; ++i) {
#if KVO_MUTANT == 8
            const double freq = pow(base, -(double)i / (double)d);   /* planted mistake: exponent i/d */
#else
            const double freq = pow(base, -2.0 * (double)i / (double)d);
#endif
            const double theta = (double)pos[r] * freq;
            const int a = interleaved ? 2 * i : i;
            const int b = interleaved ? 2 * i + 1 : i + half;
            const double xa = xr[a], xb = xr[b];
#if KVO_MUTANT == 7
            yr[a] = xa * cos(theta) + xb * sin(theta);                 /* planted mistake: sign */
            yr[b] = -xa * sin(theta) + xb * cos(theta);
#else
            yr[a] = xa * cos(theta) - xb * sin(theta);
            yr[b] = xa * sin(theta) + xb * cos(theta);
#endif
        }
    }
    return 0;
}

/*
 * Quantised (fp8) KV cache.  The pages list quantised caches among what the libraries
 * build around the attention module ("Attention variants: MQA, GQA, and MLA", section
 * "Against the real libraries"); stored in 8 bits, the cache a decode step reads halves.
 * They fix no format.  Reading: the 8-bit floating-point format
 * E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
 * holds the subnormals m * 2^-9; no infinities; S.1111.111 is the only NaN, so the
 * largest finite magnitude is 1.75 * 2^8 = 448), with one float scale per cache tensor:
 * the cached value is  code_value * scale.
 */

/* Value of one E4M3 code, from the format's definition. */
double kvo_e4m3_value(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
#if KVO_MUTANT == 11
    if (e == 0) mag = ldexp(1.0 + m / 8.0, -6);       /* planted mistake: no subnormals */
#else
    if (e == 0) mag = ldexp((double)m, -9);           /* subnormal: m/8 * 2^(1-7) */
#endif
#if KVO_MUTANT == 12
    else mag = ldexp(1.0 + m / 8.0, e - 8);           /* planted mistake: bias 8 */
#else
    else mag = ldexp(1.0 + m / 8.0, e - 7);
#endif
    return sign ? -mag : mag;
}

/* out[i] = value(in[i]) * scale (the dequantised cache), n codes. */
int kvo_e4m3_dequant(const uint8_t *in, long long n, double scale, double *out) {
    if (n < 0) return 1;
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; ++i) out[i] = kvo_e4m3_value(in[i]) * scale;
    return 0;
}

/* Nearest E4M3 code to the float x, ties to the even code, magnitudes past the largest
 * finite value saturated to +-448; NaN gives the NaN code.  (Quantising a value for the
 * cache: the caller has already divided it by the tensor's scale in float.) */
uint8_t kvo_e4m3_code(float x) {
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: spacing 2^-9; m = 8 is the smallest normal, code 0x08 */
        const double m = rint(a / ldexp(1.0, -9));   /* round half to even (default mode) */
        return sign | (uint8_t)m;
    }
    int e = (int)floor(log2(a));
    if (ldexp(1.0, e) > a) --e;                        /* guard log2 rounding */
    if (ldexp(1.0, e + 1) <= a) ++e;
#if KVO_MUTANT == 13
    double n = floor(a / ldexp(1.0, e - 3) + 0.5);     /* planted mistake: ties away from zero */
#else
    double n = rint(a / ldexp(1.0, e - 3));            /* 8 .. 16 steps of 2^(e-3) */
#endif
    if (n >= 16.0) { n = 8.0; ++e; }
    if (e > 8 || (e == 8 && n > 14.0)) return sign | 0x7E;
    return sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8));
}

/* codes[i] = kvo_e4m3_code(x[i] / scale), the division in float. */
int kvo_e4m3_quant(const float *x, long long n, float scale, uint8_t *codes) {
    if (n < 0 || !(scale > 0.0f)) return 1;
    for (long long i = 0; i < n; ++i) {
        const float y = x[i] / scale;
        codes[i] = kvo_e4m3_code(y);
    }
    return 0;
}

/* Number of OpenMP threads a parallel region of this library uses. */
int kvo_num_threads(void) {
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
