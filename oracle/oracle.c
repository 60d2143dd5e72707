/*
 * oracle.c -- CPU oracle of the routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py load this library.  It shares no
 * code, header, table or helper with the CUDA path in expert_ffn_router_b200/.
 *
 * What it computes (Colibri pages; a "[reading]" marks a step the pages leave
 * open, settled by the plainest reading the rest supports):
 *   a0  per-token int8 activation quantisation: s_x = max|x| / 127, codes by
 *       round-half-even of x / s_x, clamped to +-127; an all-zero token gets
 *       s_x = 0 and zero codes.                        [reading: agentlenshq
 *       summary, "Integer-Dot Kernels" / "Quantization"; scale rule as given]
 *   a1  DeepSeek-V3-style router: logits = W_r x on the unquantised x, sigmoid
 *       scores, selection on score + bias, top-k (ties to the lower index),
 *       weights = the selected unbiased scores renormalised to sum 1 and scaled
 *       by routed_scale.         [takumi3488 article, teacher-forcing section:
 *       "DeepSeek-V3 style router"; top-8 of 256 and top-2 of 8 from the coli
 *       info logs; no group-limited selection -- reading]
 *   a1' TOPK/TOPP truncation (opt-in, p in (0, 1)): keep the smallest prefix of
 *       the selected slots, in selection order, whose normalised scores sum to
 *       at least p; the dropped slots select no expert; the kept weights are
 *       renormalised over the kept scores.   [reading: agentlenshq benchmark
 *       table, the `--topp 0.7` rows, and the TOPK / TOPP options of the
 *       takumi3488 run logs; the pages give no definition]
 *   a3  gate/up: int32 dot products of packed int4 / int2 codes with the int8
 *       activation codes; dequantised by (per-row scale * s_x); h = SiLU(g)*u.
 *       [agentlenshq summary: packed int4/int2 with per-row scales and
 *       dequantisation on use; SwiGLU expert -- reading]
 *   a4  h requantised per (token, expert) like a0; down-projection int32 dot;
 *       dequantised by (per-row scale * s_h).
 *   a5/a6 combine: out = sum_j w_j * y_{e_j} + y_shared (shared weight 1.0).
 *       [agentlenshq "Memory split": shared experts are part of the resident
 *       dense part; the combine weight 1.0 is a reading]
 *
 * Precision.  Every float step whose result decides an integer (the a0 and a4
 * quantiser codes, the top-k selection) is done in float32 in the order
 * written above, i.e. in the kernel's precision; products of scales are formed
 * first (s_row * s_x), then multiplied into the accumulator.  Every other float
 * value (router logits before rounding, router weights, dequantised down
 * outputs, the combine, RMSNorm) is computed in float64.  Integer dot products
 * are accumulated in int64 and checked to fit int32.  Build with
 * -ffp-contract=off and without -ffast-math so the float32 steps round exactly
 * as written.
 *
 * Packing [reading]: codes are two's complement, low bits first within a byte:
 * int4 byte = c0 | c1 << 4; int2 byte = c0 | c1 << 2 | c2 << 4 | c3 << 6;
 * int8 experts (the "expert@8-bit" banner of the takumi3488 run log): one
 * code per byte, [-128, 127].
 * Expert blob [reading of "adjacent matrices stored together", remio.ai
 * analysis, the dedupe paragraph]: [gate f x d | up f x d | down d x f], each
 * matrix row-major by output row; scales [gate f | up f | down d].
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_EOVERFLOW (-2)
#define ORACLE_ENULL (-3)

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Code i of a packed row: wbits in {2, 4, 8}, two's complement, low bits first
 * (int8: one code per byte). */
static inline int code_at(const uint8_t* row, int wbits, int64_t i) {
    int per_byte = 8 / wbits;
    int shift = (int)(i % per_byte) * wbits;
    int v = (row[i / per_byte] >> shift) & ((1 << wbits) - 1);
    return v >= (1 << (wbits - 1)) ? v - (1 << wbits) : v;
}

int oracle_unpack(int wbits, const uint8_t* src, int64_t n, int8_t* dst) {
    if ((wbits != 2 && wbits != 4 && wbits != 8) || !src || !dst || n < 0) return ORACLE_EINVAL;
    for (int64_t i = 0; i < n; ++i) dst[i] = (int8_t)code_at(src, wbits, i);
    return ORACLE_OK;
}

int oracle_pack(int wbits, const int8_t* src, int64_t n, uint8_t* dst) {
    if ((wbits != 2 && wbits != 4 && wbits != 8) || !src || !dst || n < 0) return ORACLE_EINVAL;
    int per_byte = 8 / wbits;
    if (n % per_byte) return ORACLE_EINVAL;
    int lo = -(1 << (wbits - 1)), hi = (1 << (wbits - 1)) - 1;
    memset(dst, 0, (size_t)(n / per_byte));
    for (int64_t i = 0; i < n; ++i) {
        if (src[i] < lo || src[i] > hi) return ORACLE_EINVAL;
        int v = src[i] & ((1 << wbits) - 1);
        dst[i / per_byte] |= (uint8_t)(v << ((i % per_byte) * wbits));
    }
    return ORACLE_OK;
}

/* Round half to even of a float32 value already known to be finite. */
static inline float rne_f32(float v) { return nearbyintf(v); }

/* a0: quantise one row of n floats to int8 codes; returns the scale. */
static float quantize_row(const float* x, int n, int8_t* q) {
    float amax = 0.0f;
    for (int c = 0; c < n; ++c) {
        float a = fabsf(x[c]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        memset(q, 0, (size_t)n);
        return 0.0f;
    }
    float s = amax / 127.0f;
    for (int c = 0; c < n; ++c) {
        float v = rne_f32(x[c] / s);
        if (v > 127.0f) v = 127.0f;
        if (v < -127.0f) v = -127.0f;
        q[c] = (int8_t)v;
    }
    return s;
}

int oracle_quantize(const float* x, int T, int d, int8_t* q, float* s) {
    if (!x || !q || !s || T < 0 || d <= 0) return ORACLE_EINVAL;
    for (int t = 0; t < T; ++t) s[t] = quantize_row(x + (int64_t)t * d, d, q + (int64_t)t * d);
    return ORACLE_OK;
}

/* a1 (+ a1'): router.  x fp32 [T][d], wr fp32 [E][d], bias fp32 [E].
 * Outputs idx [T][k] (slot order = selection score descending, ties to the
 * lower expert index), w fp64 [T][k]; optional logits/scores/sel fp32 [T][E].
 * topp in (0, 1) truncates (a1'): the decision, an integer, is taken in
 * float32 in slot order -- S = the float sum of the k selected scores, thr =
 * float(topp * S); slot j is kept iff j == 0 or the float sum of the scores of
 * slots 0..j-1 is below thr -- and a dropped slot gets idx -1 and weight 0;
 * the kept weights are the kept scores over their (float64) sum, times
 * routed_scale.  Any other topp: no truncation. */
int oracle_route_p(const float* x, int T, int d, int E, int k, const float* wr, const float* bias,
                   double routed_scale, float topp, int32_t* idx, double* w, float* logits_out,
                   float* s_out, float* sel_out) {
    if (!x || !wr || !bias || !idx || !w || T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E)
        return ORACLE_EINVAL;
    float* s = (float*)malloc(sizeof(float) * (size_t)E);
    float* sel = (float*)malloc(sizeof(float) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    if (!s || !sel || !taken) { free(s); free(sel); free(taken); return ORACLE_EINVAL; }
    for (int t = 0; t < T; ++t) {
        const float* xt = x + (int64_t)t * d;
        for (int e = 0; e < E; ++e) {
            const float* we = wr + (int64_t)e * d;
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += (double)we[c] * (double)xt[c];
            float logit = (float)acc;
            s[e] = 1.0f / (1.0f + expf(-logit));
            sel[e] = s[e] + bias[e];
            taken[e] = 0;
            if (logits_out) logits_out[(int64_t)t * E + e] = logit;
            if (s_out) s_out[(int64_t)t * E + e] = s[e];
            if (sel_out) sel_out[(int64_t)t * E + e] = sel[e];
        }
        int32_t* it = idx + (int64_t)t * k;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || sel[e] > sel[best]) best = e; /* strict: ties keep the lower index */
            }
            taken[best] = 1;
            it[j] = best;
        }
        int m = k; /* slots kept */
        if (topp > 0.0f && topp < 1.0f) {
            float S = 0.0f;
            for (int j = 0; j < k; ++j) S = S + s[it[j]];
            const float thr = topp * S;
            float before = 0.0f; /* float sum of the scores of the slots before j */
            for (int j = 0; j < k; ++j) {
                if (j > 0 && !(before < thr)) { m = j; break; }
                before = before + s[it[j]];
            }
        }
        double sum = 0.0;
        for (int j = 0; j < m; ++j) sum += (double)s[it[j]];
        for (int j = 0; j < k; ++j) {
            if (j < m) {
                w[(int64_t)t * k + j] = (double)s[it[j]] / sum * routed_scale;
            } else {
                it[j] = -1;
                w[(int64_t)t * k + j] = 0.0;
            }
        }
    }
    free(s); free(sel); free(taken);
    return ORACLE_OK;
}

int oracle_route(const float* x, int T, int d, int E, int k, const float* wr, const float* bias,
                 double routed_scale, int32_t* idx, double* w, float* logits_out, float* s_out,
                 float* sel_out) {
    return oracle_route_p(x, T, d, E, k, wr, bias, routed_scale, 0.0f, idx, w, logits_out, s_out, sel_out);
}

/* int dot of one packed row (n codes) with n int8 activation codes, in int64. */
static int64_t dot_row(const uint8_t* row, int wbits, const int8_t* a, int n) {
    int64_t acc = 0;
    for (int c = 0; c < n; ++c) acc += (int64_t)code_at(row, wbits, c) * (int64_t)a[c];
    return acc;
}

static int fits_i32(int64_t v) { return v >= INT32_MIN && v <= INT32_MAX; }

/* a4 (teacher-forced entry): down projection of given h codes.
 * hq int8 [T][f], sh fp32 [T] -> acc_d int32 [T][d] (nullable), y fp64 [T][d]. */
int oracle_down(int d, int f, int wbits, const uint8_t* blob, const float* sc, const int8_t* hq,
                const float* sh, int T, int32_t* acc_d, double* y) {
    if ((wbits != 2 && wbits != 4 && wbits != 8) || !blob || !sc || !hq || !sh || !y || d <= 0 || f <= 0 || T < 0)
        return ORACLE_EINVAL;
    const int64_t row_gu = (int64_t)d * wbits / 8, row_dn = (int64_t)f * wbits / 8;
    const uint8_t* wd = blob + 2 * (int64_t)f * row_gu;
    const float* sd = sc + 2 * (int64_t)f;
    int bad = 0;
    for (int t = 0; t < T; ++t) {
#pragma omp parallel for schedule(static) reduction(| : bad)
        for (int r = 0; r < d; ++r) {
            int64_t D = dot_row(wd + (int64_t)r * row_dn, wbits, hq + (int64_t)t * f, f);
            if (!fits_i32(D)) bad = 1;
            if (acc_d) acc_d[(int64_t)t * d + r] = (int32_t)D;
            y[(int64_t)t * d + r] = (double)D * (double)sd[r] * (double)sh[t];
        }
    }
    return bad ? ORACLE_EOVERFLOW : ORACLE_OK;
}

/* a3 + a4 for one expert over T tokens.
 * xq int8 [T][d], sx fp32 [T].  Outputs (each nullable except y):
 * acc_gu int32 [T][2f] (gate rows then up rows), h fp32 [T][f], hq int8 [T][f],
 * sh fp32 [T], acc_d int32 [T][d], y fp64 [T][d]. */
int oracle_expert(int d, int f, int wbits, const uint8_t* blob, const float* sc, const int8_t* xq,
                  const float* sx, int T, int32_t* acc_gu, float* h_out, int8_t* hq_out,
                  float* sh_out, int32_t* acc_d, double* y) {
    if ((wbits != 2 && wbits != 4 && wbits != 8) || !blob || !sc || !xq || !sx || !y || d <= 0 || f <= 0 || T < 0)
        return ORACLE_EINVAL;
    const int64_t row_gu = (int64_t)d * wbits / 8;
    const uint8_t* wg = blob;
    const uint8_t* wu = blob + (int64_t)f * row_gu;
    const float* sg = sc;
    const float* su = sc + f;
    float* h = (float*)malloc(sizeof(float) * (size_t)f);
    int8_t* hq = (int8_t*)malloc((size_t)f);
    if (!h || !hq) { free(h); free(hq); return ORACLE_EINVAL; }
    int bad = 0;
    for (int t = 0; t < T; ++t) {
        const int8_t* xt = xq + (int64_t)t * d;
#pragma omp parallel for schedule(static) reduction(| : bad)
        for (int r = 0; r < f; ++r) {
            int64_t G = dot_row(wg + (int64_t)r * row_gu, wbits, xt, d);
            int64_t U = dot_row(wu + (int64_t)r * row_gu, wbits, xt, d);
            if (!fits_i32(G) || !fits_i32(U)) bad = 1;
            if (acc_gu) {
                acc_gu[(int64_t)t * 2 * f + r] = (int32_t)G;
                acc_gu[(int64_t)t * 2 * f + f + r] = (int32_t)U;
            }
            float g = (float)G * (sg[r] * sx[t]);
            float u = (float)U * (su[r] * sx[t]);
            h[r] = g / (1.0f + expf(-g)) * u;
        }
        float s_h = quantize_row(h, f, hq);
        if (h_out) memcpy(h_out + (int64_t)t * f, h, sizeof(float) * (size_t)f);
        if (hq_out) memcpy(hq_out + (int64_t)t * f, hq, (size_t)f);
        if (sh_out) sh_out[t] = s_h;
        int rc = oracle_down(d, f, wbits, blob, sc, hq, &s_h, 1, acc_d ? acc_d + (int64_t)t * d : NULL,
                             y + (int64_t)t * d);
        if (rc == ORACLE_EOVERFLOW) bad = 1;
        else if (rc) { free(h); free(hq); return rc; }
    }
    free(h); free(hq);
    return bad ? ORACLE_EOVERFLOW : ORACLE_OK;
}

/* Full layer.  blobs / scales: tables of n_experts + has_shared pointers
 * (entry n_experts = shared expert); an entry may be NULL if no token selects
 * that expert.  x fp32 [T][d].  Outputs: out fp64 [T][d], idx [T][k], w fp64
 * [T][k]; xq/sx (nullable) the quantised input.  topp as in oracle_route_p
 * (a dropped slot contributes nothing). */
int oracle_layer_p(int d, int f, int E, int k, int has_shared, int wbits, double routed_scale, float topp,
                   const uint8_t* const* blobs, const float* const* scales, const float* wr,
                   const float* bias, const float* x, int T, double* out, int32_t* idx, double* w,
                   int8_t* xq_out, float* sx_out) {
    if (!blobs || !scales || !wr || !bias || !x || !out || !idx || !w || T < 0) return ORACLE_EINVAL;
    int8_t* xq = (int8_t*)malloc((size_t)T * (size_t)d + 1);
    float* sx = (float*)malloc(sizeof(float) * (size_t)T + 1);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    if (!xq || !sx || !y) { free(xq); free(sx); free(y); return ORACLE_EINVAL; }
    int rc = oracle_quantize(x, T, d, xq, sx);
    if (!rc) rc = oracle_route_p(x, T, d, E, k, wr, bias, routed_scale, topp, idx, w, NULL, NULL, NULL);
    for (int t = 0; !rc && t < T; ++t) {
        double* o = out + (int64_t)t * d;
        for (int r = 0; r < d; ++r) o[r] = 0.0;
        for (int j = 0; j <= k && !rc; ++j) {
            int e;
            double wt;
            if (j < k) { e = idx[(int64_t)t * k + j]; wt = w[(int64_t)t * k + j]; }
            else if (has_shared) { e = E; wt = 1.0; }
            else break;
            if (e < 0) continue; /* a slot dropped by the truncation */
            if (!blobs[e] || !scales[e]) { rc = ORACLE_ENULL; break; }
            rc = oracle_expert(d, f, wbits, blobs[e], scales[e], xq + (int64_t)t * d, sx + t, 1,
                               NULL, NULL, NULL, NULL, NULL, y);
            for (int r = 0; !rc && r < d; ++r) o[r] += wt * y[r];
        }
    }
    if (!rc && xq_out) memcpy(xq_out, xq, (size_t)T * (size_t)d);
    if (!rc && sx_out) memcpy(sx_out, sx, sizeof(float) * (size_t)T);
    free(xq); free(sx); free(y);
    return rc;
}

int oracle_layer(int d, int f, int E, int k, int has_shared, int wbits, double routed_scale,
                 const uint8_t* const* blobs, const float* const* scales, const float* wr,
                 const float* bias, const float* x, int T, double* out, int32_t* idx, double* w,
                 int8_t* xq_out, float* sx_out) {
    return oracle_layer_p(d, f, E, k, has_shared, wbits, routed_scale, 0.0f, blobs, scales, wr, bias, x, T,
                          out, idx, w, xq_out, sx_out);
}

/* Parameter-free RMSNorm of the residual stream (stacked workloads; reading):
 * x_in = x / sqrt(mean(x^2) + eps), computed in fp64, rounded to fp32. */
int oracle_rmsnorm(const double* x, int T, int d, double eps, float* x_in) {
    if (!x || !x_in || T < 0 || d <= 0) return ORACLE_EINVAL;
    for (int t = 0; t < T; ++t) {
        const double* xt = x + (int64_t)t * d;
        double ss = 0.0;
        for (int c = 0; c < d; ++c) ss += xt[c] * xt[c];
        double r = 1.0 / sqrt(ss / d + eps);
        for (int c = 0; c < d; ++c) x_in[(int64_t)t * d + c] = (float)(xt[c] * r);
    }
    return ORACLE_OK;
}
