/*
 * oracle.c -- plain, slow, single-threaded CPU reference of the MoGE FFN layer
 * forward and backward passes, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: it is used by the tests, by the package's smoke check and by the
 * timed CPU baseline of the benchmark. It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Sources (web pages on Huawei's Pangu Pro MoE; the method is stated in prose
 * only, the formulas below restate it):
 *  [A] "Huawei releases Pangu Pro MoE: the first 72B sparse language model,
 *      designed for Ascend NPUs" (techwalker.com), section 1 "Innovative
 *      architecture: the design of the mixture of grouped experts" --
 *      N experts split evenly into M groups of N/M; per token K' = K/M experts
 *      are chosen inside EVERY group; the scores are a GLOBAL softmax over all
 *      N experts, taken BEFORE the in-group top-K'; the imbalance score is the
 *      load gap between the busiest and the idlest device (group) in a batch.
 *  [B] same page, section 2 "Hardware co-design" -- 64 routed experts plus 4
 *      shared experts, hidden size 5120.
 *  [C] reportify.cn concept page "Mixture of grouped experts", bullet
 *      "technical innovation details" -- each group does its own top-K
 *      routing, the inter-group load difference is zero.
 *  [D] mokono.cn news page, "three breakthroughs of MoGE", item 1 -- 64
 *      routed experts in 8 groups, 1 active per group, 4 shared experts kept
 *      for general work.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - the chosen experts' weights are their global-softmax probabilities, not
 *    renormalised;
 *  - shared experts are always on and enter with weight 1;
 *  - an expert is a SwiGLU FFN: W_down (silu(W_gate x) * (W_up x)),
 *    silu(z) = z / (1 + e^-z), no biases;
 *  - group g holds the contiguous experts [g*N/M, (g+1)*N/M);
 *  - inside a group the K' picks are taken in descending score order, equal
 *    scores going to the lower expert index; the selection compares the
 *    scores rounded to fp32, the precision the GPU path decides in;
 *  - the imbalance score is (max_g L_g - min_g L_g) / (T K), L_g the number
 *    of (token, expert) assignments that land in group g;
 *  - within one expert's block of permuted rows, tokens keep ascending order.
 *
 * Layouts are row-major: x [T][d]; w_router [N][d]; w_gate, w_up [E][I][d];
 * w_down [E][d][I] (E = N routed or S shared). Weights are fp32 (dtype 0) or
 * bf16 bit patterns (dtype 1); every element is widened to double exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1

static double bf16_bits_to_double(uint16_t h) {
    uint32_t b = (uint32_t)h << 16;
    float f;
    memcpy(&f, &b, 4);
    return (double)f;
}

/* row of a weight matrix widened to double */
static void load_row(const void *base, int dtype, size_t first, int n, double *out) {
    if (dtype == OR_F32) {
        const float *p = (const float *)base + first;
        for (int j = 0; j < n; ++j) out[j] = (double)p[j];
    } else {
        const uint16_t *p = (const uint16_t *)base + first;
        for (int j = 0; j < n; ++j) out[j] = bf16_bits_to_double(p[j]);
    }
}

static double dot(const double *a, const double *b, int n) {
    double s = 0.0;
    for (int j = 0; j < n; ++j) s += a[j] * b[j];
    return s;
}

/* ---------------------------------------------------------------------------
 * Router scores [A]: logits l_e = x . w_router[e] (+ bias_e), then ONE softmax
 * over all N experts (max subtracted for range only).
 * x: [T][d] double; p_out: [T][N] double.
 */
int oracle_router_probs(const double *x, const void *w_router, const float *bias, int dtype,
                        int T, int d, int N, double *p_out) {
    if (T < 0 || d <= 0 || N <= 0) return 1;
    double *w = (double *)malloc(sizeof(double) * (size_t)d);
    double *l = (double *)malloc(sizeof(double) * (size_t)N);
    if (!w || !l) { free(w); free(l); return 2; }
    for (int t = 0; t < T; ++t) {
        const double *xt = x + (size_t)t * d;
        for (int e = 0; e < N; ++e) {
            load_row(w_router, dtype, (size_t)e * d, d, w);
            l[e] = dot(xt, w, d) + (bias ? (double)bias[e] : 0.0);
        }
        double m = l[0];
        for (int e = 1; e < N; ++e) if (l[e] > m) m = l[e];
        double z = 0.0;
        for (int e = 0; e < N; ++e) z += exp(l[e] - m);
        for (int e = 0; e < N; ++e) p_out[(size_t)t * N + e] = exp(l[e] - m) / z;
    }
    free(w);
    free(l);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Group-balanced selection [A][C] on given scores p [T][N]: for every group g,
 * the Kp experts of [g*G, (g+1)*G) with the largest score (G = N/M).
 * idx/w: [T][M*Kp], group-major, picks inside a group in descending order.
 * margin[t]: min over groups of p(Kp-th pick) - p(best unpicked), in fp64;
 * +inf when a group has no unpicked expert.
 */
int oracle_select_grouped(const double *p, int T, int N, int M, int Kp,
                          int32_t *idx, double *w, double *margin) {
    if (M <= 0 || N % M != 0 || Kp < 1 || Kp > N / M) return 1;
    int G = N / M, K = M * Kp;
    unsigned char *taken = (unsigned char *)malloc((size_t)N);
    if (!taken) return 2;
    for (int t = 0; t < T; ++t) {
        const double *pt = p + (size_t)t * N;
        memset(taken, 0, (size_t)N);
        double mg = INFINITY;
        for (int g = 0; g < M; ++g) {
            double last = 0.0;
            for (int j = 0; j < Kp; ++j) {
                int best = -1;
                float bv = 0.0f;
                for (int e = g * G; e < (g + 1) * G; ++e) {
                    if (taken[e]) continue;
                    float v = (float)pt[e];
                    if (best < 0 || v > bv) { best = e; bv = v; }  /* ties: lower index stays */
                }
                taken[best] = 1;
                idx[(size_t)t * K + g * Kp + j] = best;
                w[(size_t)t * K + g * Kp + j] = pt[best];
                last = pt[best];
            }
            double next = -INFINITY;
            for (int e = g * G; e < (g + 1) * G; ++e)
                if (!taken[e] && pt[e] > next) next = pt[e];
            if (next > -INFINITY && last - next < mg) mg = last - next;
        }
        if (margin) margin[t] = mg;
    }
    free(taken);
    return 0;
}

/* Conventional global top-K [A] (the routing MoGE replaces): the K largest
 * scores over all N experts, same ordering and tie rule. */
int oracle_select_global(const double *p, int T, int N, int K, int32_t *idx) {
    if (K < 1 || K > N) return 1;
    unsigned char *taken = (unsigned char *)malloc((size_t)N);
    if (!taken) return 2;
    for (int t = 0; t < T; ++t) {
        const double *pt = p + (size_t)t * N;
        memset(taken, 0, (size_t)N);
        for (int j = 0; j < K; ++j) {
            int best = -1;
            float bv = 0.0f;
            for (int e = 0; e < N; ++e) {
                if (taken[e]) continue;
                float v = (float)pt[e];
                if (best < 0 || v > bv) { best = e; bv = v; }
            }
            taken[best] = 1;
            idx[(size_t)t * K + j] = best;
        }
    }
    free(taken);
    return 0;
}

/* Routing of a whole batch [A]: scores then group-balanced selection. */
int oracle_route(const double *x, const void *w_router, const float *bias, int dtype,
                 int T, int d, int N, int M, int Kp,
                 int32_t *idx, double *w, double *margin) {
    double *p = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * N);
    if (!p) return 2;
    int rc = oracle_router_probs(x, w_router, bias, dtype, T, d, N, p);
    if (rc == 0) rc = oracle_select_grouped(p, T, N, M, Kp, idx, w, margin);
    free(p);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Imbalance score [A]: loads L_g = number of assignments in group g (experts
 * [g*N/M, (g+1)*N/M)); loads_out[M] receives them; returns (max - min)/(T K).
 */
double oracle_imbalance(const int32_t *idx, int T, int K, int N, int M, int64_t *loads_out) {
    int G = N / M;
    int64_t *L = (int64_t *)calloc((size_t)M, sizeof(int64_t));
    if (!L) return NAN;
    for (size_t a = 0; a < (size_t)T * K; ++a) L[idx[a] / G] += 1;
    int64_t mx = L[0], mn = L[0];
    for (int g = 1; g < M; ++g) { if (L[g] > mx) mx = L[g]; if (L[g] < mn) mn = L[g]; }
    if (loads_out) memcpy(loads_out, L, sizeof(int64_t) * (size_t)M);
    free(L);
    return (T > 0 && K > 0) ? (double)(mx - mn) / ((double)T * K) : 0.0;
}

/* ---------------------------------------------------------------------------
 * Expert-major dispatch, written from its definition: counts[e] = number of
 * assignments to e; offsets = exclusive prefix sum (offsets[N] = T K); the
 * rows of expert e are offsets[e] .. offsets[e+1]-1, holding its tokens in
 * ascending token order; perm_src[row] = token, perm_dst[t][k] = row.
 */
int oracle_dispatch(const int32_t *idx, int T, int K, int N,
                    int32_t *counts, int32_t *offsets, int32_t *perm_src, int32_t *perm_dst) {
    for (int e = 0; e < N; ++e) counts[e] = 0;
    for (size_t a = 0; a < (size_t)T * K; ++a) {
        if (idx[a] < 0 || idx[a] >= N) return 1;
        counts[idx[a]] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < N; ++e) offsets[e + 1] = offsets[e] + counts[e];
    for (int e = 0; e < N; ++e) {
        int32_t row = offsets[e];
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k)
                if (idx[(size_t)t * K + k] == e) {
                    perm_src[row] = t;
                    perm_dst[(size_t)t * K + k] = row;
                    ++row;
                }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * One expert on one token: y = W_down (silu(W_gate x) * (W_up x)).
 * wg, wu point at the expert's [I][d] matrices, wd at its [d][I] matrix.
 */
int oracle_expert_ffn(const double *x, const void *wg, const void *wu, const void *wd,
                      int dtype, int d, int I, double *y) {
    double *w = (double *)malloc(sizeof(double) * (size_t)(d > I ? d : I));
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    if (!w || !h) { free(w); free(h); return 2; }
    for (int i = 0; i < I; ++i) {
        load_row(wg, dtype, (size_t)i * d, d, w);
        double g = dot(x, w, d);
        load_row(wu, dtype, (size_t)i * d, d, w);
        double u = dot(x, w, d);
        h[i] = (g / (1.0 + exp(-g))) * u;
    }
    for (int o = 0; o < d; ++o) {
        load_row(wd, dtype, (size_t)o * I, I, w);
        y[o] = dot(h, w, I);
    }
    free(w);
    free(h);
    return 0;
}

static const void *expert_ptr(const void *base, int dtype, size_t e, size_t per_expert) {
    size_t esz = dtype == OR_F32 ? 4 : 2;
    return (const char *)base + e * per_expert * esz;
}

/* ---------------------------------------------------------------------------
 * The layer [A][B][D] for the listed tokens only (each token is independent):
 *   y_t = sum_g sum_{e picked in g} p_e FFN_e(x_t)  +  sum_s FFN_s(x_t)
 * summed in pick order (group-major), then the shared experts in index order.
 * x [T][d] double (all tokens; only listed rows are read); y_out [n][d].
 * idx_out/w_out [n][M*Kp] and margin_out [n] may be NULL.
 */
int oracle_layer(const double *x, int T, int d, int N, int M, int Kp, int S, int I, int dtype,
                 const void *w_router, const float *bias,
                 const void *w_gate, const void *w_up, const void *w_down,
                 const void *s_gate, const void *s_up, const void *s_down,
                 const int32_t *tokens, int n, double *y_out,
                 int32_t *idx_out, double *w_out, double *margin_out) {
    if (N % M != 0 || Kp < 1 || Kp > N / M) return 1;
    int K = M * Kp;
    size_t per = (size_t)I * d;
    double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    double *w = (double *)malloc(sizeof(double) * (size_t)K);
    if (!tmp || !idx || !w) { free(tmp); free(idx); free(w); return 2; }
    int rc = 0;
    for (int q = 0; q < n && rc == 0; ++q) {
        int t = tokens[q];
        if (t < 0 || t >= T) { rc = 1; break; }
        const double *xt = x + (size_t)t * d;
        double *yt = y_out + (size_t)q * d;
        double mg;
        rc = oracle_route(xt, w_router, bias, dtype, 1, d, N, M, Kp, idx, w, &mg);
        if (rc) break;
        for (int o = 0; o < d; ++o) yt[o] = 0.0;
        for (int k = 0; k < K; ++k) {
            size_t e = (size_t)idx[k];
            rc = oracle_expert_ffn(xt, expert_ptr(w_gate, dtype, e, per),
                                   expert_ptr(w_up, dtype, e, per),
                                   expert_ptr(w_down, dtype, e, per), dtype, d, I, tmp);
            if (rc) break;
            for (int o = 0; o < d; ++o) yt[o] += w[k] * tmp[o];
        }
        for (int s = 0; s < S && rc == 0; ++s) {
            rc = oracle_expert_ffn(xt, expert_ptr(s_gate, dtype, (size_t)s, per),
                                   expert_ptr(s_up, dtype, (size_t)s, per),
                                   expert_ptr(s_down, dtype, (size_t)s, per), dtype, d, I, tmp);
            for (int o = 0; o < d; ++o) yt[o] += tmp[o];
        }
        if (idx_out) memcpy(idx_out + (size_t)q * K, idx, sizeof(int32_t) * (size_t)K);
        if (w_out) memcpy(w_out + (size_t)q * K, w, sizeof(double) * (size_t)K);
        if (margin_out) margin_out[q] = mg;
    }
    free(tmp);
    free(idx);
    free(w);
    return rc;
}

/* ---------------------------------------------------------------------------
 * RMSNorm with unit gain (pre-norm of the 12-layer stack; the page mentions
 * RMSNorm in section 2, the form and eps are spec choices):
 *   u = x / sqrt(mean(x^2) + eps)
 */
int oracle_rmsnorm(const double *x, int T, int d, double eps, double *u) {
    for (int t = 0; t < T; ++t) {
        const double *xt = x + (size_t)t * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += xt[j] * xt[j];
        double r = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j) u[(size_t)t * d + j] = xt[j] * r;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * 8-bit expert weights. The pages report 8-bit weight quantisation of the
 * model (hwcomputing.csdn.net news piece, deployment section: W8A8 with a
 * small accuracy loss) and an expert-aware quantisation method (techwalker.com
 * article, section 3), but fix no number format. Reading taken: weights-only
 * 8-bit, OCP FP8 E4M3 codes (1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits; no infinities; S.1111.111 is NaN; largest finite 448;
 * subnormals m * 2^-9), one fp32 scale per weight row (output channel):
 *   scale_r = amax_r / 448 (fp32 division; 1 for an all-zero row),
 *   q[r][c] = E4M3 round-to-nearest-even, saturating, of fp32(w[r][c] / scale_r),
 *   dequantised weight = decode(q) * scale_r.
 * Activations stay at the layer's precision (bf16).
 */

/* value of an E4M3 code (NaN codes decode to NaN) */
double oracle_e4m3_decode(uint8_t code) {
    int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* nearest E4M3 code to v, ties to even mantissa, finite results saturating at
 * +-448 (so every finite input maps to a finite code) */
uint8_t oracle_e4m3_encode(float v) {
    double a = fabs((double)v);
    uint8_t sign = signbit(v) ? 0x80 : 0;
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {               /* subnormal range: steps of 2^-9 */
        double n = rint(ldexp(a, 9));       /* current rounding mode: to nearest even */
        return (uint8_t)(sign | (uint8_t)n); /* n == 8 is the smallest normal, code 0x08 */
    }
    int ex;
    double fr = frexp(a, &ex);              /* a = fr * 2^ex, fr in [0.5, 1) */
    int e = ex - 1;                         /* a = (2 fr) * 2^e, 2 fr in [1, 2) */
    double mm = rint((2.0 * fr - 1.0) * 8.0);
    if (mm >= 8.0) { mm = 0.0; e += 1; }
    int be = e + 7;
    if (be > 15 || (be == 15 && mm >= 7.0)) return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | (be << 3) | (int)mm);
}

/* per-row quantisation of bf16 rows (bit patterns) w [rows][cols] */
int oracle_quantize_rows_fp8(const uint16_t *w, int64_t rows, int64_t cols, uint8_t *q,
                             float *scale) {
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *wr = w + r * cols;
        float amax = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            float a = (float)fabs(bf16_bits_to_double(wr[c]));
            if (a > amax) amax = a;
        }
        volatile float s = amax > 0.0f ? amax / 448.0f : 1.0f;  /* one fp32 division */
        scale[r] = s;
        for (int64_t c = 0; c < cols; ++c) {
            volatile float v = (float)bf16_bits_to_double(wr[c]) / s;
            q[r * cols + c] = oracle_e4m3_encode(v);
        }
    }
    return 0;
}

/* row of an fp8 matrix, dequantised: decode(q) * scale (exact in double) */
static void load_row_fp8(const uint8_t *q, const float *scale, size_t row, int n, double *out) {
    const uint8_t *p = q + row * (size_t)n;
    double s = (double)scale[row];
    for (int j = 0; j < n; ++j) out[j] = oracle_e4m3_decode(p[j]) * s;
}

/* One expert on one token with fp8 weights: the same SwiGLU expert as
 * oracle_expert_ffn, on the dequantised matrices. qg, qu [I][d] with scales
 * sg, su [I]; qd [d][I] with scales sd [d]. */
int oracle_expert_ffn_fp8(const double *x, const uint8_t *qg, const float *sg, const uint8_t *qu,
                          const float *su, const uint8_t *qd, const float *sd, int d, int I,
                          double *y) {
    double *w = (double *)malloc(sizeof(double) * (size_t)(d > I ? d : I));
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    if (!w || !h) { free(w); free(h); return 2; }
    for (int i = 0; i < I; ++i) {
        load_row_fp8(qg, sg, (size_t)i, d, w);
        double g = dot(x, w, d);
        load_row_fp8(qu, su, (size_t)i, d, w);
        double u = dot(x, w, d);
        h[i] = (g / (1.0 + exp(-g))) * u;
    }
    for (int o = 0; o < d; ++o) {
        load_row_fp8(qd, sd, (size_t)o, I, w);
        y[o] = dot(h, w, I);
    }
    free(w);
    free(h);
    return 0;
}

/* ---------------------------------------------------------------------------
 * 8-bit weights and 8-bit activations (W8A8). The same deployment section
 * reports a W8A8 configuration; the pages fix neither the format nor where
 * the activations are quantised. Reading taken: the weights as above, and the
 * input of every expert matrix product quantised per token with the same
 * rule: the token's row of x (for the gate and up products) and of h (for
 * the down product), each taken in fp32 first, get
 *   scale = amax / 448 (fp32 division; 1 for an all-zero row),
 *   code  = E4M3 round-to-nearest-even, saturating, of fp32(v / scale),
 * and the product uses decode(code) * scale. The router stays unquantised.
 */

/* per-row activation quantisation of fp64 rows v [rows][cols] (taken in fp32) */
int oracle_quantize_act_rows(const double *v, int64_t rows, int64_t cols, uint8_t *q,
                             float *scale) {
    for (int64_t r = 0; r < rows; ++r) {
        const double *vr = v + r * cols;
        float amax = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf((float)vr[c]);
            if (a > amax) amax = a;
        }
        volatile float s = amax > 0.0f ? amax / 448.0f : 1.0f;  /* one fp32 division */
        scale[r] = s;
        for (int64_t c = 0; c < cols; ++c) {
            volatile float f = (float)vr[c];
            volatile float qv = f / s;
            q[r * cols + c] = oracle_e4m3_encode(qv);
        }
    }
    return 0;
}

/* one activation row replaced by its dequantised 8-bit form, in place */
static void quantize_act_inplace(double *v, int n, uint8_t *codes) {
    float s;
    oracle_quantize_act_rows(v, 1, n, codes, &s);
    for (int j = 0; j < n; ++j) v[j] = oracle_e4m3_decode(codes[j]) * (double)s;
}

/* One expert on one token in W8A8: as oracle_expert_ffn_fp8, with x
 * quantised before the gate and up products and h before the down product. */
int oracle_expert_ffn_w8a8(const double *x, const uint8_t *qg, const float *sg, const uint8_t *qu,
                           const float *su, const uint8_t *qd, const float *sd, int d, int I,
                           double *y) {
    int n = d > I ? d : I;
    double *w = (double *)malloc(sizeof(double) * (size_t)n);
    double *xq = (double *)malloc(sizeof(double) * (size_t)d);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    uint8_t *codes = (uint8_t *)malloc((size_t)n);
    if (!w || !xq || !h || !codes) { free(w); free(xq); free(h); free(codes); return 2; }
    memcpy(xq, x, sizeof(double) * (size_t)d);
    quantize_act_inplace(xq, d, codes);
    for (int i = 0; i < I; ++i) {
        load_row_fp8(qg, sg, (size_t)i, d, w);
        double g = dot(xq, w, d);
        load_row_fp8(qu, su, (size_t)i, d, w);
        double u = dot(xq, w, d);
        h[i] = (g / (1.0 + exp(-g))) * u;
    }
    quantize_act_inplace(h, I, codes);
    for (int o = 0; o < d; ++o) {
        load_row_fp8(qd, sd, (size_t)o, I, w);
        y[o] = dot(h, w, I);
    }
    free(w);
    free(xq);
    free(h);
    free(codes);
    return 0;
}

typedef int (*expert_fn8)(const double *, const uint8_t *, const float *, const uint8_t *,
                          const float *, const uint8_t *, const float *, int, int, double *);

/* The layer [A][B][D] with 8-bit expert weights (routed and shared), router
 * weights and activations as in oracle_layer (dtype of x / w_router):
 * routed expert e uses qg + e I d, sg + e I, ..., qd + e d I, sd + e d;
 * each expert evaluated by `ffn` (weights-only or W8A8). */
static int layer_8bit(const double *x, int T, int d, int N, int M, int Kp, int S, int I, int dtype,
                      const void *w_router, const float *bias,
                      const uint8_t *qg, const float *sg, const uint8_t *qu, const float *su,
                      const uint8_t *qd, const float *sd,
                      const uint8_t *sqg, const float *ssg, const uint8_t *squ, const float *ssu,
                      const uint8_t *sqd, const float *ssd,
                      const int32_t *tokens, int n, double *y_out,
                      int32_t *idx_out, double *w_out, double *margin_out, expert_fn8 ffn) {
    if (N % M != 0 || Kp < 1 || Kp > N / M) return 1;
    int K = M * Kp;
    size_t per = (size_t)I * d;
    double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    double *w = (double *)malloc(sizeof(double) * (size_t)K);
    if (!tmp || !idx || !w) { free(tmp); free(idx); free(w); return 2; }
    int rc = 0;
    for (int q = 0; q < n && rc == 0; ++q) {
        int t = tokens[q];
        if (t < 0 || t >= T) { rc = 1; break; }
        const double *xt = x + (size_t)t * d;
        double *yt = y_out + (size_t)q * d;
        double mg;
        rc = oracle_route(xt, w_router, bias, dtype, 1, d, N, M, Kp, idx, w, &mg);
        if (rc) break;
        for (int o = 0; o < d; ++o) yt[o] = 0.0;
        for (int k = 0; k < K; ++k) {
            size_t e = (size_t)idx[k];
            rc = ffn(xt, qg + e * per, sg + e * I, qu + e * per, su + e * I, qd + e * per,
                     sd + e * d, d, I, tmp);
            if (rc) break;
            for (int o = 0; o < d; ++o) yt[o] += w[k] * tmp[o];
        }
        for (int s = 0; s < S && rc == 0; ++s) {
            size_t e = (size_t)s;
            rc = ffn(xt, sqg + e * per, ssg + e * I, squ + e * per, ssu + e * I, sqd + e * per,
                     ssd + e * d, d, I, tmp);
            for (int o = 0; o < d; ++o) yt[o] += tmp[o];
        }
        if (idx_out) memcpy(idx_out + (size_t)q * K, idx, sizeof(int32_t) * (size_t)K);
        if (w_out) memcpy(w_out + (size_t)q * K, w, sizeof(double) * (size_t)K);
        if (margin_out) margin_out[q] = mg;
    }
    free(tmp);
    free(idx);
    free(w);
    return rc;
}

int oracle_layer_fp8(const double *x, int T, int d, int N, int M, int Kp, int S, int I, int dtype,
                     const void *w_router, const float *bias,
                     const uint8_t *qg, const float *sg, const uint8_t *qu, const float *su,
                     const uint8_t *qd, const float *sd,
                     const uint8_t *sqg, const float *ssg, const uint8_t *squ, const float *ssu,
                     const uint8_t *sqd, const float *ssd,
                     const int32_t *tokens, int n, double *y_out,
                     int32_t *idx_out, double *w_out, double *margin_out) {
    return layer_8bit(x, T, d, N, M, Kp, S, I, dtype, w_router, bias, qg, sg, qu, su, qd, sd, sqg,
                      ssg, squ, ssu, sqd, ssd, tokens, n, y_out, idx_out, w_out, margin_out,
                      oracle_expert_ffn_fp8);
}

/* The layer in W8A8 (oracle_expert_ffn_w8a8 per expert), otherwise as oracle_layer_fp8. */
int oracle_layer_w8a8(const double *x, int T, int d, int N, int M, int Kp, int S, int I, int dtype,
                      const void *w_router, const float *bias,
                      const uint8_t *qg, const float *sg, const uint8_t *qu, const float *su,
                      const uint8_t *qd, const float *sd,
                      const uint8_t *sqg, const float *ssg, const uint8_t *squ, const float *ssu,
                      const uint8_t *sqd, const float *ssd,
                      const int32_t *tokens, int n, double *y_out,
                      int32_t *idx_out, double *w_out, double *margin_out) {
    return layer_8bit(x, T, d, N, M, Kp, S, I, dtype, w_router, bias, qg, sg, qu, su, qd, sd, sqg,
                      ssg, squ, ssu, sqd, ssd, tokens, n, y_out, idx_out, w_out, margin_out,
                      oracle_expert_ffn_w8a8);
}

/* One (token, expert) term of the backward pass below, with the expert's
 * weight w for this token: accumulates w dy h^T into gd, dg x^T into gg and
 * du x^T into gu, and Wg^T dg + Wu^T du into dxt (any of them may be NULL); returns
 * dy . (Wd h). Scratch: row [max(d, I)], g, u, h, dh [I]. */
static double expert_token_backward(const double *xt, const double *dyt, double w,
                                    const void *wg, const void *wu, const void *wd, int dtype,
                                    int d, int I, double *gg, double *gu, double *gd, double *dxt,
                                    double *row, double *g, double *u, double *h, double *dh) {
    for (int i = 0; i < I; ++i) {
        load_row(wg, dtype, (size_t)i * d, d, row);
        g[i] = dot(xt, row, d);
        load_row(wu, dtype, (size_t)i * d, d, row);
        u[i] = dot(xt, row, d);
        h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
        dh[i] = 0.0;
    }
    double o_dot = 0.0;
    for (int o = 0; o < d; ++o) {
        load_row(wd, dtype, (size_t)o * I, I, row);
        o_dot += dyt[o] * dot(h, row, I);
        for (int i = 0; i < I; ++i) {
            dh[i] += w * dyt[o] * row[i];
            if (gd) gd[(size_t)o * I + i] += w * dyt[o] * h[i];
        }
    }
    for (int i = 0; i < I; ++i) {
        const double s = 1.0 / (1.0 + exp(-g[i]));
        const double dg = dh[i] * u[i] * s * (1.0 + g[i] * (1.0 - s));
        const double du = dh[i] * g[i] * s;
        load_row(wg, dtype, (size_t)i * d, d, row);
        for (int c = 0; c < d; ++c) {
            if (gg) gg[(size_t)i * d + c] += dg * xt[c];
            if (dxt) dxt[c] += dg * row[c];
        }
        load_row(wu, dtype, (size_t)i * d, d, row);
        for (int c = 0; c < d; ++c) {
            if (gu) gu[(size_t)i * d + c] += du * xt[c];
            if (dxt) dxt[c] += du * row[c];
        }
    }
    return o_dot;
}

/* ---------------------------------------------------------------------------
 * Backward pass of the layer [A][B][D] for an upstream gradient dy [T][d],
 * with the routing held at its forward value (the picks are piecewise
 * constant in the inputs), plus the batch-level balance loss named in [E]:
 *   L_aux = alpha * sum_i f_i P_i,  f_i = c_i / T,  P_i = (1/T) sum_t p[t][i],
 * c_i the number of tokens routed to expert i in the batch; f_i is a count,
 * so only P_i carries a gradient. ([E]: reportify.cn concept page "Mixture of
 * grouped experts", bullet "technical innovation details": a batch-level
 * auxiliary balance loss whose strength is alpha and whose f_i is the share of
 * the batch's tokens routed to expert i; the page prints no formula, the
 * product form above is a reading.)
 *
 * For token t and each picked expert e with weight w = p[t][e] (shared
 * experts: w = 1), writing g = Wg x, u = Wu x, h = silu(g) * u, o = Wd h:
 *   dp[t][e]  = dy_t . o                       (routed experts only)
 *   dh        = w * Wd^T dy_t
 *   dg        = dh * u * silu'(g),  du = dh * silu(g),
 *               silu'(g) = s (1 + g (1 - s)),  s = 1 / (1 + e^-g)
 *   dWd      += w * dy_t h^T,  dWg += dg x_t^T,  dWu += du x_t^T
 *   dx_t     += Wg^T dg + Wu^T du
 * then, with dp[t][i] += alpha * f_i / T for every expert i,
 *   dl[t][i]  = p[t][i] (dp[t][i] - sum_j p[t][j] dp[t][j])   (softmax)
 *   dWr[i]   += dl[t][i] x_t,   dx_t += sum_i dl[t][i] Wr[i].
 * idx_in (may be NULL): picks [T][M*Kp] to hold the routing at instead of the
 * oracle's own selection (tokens whose top scores tie within rounding have
 * more than one correct pick; each must lie in its group).
 * tokens (may be NULL): only these n_tokens tokens' terms are taken -- their
 * dx rows are then exact (other rows zero), the weight gradients partial; the
 * routing and the balance loss's f still come from the whole batch.
 * Each group of weight-gradient outputs may be NULL on its own (the router's
 * dwr; the routed experts' dwg, dwu, dwd together; the shared experts' dsg,
 * dsu, dsd together): that group is then not formed. All NULL: only dx.
 * Every output array is overwritten. Shapes: dx [T][d], dwr [N][d],
 * dwg/dwu [N][I][d], dwd [N][d][I], dsg/dsu [S][I][d], dsd [S][d][I].
 * aux_out (may be NULL) receives L_aux.
 */
int oracle_layer_backward(const double *x, int T, int d, int N, int M, int Kp, int S, int I,
                          int dtype, const void *w_router, const float *bias,
                          const void *w_gate, const void *w_up, const void *w_down,
                          const void *s_gate, const void *s_up, const void *s_down,
                          const double *dy, double alpha, const int32_t *idx_in,
                          const int32_t *tokens, int n_tokens, double *dx,
                          double *dwr, double *dwg,
                          double *dwu, double *dwd, double *dsg, double *dsu, double *dsd,
                          double *aux_out) {
    if (T < 0 || N <= 0 || M <= 0 || N % M != 0 || Kp < 1 || Kp > N / M) return 1;
    const int K = M * Kp;
    const size_t per = (size_t)I * d;
    double *p = (double *)malloc(sizeof(double) * ((size_t)T * N + 1));
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * ((size_t)T * K + 1));
    double *wk = (double *)malloc(sizeof(double) * ((size_t)T * K + 1));
    double *f = (double *)calloc((size_t)N, sizeof(double));
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    double *row = (double *)malloc(sizeof(double) * (size_t)(d > I ? d : I));
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    double *dh = (double *)malloc(sizeof(double) * (size_t)I);
    if (!p || !idx || !wk || !f || !dp || !row || !g || !u || !h || !dh) {
        free(p); free(idx); free(wk); free(f); free(dp); free(row); free(g); free(u); free(h);
        free(dh);
        return 2;
    }
    const int wgr = dwr != NULL, wge = dwg != NULL, wgs = dsg != NULL;
    memset(dx, 0, sizeof(double) * (size_t)T * d);
    if (wgr) memset(dwr, 0, sizeof(double) * (size_t)N * d);
    if (wge) {
        memset(dwg, 0, sizeof(double) * (size_t)N * per);
        memset(dwu, 0, sizeof(double) * (size_t)N * per);
        memset(dwd, 0, sizeof(double) * (size_t)N * per);
    }
    if (wgs && S > 0) {
        memset(dsg, 0, sizeof(double) * (size_t)S * per);
        memset(dsu, 0, sizeof(double) * (size_t)S * per);
        memset(dsd, 0, sizeof(double) * (size_t)S * per);
    }
    int rc = oracle_router_probs(x, w_router, bias, dtype, T, d, N, p);
    if (!rc) rc = oracle_select_grouped(p, T, N, M, Kp, idx, wk, NULL);
    if (!rc && idx_in) {
        const int G = N / M;
        for (int t = 0; t < T && !rc; ++t)
            for (int k = 0; k < K; ++k) {
                const int e = idx_in[(size_t)t * K + k];
                if (e < (k / Kp) * G || e >= (k / Kp + 1) * G) { rc = 1; break; }
                idx[(size_t)t * K + k] = e;
                wk[(size_t)t * K + k] = p[(size_t)t * N + e];
            }
    }
    double aux = 0.0;
    if (!rc && T > 0) {
        for (size_t i = 0; i < (size_t)T * K; ++i) f[idx[i]] += 1.0 / T;
        for (int e = 0; e < N; ++e) {
            double P = 0.0;
            for (int t = 0; t < T; ++t) P += p[(size_t)t * N + e];
            aux += alpha * f[e] * (P / T);
        }
    }
    const int n_run = tokens ? n_tokens : T;
    for (int q = 0; q < n_run && !rc; ++q) {
        const int t = tokens ? tokens[q] : q;
        if (t < 0 || t >= T) { rc = 1; break; }
        const double *xt = x + (size_t)t * d;
        const double *dyt = dy + (size_t)t * d;
        double *dxt = dx + (size_t)t * d;
        for (int e = 0; e < N; ++e) dp[e] = alpha * f[e] / T;
        for (int k = 0; k < K + S; ++k) {
            const int routed = k < K;
            const size_t e = routed ? (size_t)idx[(size_t)t * K + k] : (size_t)(k - K);
            const double w = routed ? wk[(size_t)t * K + k] : 1.0;
            const double o_dot = expert_token_backward(
                xt, dyt, w,
                routed ? expert_ptr(w_gate, dtype, e, per) : expert_ptr(s_gate, dtype, e, per),
                routed ? expert_ptr(w_up, dtype, e, per) : expert_ptr(s_up, dtype, e, per),
                routed ? expert_ptr(w_down, dtype, e, per) : expert_ptr(s_down, dtype, e, per),
                dtype, d, I, (routed ? wge : wgs) ? (routed ? dwg : dsg) + e * per : NULL,
                (routed ? wge : wgs) ? (routed ? dwu : dsu) + e * per : NULL,
                (routed ? wge : wgs) ? (routed ? dwd : dsd) + e * per : NULL, dxt, row, g, u, h, dh);
            if (routed) dp[e] += o_dot;
        }
        const double *pt = p + (size_t)t * N;
        double pdp = 0.0;
        for (int e = 0; e < N; ++e) pdp += pt[e] * dp[e];
        for (int e = 0; e < N; ++e) {
            const double dl = pt[e] * (dp[e] - pdp);
            load_row(w_router, dtype, (size_t)e * d, d, row);
            for (int c = 0; c < d; ++c) {
                if (wgr) dwr[(size_t)e * d + c] += dl * xt[c];
                dxt[c] += dl * row[c];
            }
        }
    }
    if (aux_out) *aux_out = aux;
    free(p); free(idx); free(wk); free(f); free(dp); free(row); free(g); free(u); free(h); free(dh);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Weight gradients of ONE expert from the n tokens that chose it (rows x and
 * dy [n][d], weights w [n]: the tokens' routing scores, 1 for a shared expert):
 * the same terms as oracle_layer_backward, summed over those tokens only --
 * which is the whole of that expert's gradient. dwg, dwu [I][d], dwd [d][I]
 * are overwritten. wg, wu point at the expert's [I][d], wd at its [d][I].
 */
int oracle_expert_backward(const double *x, const double *dy, const double *w, int n,
                           const void *wg, const void *wu, const void *wd, int dtype, int d, int I,
                           double *dwg, double *dwu, double *dwd) {
    const size_t per = (size_t)I * d;
    double *row = (double *)malloc(sizeof(double) * (size_t)(d > I ? d : I));
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    double *dh = (double *)malloc(sizeof(double) * (size_t)I);
    if (!row || !g || !u || !h || !dh) {
        free(row); free(g); free(u); free(h); free(dh);
        return 2;
    }
    memset(dwg, 0, sizeof(double) * per);
    memset(dwu, 0, sizeof(double) * per);
    memset(dwd, 0, sizeof(double) * per);
    for (int q = 0; q < n; ++q)
        expert_token_backward(x + (size_t)q * d, dy + (size_t)q * d, w[q], wg, wu, wd, dtype, d, I,
                              dwg, dwu, dwd, NULL, row, g, u, h, dh);
    free(row); free(g); free(u); free(h); free(dh);
    return 0;
}

/* ---------------------------------------------------------------------------
 * One rank's share of the layer under expert parallelism ([A] section 1:
 * experts reorganised by device, one group per device; section 2: the shared
 * experts split across devices): with the router over ALL N experts, the
 * picks that fall on experts [e0, e0 + n_loc) -- whose weights are given
 * alone, wg/wu [n_loc][I][d], wd [n_loc][d][I] -- weighted by their global
 * scores, plus every shared expert restricted to I_s of its intermediate
 * features (sg/su [S][I_s][d], sd [S][d][I_s]; W_down's matching columns):
 *   y_r(t) = sum_{picks e in [e0, e0 + n_loc)} p_e FFN_e(x_t)
 *          + sum_s W_down,s[:, slice] (silu(W_gate,s[slice] x_t) * (W_up,s[slice] x_t)).
 * Summed over a partition of the experts and of the shared features, the
 * partials are the layer. Listed tokens only; y_out [n][d].
 */
int oracle_layer_ep_partial(const double *x, int T, int d, int N, int M, int Kp, int S, int I,
                            int dtype, const void *w_router, const float *bias, int e0, int n_loc,
                            const void *w_gate, const void *w_up, const void *w_down, int I_s,
                            const void *s_gate, const void *s_up, const void *s_down,
                            const int32_t *tokens, int n, double *y_out) {
    if (N % M != 0 || Kp < 1 || Kp > N / M || e0 < 0 || n_loc < 0 || e0 + n_loc > N) return 1;
    const int K = M * Kp;
    const size_t per = (size_t)I * d, per_s = (size_t)I_s * d;
    double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    double *w = (double *)malloc(sizeof(double) * (size_t)K);
    if (!tmp || !idx || !w) { free(tmp); free(idx); free(w); return 2; }
    int rc = 0;
    for (int q = 0; q < n && rc == 0; ++q) {
        const int t = tokens[q];
        if (t < 0 || t >= T) { rc = 1; break; }
        const double *xt = x + (size_t)t * d;
        double *yt = y_out + (size_t)q * d;
        double mg;
        rc = oracle_route(xt, w_router, bias, dtype, 1, d, N, M, Kp, idx, w, &mg);
        if (rc) break;
        for (int o = 0; o < d; ++o) yt[o] = 0.0;
        for (int k = 0; k < K; ++k) {
            const int e = idx[k];
            if (e < e0 || e >= e0 + n_loc) continue;
            const size_t le = (size_t)(e - e0);
            rc = oracle_expert_ffn(xt, expert_ptr(w_gate, dtype, le, per),
                                   expert_ptr(w_up, dtype, le, per),
                                   expert_ptr(w_down, dtype, le, per), dtype, d, I, tmp);
            if (rc) break;
            for (int o = 0; o < d; ++o) yt[o] += w[k] * tmp[o];
        }
        for (int s = 0; s < S && rc == 0 && I_s > 0; ++s) {
            rc = oracle_expert_ffn(xt, expert_ptr(s_gate, dtype, (size_t)s, per_s),
                                   expert_ptr(s_up, dtype, (size_t)s, per_s),
                                   expert_ptr(s_down, dtype, (size_t)s, per_s), dtype, d, I_s, tmp);
            for (int o = 0; o < d; ++o) yt[o] += tmp[o];
        }
    }
    free(tmp);
    free(idx);
    free(w);
    return rc;
}
