/*
 * CPU oracle for the forward pass of one Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file defines what the layer computes, in the
 * plainest form: one token at a time, every sum in double precision in index
 * order, no tiling, blocking or fusion.  It shares no code with the CUDA
 * library; only the test suite, the smoke check and the benchmark's CPU
 * baseline may load it.
 *
 * The pages name the layer's parts without writing its formulas:
 *   - routing: each token picks k of E experts ("3-in-48" expert selection,
 *     Step3 推論最適化 (MI308X vs H20), §背景);
 *   - expert FFN with gate/up and a down projection GEMM ("MoE one-stage
 *     kernel" tuned along inter_dim, same page §最適化技術; "down projection
 *     GEMM", [SGLang] MoE 모델을 위한 Single Batch Overlap 기법, §들어가며);
 *   - weighted combine of the k expert outputs (combine phase, same page);
 *   - an always-on shared expert fused into the layer (Step3 page,
 *     §最適化技術, "Shared-expert MLP 融合");
 *   - mixed BF16 / FP8-blockscale arithmetic (Step3 page, §最適化技術;
 *     "GEMM à l'échelle bloc", AMD Instinct MI355X : ATOM, kernels fusionnés
 *     et montée en charge, introduction).
 * Where the pages are silent the plainest standard reading is taken:
 *   logits  l[e] = sum_h x[h] * Wr[e,h] (+ b[e])
 *   top-k   the k largest logits, ties to the lower expert index
 *   weights softmax of the selected logits (renormalised), or of all E
 *   expert  y = Wd (silu(Wg x) * (Wu x)),  silu(z) = z / (1 + e^-z)
 *   combine out = bf16_rne( sum_j w_j y_j + y_shared )
 *   padding rows are not routed, not computed, and give +0.0.
 *
 * Precision: double everywhere, except where a floating-point value decides
 * an integer and must be decided exactly as the GPU decides it: expert
 * selection compares fp32 logits, and the FP8 activation codes are taken from
 * the fp32 quotient x / s with s = amax / 448 in fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the token loops below run on (what a timing of the oracle used). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---------------------------------------------------------------- codecs */

/* bf16 -> double: a bf16 is the top 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static uint16_t float_bits_top(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* double -> bf16, one rounding, to nearest with ties to even.
 * bf16 keeps 8 significant bits and binary32's exponent range: normal values
 * have a quantum of 2^(e-7) for |v| in [2^e, 2^(e+1)), and below 2^-126 the
 * quantum is fixed at 2^-133.  Dividing by a power of two is exact in double,
 * and rint() rounds to nearest-even in the default rounding mode. */
uint16_t oracle_double_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    double q;
    if (a < ldexp(1.0, -126)) {
        q = rint(a / ldexp(1.0, -133)) * ldexp(1.0, -133);
    } else {
        int ex;
        frexp(a, &ex);                    /* a = f * 2^ex, f in [0.5, 1) */
        double quantum = ldexp(1.0, ex - 8);
        q = rint(a / quantum) * quantum;
    }
    if (q >= ldexp(1.0, 128)) return signbit(v) ? 0xFF80 : 0x7F80;   /* overflow to inf */
    float f = (float)q;                   /* exact: q has <= 8 significant bits */
    uint16_t bits = float_bits_top(f);
    return signbit(v) ? (uint16_t)(bits | 0x8000) : bits;
}

/* OCP OFP8 E4M3 (exponent bias 7, 3 mantissa bits, no infinities,
 * S.1111.111 is NaN, largest finite 448, subnormal step 2^-9). */
double oracle_e4m3_to_double(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? (m / 8.0) * ldexp(1.0, -6) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return s ? -mag : mag;
}

/* fp32 -> E4M3, round to nearest even, saturating to +-448; NaN -> 0x7F. */
uint8_t oracle_float_to_e4m3_sat(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    double q;
    if (a < ldexp(1.0, -6)) {
        q = rint(a / ldexp(1.0, -9)) * ldexp(1.0, -9);
    } else {
        int ex;
        frexp(a, &ex);                    /* a in [2^(ex-1), 2^ex) */
        double quantum = ldexp(1.0, ex - 1 - 3);
        q = rint(a / quantum) * quantum;
    }
    if (q > 448.0) q = 448.0;
    if (q == 0.0) return sign;
    /* encode the representable magnitude q */
    if (q < ldexp(1.0, -6)) {
        int m = (int)(q / ldexp(1.0, -9));            /* 1..7 */
        return (uint8_t)(sign | m);
    }
    int ex;
    double f = frexp(q, &ex);            /* q = f * 2^ex, f in [0.5,1) */
    int e = ex - 1 + 7;                  /* biased exponent */
    int m = (int)((f * 2.0 - 1.0) * 8.0);
    return (uint8_t)(sign | (e << 3) | m);
}

/* --------------------------------------------------------- a1: router logits */

/* l[t,e] = sum_h x[t,h] * Wr[e,h] (+ b[e]), double sum over h ascending, one
 * rounding to float.  Padding rows (valid[t] == 0) get 0. */
void oracle_router_logits(const uint16_t *x, const uint8_t *valid, int T, int H,
                          const float *Wr, const float *b, int E, float *logits) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            if (valid && !valid[t]) { logits[(size_t)t * E + e] = 0.0f; continue; }
            double s = 0.0;
            for (int h = 0; h < H; ++h)
                s += oracle_bf16_to_double(x[(size_t)t * H + h]) * (double)Wr[(size_t)e * H + h];
            if (b) s += (double)b[e];
            logits[(size_t)t * E + e] = (float)s;
        }
    }
}

/* ------------------------------------------------ a2: top-k and the weights */

/* Expert a precedes expert b iff l[a] > l[b], or l[a] == l[b] and a < b. */
static int precedes(const float *l, int a, int b) {
    return l[a] > l[b] || (l[a] == l[b] && a < b);
}

/* ids[t, 0..k-1]: the first k experts in that order (selection by repeated
 * minimum search).  w[t,j]: renorm != 0 -> exp(l_j - l_0) / sum_j' exp(l_j' - l_0)
 * over the k selected; renorm == 0 -> softmax over all E experts.
 * Padding rows: ids = -1, w = 0. */
void oracle_topk(const float *logits, const uint8_t *valid, int T, int E, int k, int renorm,
                 int *ids, double *w) {
    for (int t = 0; t < T; ++t) {
        int *id = ids + (size_t)t * k;
        double *wt = w + (size_t)t * k;
        if (valid && !valid[t]) {
            for (int j = 0; j < k; ++j) { id[j] = -1; wt[j] = 0.0; }
            continue;
        }
        const float *l = logits + (size_t)t * E;
        unsigned char *taken = (unsigned char *)calloc((size_t)E, 1);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || precedes(l, e, best))) best = e;
            taken[best] = 1;
            id[j] = best;
        }
        free(taken);
        double m = (double)l[id[0]];
        double z = 0.0;
        if (renorm) {
            for (int j = 0; j < k; ++j) z += exp((double)l[id[j]] - m);
        } else {
            for (int e = 0; e < E; ++e) z += exp((double)l[e] - m);
        }
        for (int j = 0; j < k; ++j) wt[j] = exp((double)l[id[j]] - m) / z;
    }
}

/* ------------------------------- a3: histogram, offsets and the permutation */

/* counts[e] = number of valid (t, j) routed to e; offsets = exclusive prefix
 * sum (E + 1 entries); perm[offsets[e] + r] = t*k + j for the r-th such pair in
 * ascending t; inv[t*k + j] = its position (-1 for padding rows).
 * Returns the number of routed pairs. */
int oracle_route(const int *ids, const uint8_t *valid, int T, int E, int k,
                 int *counts, int *offsets, int *perm, int *inv) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int t = 0; t < T; ++t) {
        if (valid && !valid[t]) continue;
        for (int j = 0; j < k; ++j) counts[ids[(size_t)t * k + j]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int *fill = (int *)calloc((size_t)E, sizeof(int));
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            size_t p = (size_t)t * k + j;
            if (valid && !valid[t]) { inv[p] = -1; continue; }
            int e = ids[p];
            int pos = offsets[e] + fill[e]++;
            perm[pos] = (int)p;
            inv[p] = pos;
        }
    }
    free(fill);
    return offsets[E];
}

/* --------------------------------------------- a4-a6: expert FFN and combine */

/* One bf16 SwiGLU expert on one token: y[o] = sum_i h[i] Wd[o,i] with
 * h[i] = silu(g[i]) u[i], g = Wgu[0:I] x, u = Wgu[I:2I] x.  Adds scale * y to acc. */
static void expert_bf16(const uint16_t *xt, int H, const uint16_t *Wgu, const uint16_t *Wd,
                        int I, double scale, double *acc, double *hbuf) {
    for (int i = 0; i < I; ++i) {
        const uint16_t *wg = Wgu + (size_t)i * H;
        const uint16_t *wu = Wgu + (size_t)(I + i) * H;
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            double xv = oracle_bf16_to_double(xt[h]);
            g += xv * oracle_bf16_to_double(wg[h]);
            u += xv * oracle_bf16_to_double(wu[h]);
        }
        hbuf[i] = g / (1.0 + exp(-g)) * u;
    }
    for (int o = 0; o < H; ++o) {
        const uint16_t *wd = Wd + (size_t)o * I;
        double y = 0.0;
        for (int i = 0; i < I; ++i) y += hbuf[i] * oracle_bf16_to_double(wd[i]);
        acc[o] += scale * y;
    }
}

/* acc[n, :] = sum_j w[t,j] * expert_{ids[t,j]}(x[t]) + shared(x[t]) for each
 * t = tokens[n] (a padding row, ids[t,0] < 0, leaves zeros).  The j sum runs
 * in ascending j, then the shared expert (weight 1) is added. */
void oracle_moe_tokens_bf16(const uint16_t *x, int H, const int *ids, const double *w, int k,
                            const uint16_t *Wgu, const uint16_t *Wd, int I,
                            const uint16_t *Wsgu, const uint16_t *Wsd, int Is,
                            const int *tokens, int n_tokens, double *acc) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_tokens; ++n) {
        int t = tokens[n];
        double *a = acc + (size_t)n * H;
        for (int o = 0; o < H; ++o) a[o] = 0.0;
        if (ids[(size_t)t * k] < 0) continue;
        int hmax = I > Is ? I : Is;
        double *hbuf = (double *)malloc(sizeof(double) * (size_t)(hmax > 0 ? hmax : 1));
        const uint16_t *xt = x + (size_t)t * H;
        for (int j = 0; j < k; ++j) {
            int e = ids[(size_t)t * k + j];
            expert_bf16(xt, H, Wgu + (size_t)e * 2 * I * H, Wd + (size_t)e * H * I, I,
                        w[(size_t)t * k + j], a, hbuf);
        }
        if (Wsgu && Wsd) expert_bf16(xt, H, Wsgu, Wsd, Is, 1.0, a, hbuf);
        free(hbuf);
    }
}

/* ------------------------------------------------------ FP8 block-scale path */

/* Activation quantisation, one 1x128 group at a time along a row of n values:
 * amax over the group's fp32 values, s = amax / 448 (fp32 division; 1 when
 * amax == 0), q = e4m3_rne_sat(v / s) with v / s an fp32 division. */
void oracle_quant_row_e4m3(const float *v, int n, uint8_t *q, float *s) {
    for (int g = 0; g < n / 128; ++g) {
        float amax = 0.0f;
        for (int i = 0; i < 128; ++i) {
            float a = fabsf(v[g * 128 + i]);
            if (a > amax) amax = a;
        }
        float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
        s[g] = sc;
        for (int i = 0; i < 128; ++i) q[g * 128 + i] = oracle_float_to_e4m3_sat(v[g * 128 + i] / sc);
    }
}

/* Block-scaled dot product of row n of an e4m3 matrix W [N, K] (scales
 * sw [N/128, K/128]) with a quantised activation row (qa, sa [K/128]):
 * sum_kb sa[kb] * sw[n/128, kb] * sum_{k in kb} qa[k] * W[n, k]. */
static double dot_fp8(const uint8_t *qa, const float *sa, const uint8_t *W, const float *sw,
                      int n, int K) {
    double total = 0.0;
    for (int kb = 0; kb < K / 128; ++kb) {
        double part = 0.0;
        const uint8_t *wr = W + (size_t)n * K + (size_t)kb * 128;
        for (int i = 0; i < 128; ++i)
            part += oracle_e4m3_to_double(qa[kb * 128 + i]) * oracle_e4m3_to_double(wr[i]);
        total += (double)sa[kb] * (double)sw[(size_t)(n / 128) * (K / 128) + kb] * part;
    }
    return total;
}

static void expert_fp8(const uint8_t *qx, const float *sx, int H,
                       const uint8_t *Wgu, const float *sgu, const uint8_t *Wd, const float *sd,
                       int I, double scale, double *acc, float *hbuf, uint8_t *qh, float *sh) {
    for (int i = 0; i < I; ++i) {
        double g = dot_fp8(qx, sx, Wgu, sgu, i, H);
        double u = dot_fp8(qx, sx, Wgu, sgu, I + i, H);
        hbuf[i] = (float)(g / (1.0 + exp(-g)) * u);
    }
    oracle_quant_row_e4m3(hbuf, I, qh, sh);
    for (int o = 0; o < H; ++o) acc[o] += scale * dot_fp8(qh, sh, Wd, sd, o, I);
}

/* As oracle_moe_tokens_bf16 with e4m3 weights and 128x128 fp32 block scales:
 * Wgu [E,2I,H] + sgu [E,2I/128,H/128], Wd [E,H,I] + sd [E,H/128,I/128]; the
 * shared expert likewise (NULL when absent).  x rows are quantised 1x128 from
 * their fp32 values, h rows likewise from fp32(h). */
void oracle_moe_tokens_fp8(const uint16_t *x, int H, const int *ids, const double *w, int k,
                           const uint8_t *Wgu, const float *sgu, const uint8_t *Wd,
                           const float *sd, int I,
                           const uint8_t *Wsgu, const float *ssgu, const uint8_t *Wsd,
                           const float *ssd, int Is,
                           const int *tokens, int n_tokens, double *acc) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_tokens; ++n) {
        int t = tokens[n];
        double *a = acc + (size_t)n * H;
        for (int o = 0; o < H; ++o) a[o] = 0.0;
        if (ids[(size_t)t * k] < 0) continue;
        int hmax = I > Is ? I : Is;
        float *xf = (float *)malloc(sizeof(float) * (size_t)H);
        uint8_t *qx = (uint8_t *)malloc((size_t)H);
        float *sx = (float *)malloc(sizeof(float) * (size_t)(H / 128));
        float *hbuf = (float *)malloc(sizeof(float) * (size_t)hmax);
        uint8_t *qh = (uint8_t *)malloc((size_t)hmax);
        float *sh = (float *)malloc(sizeof(float) * (size_t)(hmax / 128 + 1));
        for (int h = 0; h < H; ++h) xf[h] = (float)oracle_bf16_to_double(x[(size_t)t * H + h]);
        oracle_quant_row_e4m3(xf, H, qx, sx);
        size_t gu_sz = (size_t)2 * I * H, gu_s = (size_t)(2 * I / 128) * (H / 128);
        size_t d_sz = (size_t)H * I, d_s = (size_t)(H / 128) * (I / 128);
        for (int j = 0; j < k; ++j) {
            int e = ids[(size_t)t * k + j];
            expert_fp8(qx, sx, H, Wgu + e * gu_sz, sgu + e * gu_s, Wd + e * d_sz, sd + e * d_s,
                       I, w[(size_t)t * k + j], a, hbuf, qh, sh);
        }
        if (Wsgu && Wsd) expert_fp8(qx, sx, H, Wsgu, ssgu, Wsd, ssd, Is, 1.0, a, hbuf, qh, sh);
        free(xf); free(qx); free(sx); free(hbuf); free(qh); free(sh);
    }
}

/* out[n,:] = bf16_rne(acc[n,:]) */
void oracle_round_bf16(const double *acc, size_t n, uint16_t *out) {
    for (size_t i = 0; i < n; ++i) out[i] = oracle_double_to_bf16(acc[i]);
}
