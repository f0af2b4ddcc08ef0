/*
 * fg_oracle.c -- plain, slow, obviously-correct CPU oracle for the group-wise
 * 4-bit ("W4 KV4") OPT decode step.
 *
 * TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code, header,
 * table or constant with the CUDA library and never calls it.
 *
 * What it follows (the web pages the method is described on):
 *   [G3]  "FlexGen Guide: High-Throughput LLM Offloading on One GPU",
 *         section "3. Group-Wise 4-Bit Quantization for Weights and KV Cache":
 *         weights and KV cache compressed to 4-bit integers, per-group scaling
 *         over small contiguous groups (64), dequantised to FP16 for compute.
 *   [G2]  same page, section "2. The Zig-Zag Block Schedule": a loaded layer
 *         is reused for every micro-batch of the block, so a row's result
 *         does not depend on the batch split.
 *   [OPT] the OPT entry in the PIPO paper's list of references (model family):
 *         pre-LayerNorm decoder layer, multi-head attention, ReLU FFN.
 *
 * Readings where the pages are silent (all listed in the design notes):
 *   - asymmetric min-max per group: scale = fp16((max-min)/15), codes
 *     round-half-even of (x-min)*(1/scale) in fp32, clamp to [0,15], two
 *     codes per byte with the even element in the low nibble, fp16 min and
 *     fp16 scale stored in separate planar arrays;
 *   - a zero scale (constant group, or a scale that underflows fp16) gives
 *     all codes 0 and a stored +0 scale; -0 min is stored as +0;
 *   - dequantised value = min + code*scale computed exactly, rounded once to
 *     fp16 (the FP16 fused multiply-add);
 *   - the layer is an FP16 layer: every op is evaluated in float64 from fp16
 *     operands (the dequantised fp16 weights and fp16 activations), and every
 *     activation tensor one op hands to the next is rounded to fp16: the
 *     LayerNorm outputs, q (after its bias and the d^-1/2 scale), k and v,
 *     the attention output, the residual stream h1 and the ReLU output.  The
 *     layer output itself is returned unrounded (float64).  The new token's
 *     k and v are appended to the cache in 4-bit form before attention, which
 *     runs over the dequantised cache including the new token.  LayerNorm eps
 *     as passed (1e-5 for OPT).
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared -pthread (no fast-math), so
 * every float operation below is one IEEE-754 operation rounded to nearest.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_GROUP 64       /* the default group size (the layer takes 64 or 128) */
#define OR_GROUP_MAX 128  /* quantise/dequantise/linear also take groups of 128 [G3] */

/* ------------------------------------------------------------------------- */
/* binary16 conversions, written from the IEEE 754 binary16 format:          */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.                  */
/* ------------------------------------------------------------------------- */

double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 0x400), e - 25);    /* (1024+m) * 2^(e-15-10) */
    return sign ? -v : v;
}

float oracle_f16_to_f32(uint16_t h) { return (float)oracle_f16_to_f64(h); } /* exact */

/* Round a binary64 value to the nearest binary16, ties to even. */
uint16_t oracle_f64_to_f16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7e00;
    /* 65504 is the largest finite half; halfway to 2^16 is 65520, and a tie
       there goes to the even neighbour 2^16, i.e. overflows to infinity. */
    if (a >= 65520.0) return sign | 0x7c00;
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);            /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;           /* unbiased exponent: 2^E <= a < 2^(E+1) */
    if (E < -14) E = -14;     /* subnormal range shares the 2^-24 spacing */
    double ulp = ldexp(1.0, E - 10);
    double r = nearbyint(a / ulp);   /* a/ulp is exact (power-of-two scale) */
    /* r is an integer multiple count of ulp; r may equal 2048 (next binade). */
    long n = (long)r;
    uint16_t bits;
    if (E == -14 && n < 1024) {
        bits = (uint16_t)n;                          /* subnormal (or 0) */
    } else {
        if (n >= 2048) { n >>= 1; E += 1; }          /* carried into next binade */
        if (E > 15) return sign | 0x7c00;
        bits = (uint16_t)(((E + 15) << 10) | (n - 1024));
    }
    return sign | bits;
}

uint16_t oracle_f32_to_f16(float x) { return oracle_f64_to_f16((double)x); } /* float->double exact */

void oracle_f16_to_f64_array(const uint16_t *h, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++) out[i] = oracle_f16_to_f64(h[i]);
}

void oracle_f64_to_f16_array(const double *x, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++) out[i] = oracle_f64_to_f16(x[i]);
}

/* ------------------------------------------------------------------------- */
/* Group-wise 4-bit min-max quantisation [G3]                                 */
/* ------------------------------------------------------------------------- */

/*
 * One group of `group` (64 or 128) fp16 values x[i*xs] -> its codes, fp16 min and fp16 scale.
 * bits = 4: group/2 packed bytes codes[j*cs], byte j = code(2j) | code(2j+1) << 4;
 * bits = 8: group bytes codes[j*cs] = code(j).  With levels = 2^bits - 1 (15 or 255), the
 * steps, in this order, each one IEEE fp32 operation:
 *   1. mn = min(x), mx = max(x);  mn = mn + 0  (turns -0 into +0)
 *   2. d = mx - mn
 *   3. scale_h = fp16_rn(d / levels)
 *   4. scale_h == 0  ->  every code 0, stored scale +0
 *   5. inv = 1 / scale_h
 *   6. t = (x - mn) * inv    (two roundings, no fused multiply-add)
 *   7. code = clamp(round_half_even(t), 0, levels)
 *   8. min_h = fp16(mn)      (exact: mn is one of the fp16 inputs)
 * The 8-bit form is the same min-max scheme with 255 steps (INT8 next to INT4 among the
 * post-training formats the "Optimizing LLM for low memory usage" page lists).
 */
static void quantize_group_b(const uint16_t *x, ptrdiff_t xs, uint8_t *codes, ptrdiff_t cs,
                             uint16_t *min_out, uint16_t *scale_out, int group, int bits)
{
    const int levels = (1 << bits) - 1;
    float v[OR_GROUP_MAX];
    for (int i = 0; i < group; i++) v[i] = oracle_f16_to_f32(x[i * xs]);
    float mn = v[0], mx = v[0];
    for (int i = 1; i < group; i++) {
        if (v[i] < mn) mn = v[i];
        if (v[i] > mx) mx = v[i];
    }
    mn = mn + 0.0f;
    float d = mx - mn;
    float qd = d / (float)levels;
    uint16_t scale_h = oracle_f32_to_f16(qd);
    float s = oracle_f16_to_f32(scale_h);
    int q[OR_GROUP_MAX];
    if (s == 0.0f) {
        scale_h = 0;
        for (int i = 0; i < group; i++) q[i] = 0;
    } else {
        float inv = 1.0f / s;
        for (int i = 0; i < group; i++) {
            float diff = v[i] - mn;
            float t = diff * inv;
            float r = nearbyintf(t);          /* default mode: nearest, ties to even */
            int c = (int)r;
            if (c < 0) c = 0;
            if (c > levels) c = levels;
            q[i] = c;
        }
    }
    if (bits == 8) {
        for (int j = 0; j < group; j++) codes[j * cs] = (uint8_t)q[j];
    } else {
        for (int j = 0; j < group / 2; j++)
            codes[j * cs] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
    }
    *min_out = oracle_f32_to_f16(mn);
    *scale_out = scale_h;
}

static void quantize_group(const uint16_t *x, ptrdiff_t xs, uint8_t *codes, ptrdiff_t cs,
                           uint16_t *min_out, uint16_t *scale_out, int group)
{
    quantize_group_b(x, xs, codes, cs, min_out, scale_out, group, 4);
}

/* Dequantised value of one code: fp16_rn(mn + q*s), exact before the rounding
   (q*s has at most 19 significant bits -- a code of at most 8 bits times an fp16
   scale -- and every term is a multiple of 2^-24 below 2^25, so the float64 sum is
   exact). */
static uint16_t dequant_one(int q, uint16_t min_h, uint16_t scale_h)
{
    double s = oracle_f16_to_f64(scale_h);
    double m = oracle_f16_to_f64(min_h);
    return oracle_f64_to_f16((double)q * s + m);
}

static int group_ok(int group) { return group == 64 || group == 128; }
static int bits_ok(int bits) { return bits == 4 || bits == 8; }

/*
 * x viewed as [outer, n, inner]; groups of `group` (64 or 128) consecutive elements
 * along n.  codes: [outer, n/2, inner]   mins, scales: [outer, n/group, inner].
 * Returns 0, or -1 for another group size or n not a multiple of the group.
 */
/*
 * bits-bit codes (4 or 8): x viewed as [outer, n, inner]; groups of `group` consecutive
 * elements along n.  codes: [outer, n*bits/8, inner]   mins, scales: [outer, n/group, inner].
 * Returns 0, or -1 for another group size or width, or n not a multiple of the group.
 */
int oracle_quantize_gb(const uint16_t *x, int64_t outer, int64_t n, int64_t inner,
                       uint8_t *codes, uint16_t *mins, uint16_t *scales, int group, int bits)
{
    if (!group_ok(group) || !bits_ok(bits) || n % group) return -1;
    int64_t ng = n / group, nc = n * bits / 8, gc = group * bits / 8;
    for (int64_t o = 0; o < outer; o++)
        for (int64_t g = 0; g < ng; g++)
            for (int64_t i = 0; i < inner; i++) {
                const uint16_t *xp = x + (o * n + g * group) * inner + i;
                uint8_t *cp = codes + (o * nc + g * gc) * inner + i;
                int64_t m = (o * ng + g) * inner + i;
                quantize_group_b(xp, inner, cp, inner, &mins[m], &scales[m], group, bits);
            }
    return 0;
}

int oracle_quantize_g(const uint16_t *x, int64_t outer, int64_t n, int64_t inner,
                      uint8_t *codes, uint16_t *mins, uint16_t *scales, int group)
{
    return oracle_quantize_gb(x, outer, n, inner, codes, mins, scales, group, 4);
}

int oracle_quantize(const uint16_t *x, int64_t outer, int64_t n, int64_t inner,
                    uint8_t *codes, uint16_t *mins, uint16_t *scales)
{
    return oracle_quantize_g(x, outer, n, inner, codes, mins, scales, OR_GROUP);
}

int oracle_dequantize_gb(const uint8_t *codes, const uint16_t *mins, const uint16_t *scales,
                         int64_t outer, int64_t n, int64_t inner, uint16_t *y, int group, int bits)
{
    if (!group_ok(group) || !bits_ok(bits) || n % group) return -1;
    int64_t ng = n / group, nc = n * bits / 8;
    for (int64_t o = 0; o < outer; o++)
        for (int64_t e = 0; e < n; e++)
            for (int64_t i = 0; i < inner; i++) {
                int q;
                if (bits == 8) {
                    q = codes[(o * nc + e) * inner + i];
                } else {
                    uint8_t byte = codes[(o * nc + e / 2) * inner + i];
                    q = (e & 1) ? (byte >> 4) : (byte & 15);
                }
                int64_t m = (o * ng + e / group) * inner + i;
                y[(o * n + e) * inner + i] = dequant_one(q, mins[m], scales[m]);
            }
    return 0;
}

int oracle_dequantize_g(const uint8_t *codes, const uint16_t *mins, const uint16_t *scales,
                        int64_t outer, int64_t n, int64_t inner, uint16_t *y, int group)
{
    return oracle_dequantize_gb(codes, mins, scales, outer, n, inner, y, group, 4);
}

int oracle_dequantize(const uint8_t *codes, const uint16_t *mins, const uint16_t *scales,
                      int64_t outer, int64_t n, int64_t inner, uint16_t *y)
{
    return oracle_dequantize_g(codes, mins, scales, outer, n, inner, y, OR_GROUP);
}

/* ------------------------------------------------------------------------- */
/* OPT layer pieces, float64 [OPT]                                            */
/* ------------------------------------------------------------------------- */

/* y = (x - mean) / sqrt(var + eps) * gamma + beta, var the biased variance. */
static void layernorm_row(const double *x, int h, const double *g, const double *b, double eps, double *y)
{
    double mean = 0.0;
    for (int i = 0; i < h; i++) mean += x[i];
    mean /= h;
    double var = 0.0;
    for (int i = 0; i < h; i++) var += (x[i] - mean) * (x[i] - mean);
    var /= h;
    double rstd = 1.0 / sqrt(var + eps);
    for (int i = 0; i < h; i++) y[i] = (x[i] - mean) * rstd * g[i] + b[i];
}

/* y[n] = sum_k W[n][k] * x[k] + b[n]  (W row-major [N][K], PyTorch Linear orientation) */
static void linear_row(const float *W, const double *b, const double *x, int N, int K, double *y)
{
    for (int n = 0; n < N; n++) {
        const float *w = W + (int64_t)n * K;
        double acc = 0.0;
        for (int k = 0; k < K; k++) acc += (double)w[k] * x[k];
        y[n] = acc + (b ? b[n] : 0.0);
    }
}

/* Dequantise a [N][K] weight (groups along K) into float (exact for fp16 values). */
static float *dequant_weight(const uint8_t *codes, const uint16_t *mins, const uint16_t *scales, int N, int K,
                             int group)
{
    float *W = (float *)malloc(sizeof(float) * (size_t)N * K);
    if (!W) return NULL;
    int ng = K / group;
    for (int64_t n = 0; n < N; n++)
        for (int k = 0; k < K; k++) {
            uint8_t byte = codes[n * (K / 2) + k / 2];
            int q = (k & 1) ? (byte >> 4) : (byte & 15);
            int64_t m = n * ng + k / group;
            W[n * K + k] = (float)oracle_f16_to_f64(dequant_one(q, mins[m], scales[m]));
        }
    return W;
}

/* The fp16 value nearest to x, as a double (an activation stored in fp16). */
static double round16(double x) { return oracle_f16_to_f64(oracle_f64_to_f16(x)); }

static void round16_vec(double *v, int64_t n)
{
    for (int64_t i = 0; i < n; i++) v[i] = round16(v[i]);
}

static double *f16_vec(const uint16_t *h, int64_t n, double dflt)
{
    double *v = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; i++) v[i] = h ? oracle_f16_to_f64(h[i]) : dflt;
    return v;
}

/* y[m][n] = epilogue(sum_k x[m][k] * deq(W)[n][k] + b[n]) in float64.
   relu: max(0, .);  residual (fp16 [M][N]) added after the activation;
   the first qscale_cols outputs of each row are multiplied by qscale after the bias. */
int oracle_linear_g(const uint16_t *x, int M, int K,
                    const uint8_t *codes, const uint16_t *mins, const uint16_t *scales, int N,
                    const uint16_t *bias, const uint16_t *residual, int relu,
                    int qscale_cols, double qscale, double *y, int group)
{
    if (!group_ok(group) || K % group) return -1;
    float *W = dequant_weight(codes, mins, scales, N, K, group);
    double *b = f16_vec(bias, N, 0.0);
    double *xr = (double *)malloc(sizeof(double) * (size_t)K);
    if (!W || !b || !xr) return -2;
    for (int64_t m = 0; m < M; m++) {
        for (int k = 0; k < K; k++) xr[k] = oracle_f16_to_f64(x[m * K + k]);
        double *yr = y + m * N;
        linear_row(W, b, xr, N, K, yr);
        for (int n = 0; n < N; n++) {
            double v = yr[n];
            if (n < qscale_cols) v *= qscale;
            if (relu && v < 0.0) v = 0.0;
            if (residual) v += oracle_f16_to_f64(residual[m * N + n]);
            yr[n] = v;
        }
    }
    free(W); free(b); free(xr);
    return 0;
}

int oracle_linear(const uint16_t *x, int M, int K,
                  const uint8_t *codes, const uint16_t *mins, const uint16_t *scales, int N,
                  const uint16_t *bias, const uint16_t *residual, int relu,
                  int qscale_cols, double qscale, double *y)
{
    return oracle_linear_g(x, M, K, codes, mins, scales, N, bias, residual, relu, qscale_cols, qscale, y, OR_GROUP);
}

int oracle_layernorm(const uint16_t *x, int M, int h, const uint16_t *gamma, const uint16_t *beta,
                     double eps, double *y)
{
    double *g = f16_vec(gamma, h, 1.0), *b = f16_vec(beta, h, 0.0);
    double *xr = (double *)malloc(sizeof(double) * (size_t)h);
    for (int64_t m = 0; m < M; m++) {
        for (int i = 0; i < h; i++) xr[i] = oracle_f16_to_f64(x[m * h + i]);
        layernorm_row(xr, h, g, b, eps, y + m * h);
    }
    free(g); free(b); free(xr);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* 4-bit KV cache [G3]: per layer, for each (sequence, head, position) the    */
/* head_dim values are quantised in groups of 64 along head_dim.              */
/*   codes [S][H][maxL][d/2], mins/scales [S][H][maxL][d/64]                  */
/* ------------------------------------------------------------------------- */

typedef struct {
    uint8_t *kc; uint16_t *km, *ks;
    uint8_t *vc; uint16_t *vm, *vs;
    int S, H, d, maxL;
    int group;   /* 64 or 128 values of head_dim per group [G3] */
    int exact;   /* attention reads min + code * scale unrounded (1) or rounded to fp16 (0) */
} kv_t;

static void kv_store(const kv_t *kv, int s, int head, int pos, const uint16_t *k16, const uint16_t *v16)
{
    int64_t slot = ((int64_t)s * kv->H + head) * kv->maxL + pos;
    int G = kv->group, ng = kv->d / G;
    for (int g = 0; g < ng; g++) {
        quantize_group(k16 + g * G, 1, kv->kc + slot * (kv->d / 2) + g * (G / 2), 1,
                       &kv->km[slot * ng + g], &kv->ks[slot * ng + g], G);
        quantize_group(v16 + g * G, 1, kv->vc + slot * (kv->d / 2) + g * (G / 2), 1,
                       &kv->vm[slot * ng + g], &kv->vs[slot * ng + g], G);
    }
}

static void kv_load(const uint8_t *c, const uint16_t *mn, const uint16_t *sc, int64_t slot, int d, int G,
                    int exact, double *out)
{
    int ng = d / G;
    for (int i = 0; i < d; i++) {
        uint8_t byte = c[slot * (d / 2) + i / 2];
        int q = (i & 1) ? (byte >> 4) : (byte & 15);
        int64_t m = slot * ng + i / G;
        if (exact)  /* min + q * scale is exact in float64 (see dequant_one) */
            out[i] = oracle_f16_to_f64(mn[m]) + (double)q * oracle_f16_to_f64(sc[m]);
        else
            out[i] = oracle_f16_to_f64(dequant_one(q, mn[m], sc[m]));
    }
}

/* Append fp16 k, v rows [R][H*d] (row stride ld) at positions pos_of_row[r] of
   sequence seq_of_row[r]; head_dim quantised in groups of `group` (64 or 128). */
int oracle_kv_append_g(const uint16_t *k, const uint16_t *v, int64_t ld, int R,
                       const int *seq_of_row, const int *pos_of_row,
                       uint8_t *kc, uint16_t *km, uint16_t *ks, uint8_t *vc, uint16_t *vm, uint16_t *vs,
                       int S, int H, int d, int maxL, int group)
{
    if (!group_ok(group) || d % group) return -1;
    kv_t kv = {kc, km, ks, vc, vm, vs, S, H, d, maxL, group, 0};
    for (int r = 0; r < R; r++) {
        if (pos_of_row[r] < 0 || pos_of_row[r] >= maxL || seq_of_row[r] < 0 || seq_of_row[r] >= S) return -2;
        for (int hd = 0; hd < H; hd++)
            kv_store(&kv, seq_of_row[r], hd, pos_of_row[r], k + (int64_t)r * ld + hd * d, v + (int64_t)r * ld + hd * d);
    }
    return 0;
}

int oracle_kv_append(const uint16_t *k, const uint16_t *v, int64_t ld, int R,
                     const int *seq_of_row, const int *pos_of_row,
                     uint8_t *kc, uint16_t *km, uint16_t *ks, uint8_t *vc, uint16_t *vm, uint16_t *vs,
                     int S, int H, int d, int maxL)
{
    return oracle_kv_append_g(k, v, ld, R, seq_of_row, pos_of_row, kc, km, ks, vc, vm, vs, S, H, d, maxL, OR_GROUP);
}

/* Softmax attention of one query head over cached positions 0..L-1:
   p_j = exp(q.K_j - max) / sum, o = sum_j p_j V_j   (q already scaled). */
static void attend_head(const kv_t *kv, int s, int head, int L, const double *q, double *o, double *kbuf, double *scores)
{
    int d = kv->d;
    int64_t base = ((int64_t)s * kv->H + head) * kv->maxL;
    double mx = -INFINITY;
    for (int j = 0; j < L; j++) {
        kv_load(kv->kc, kv->km, kv->ks, base + j, d, kv->group, kv->exact, kbuf);
        double acc = 0.0;
        for (int i = 0; i < d; i++) acc += q[i] * kbuf[i];
        scores[j] = acc;
        if (acc > mx) mx = acc;
    }
    double sum = 0.0;
    for (int j = 0; j < L; j++) { scores[j] = exp(scores[j] - mx); sum += scores[j]; }
    for (int i = 0; i < d; i++) o[i] = 0.0;
    for (int j = 0; j < L; j++) {
        kv_load(kv->vc, kv->vm, kv->vs, base + j, d, kv->group, kv->exact, kbuf);
        double p = scores[j] / sum;
        for (int i = 0; i < d; i++) o[i] += p * kbuf[i];
    }
}

/* q: fp16 rows [R][H*d] (row stride ld); each row attends over positions
   0..len_of_row[r]-1 of sequence seq_of_row[r].  out: float64 [R][H*d].
   exact = 0: K and V are the dequantised fp16 values (the layer's reading);
   exact = 1: K and V are min + code * scale before that rounding (the decode
   kernel's reading: it never forms the fp16 value). */
int oracle_attention_x(const uint16_t *q16, int64_t ld, int R, const int *seq_of_row, const int *len_of_row,
                       const uint8_t *kc, const uint16_t *km, const uint16_t *ks,
                       const uint8_t *vc, const uint16_t *vm, const uint16_t *vs,
                       int S, int H, int d, int maxL, double *out, int group, int exact)
{
    if (!group_ok(group) || d % group) return -1;
    kv_t kv = {(uint8_t *)kc, (uint16_t *)km, (uint16_t *)ks, (uint8_t *)vc, (uint16_t *)vm, (uint16_t *)vs, S, H, d, maxL,
               group, exact ? 1 : 0};
    double *q = malloc(sizeof(double) * d), *kb = malloc(sizeof(double) * d);
    double *sc = malloc(sizeof(double) * (maxL > 0 ? maxL : 1));
    for (int r = 0; r < R; r++) {
        if (len_of_row[r] < 1 || len_of_row[r] > maxL) { free(q); free(kb); free(sc); return -2; }
        for (int hd = 0; hd < H; hd++) {
            for (int i = 0; i < d; i++) q[i] = oracle_f16_to_f64(q16[(int64_t)r * ld + hd * d + i]);
            attend_head(&kv, seq_of_row[r], hd, len_of_row[r], q, out + (int64_t)r * H * d + hd * d, kb, sc);
        }
    }
    free(q); free(kb); free(sc);
    return 0;
}

int oracle_attention_g(const uint16_t *q16, int64_t ld, int R, const int *seq_of_row, const int *len_of_row,
                       const uint8_t *kc, const uint16_t *km, const uint16_t *ks,
                       const uint8_t *vc, const uint16_t *vm, const uint16_t *vs,
                       int S, int H, int d, int maxL, double *out, int group)
{
    return oracle_attention_x(q16, ld, R, seq_of_row, len_of_row, kc, km, ks, vc, vm, vs, S, H, d, maxL, out, group, 0);
}

int oracle_attention(const uint16_t *q16, int64_t ld, int R, const int *seq_of_row, const int *len_of_row,
                     const uint8_t *kc, const uint16_t *km, const uint16_t *ks,
                     const uint8_t *vc, const uint16_t *vm, const uint16_t *vs,
                     int S, int H, int d, int maxL, double *out)
{
    return oracle_attention_g(q16, ld, R, seq_of_row, len_of_row, kc, km, ks, vc, vm, vs, S, H, d, maxL, out, OR_GROUP);
}

/* ------------------------------------------------------------------------- */
/* One OPT decoder layer, row by row [OPT][G3][G2]                            */
/* ------------------------------------------------------------------------- */

/* W4A8 pieces defined with the W4A8 section at the end of this file */
#define OR_W8_BOUND 113
#define OR_A8_BOUND 127
static void quantize_row_sym8(const uint16_t *x, int64_t n, int bound, int *q, float *scale);
int oracle_w4a8_weight_int8(const uint8_t *codes, const int8_t *gmin, const uint8_t *gstep, int N, int K,
                            int8_t *w8);

typedef struct {
    int h, H, d, F;
    double eps;
    float *Wqkv, *Wo, *W1, *W2;           /* dequantised, [out][in] (W4A16) */
    int w4a8;                             /* 1: the W4A8 products of the W4A8 section */
    int8_t *Q[4];                         /* W4A8: the products' int8 weights, [out][in] */
    const float *cs[4];                   /* W4A8: their row scales */
    double *bqkv, *bo, *b1, *b2, *g1, *be1, *g2, *be2;
    kv_t kv;
    const uint16_t *x;                    /* [R][h] */
    const int *seq_of_row, *pos_of_row;
    int R, kv_only, nthreads;
    double *out, *attn;                   /* [R][h] each (attn may be NULL) */
} layer_ctx;

typedef struct { layer_ctx *c; int tid; } layer_job;

/* y = x W^T + b for one row of one of the layer's matrices (0 wqkv, 1 wo, 2 w1, 3 w2): float64
   from the dequantised fp16 weights, or (W4A8) the row's fp16 values quantised to int8 with one
   fp32 scale, exact integer sums with the int8 weights, then acc * (ascale * cscale[n]) + b[n]
   in float64.  x16 and q hold K values of scratch. */
static void layer_linear(const layer_ctx *c, int which, const double *x, int N, int K, const double *b,
                         double *y, uint16_t *x16, int *q)
{
    if (!c->w4a8) {
        const float *W[4] = {c->Wqkv, c->Wo, c->W1, c->W2};
        linear_row(W[which], b, x, N, K, y);
        return;
    }
    for (int k = 0; k < K; k++) x16[k] = oracle_f64_to_f16(x[k]);   /* exact: x holds fp16 values */
    float as;
    quantize_row_sym8(x16, K, OR_A8_BOUND, q, &as);
    const int8_t *W = c->Q[which];
    const float *cs = c->cs[which];
    for (int n = 0; n < N; n++) {
        const int8_t *wr = W + (int64_t)n * K;
        int64_t acc = 0;
        for (int k = 0; k < K; k++) acc += (int64_t)q[k] * (int64_t)wr[k];
        y[n] = (double)acc * ((double)as * (double)cs[n]) + (b ? b[n] : 0.0);
    }
}

/* The rows of one sequence are processed in the order given, so a prompt
   (positions 0..P-1) appends each token before the next one attends. */
static void *layer_worker(void *arg)
{
    layer_job *job = (layer_job *)arg;
    layer_ctx *c = job->c;
    int h = c->h, H = c->H, d = c->d, F = c->F;
    double *x = malloc(sizeof(double) * h), *a = malloc(sizeof(double) * h);
    double *qkv = malloc(sizeof(double) * 3 * h), *o = malloc(sizeof(double) * h);
    double *h1 = malloc(sizeof(double) * h), *a2 = malloc(sizeof(double) * h);
    double *f = malloc(sizeof(double) * F), *y = malloc(sizeof(double) * h);
    double *tmp = malloc(sizeof(double) * h), *kb = malloc(sizeof(double) * d);
    double *sc = malloc(sizeof(double) * c->kv.maxL);
    uint16_t *k16 = malloc(sizeof(uint16_t) * d), *v16 = malloc(sizeof(uint16_t) * d);
    int KX = F > h ? F : h;
    uint16_t *x16 = malloc(sizeof(uint16_t) * KX);
    int *q8 = malloc(sizeof(int) * KX);
    double qscale = 1.0 / sqrt((double)d);
    for (int r = 0; r < c->R; r++) {
        int s = c->seq_of_row[r], pos = c->pos_of_row[r];
        if (s % c->nthreads != job->tid) continue;
        for (int i = 0; i < h; i++) x[i] = oracle_f16_to_f64(c->x[(int64_t)r * h + i]);
        /* 1. a = fp16(LN1(x)) */
        layernorm_row(x, h, c->g1, c->be1, c->eps, a);
        round16_vec(a, h);
        /* 2. [q k v] = a Wqkv^T + b;  q = fp16(q * d^-1/2), k = fp16(k), v = fp16(v) */
        layer_linear(c, 0, a, 3 * h, h, c->bqkv, qkv, x16, q8);
        for (int i = 0; i < h; i++) qkv[i] *= qscale;
        round16_vec(qkv, 3 * h);
        /* 3. append k, v to the 4-bit cache at pos */
        for (int hd = 0; hd < H; hd++) {
            for (int i = 0; i < d; i++) {
                k16[i] = oracle_f64_to_f16(qkv[h + hd * d + i]);
                v16[i] = oracle_f64_to_f16(qkv[2 * h + hd * d + i]);
            }
            kv_store(&c->kv, s, hd, pos, k16, v16);
        }
        if (c->kv_only) continue;
        /* 4-5. o = fp16(attention of each head over cached positions 0..pos) */
        for (int hd = 0; hd < H; hd++)
            attend_head(&c->kv, s, hd, pos + 1, qkv + hd * d, o + hd * d, kb, sc);
        round16_vec(o, h);
        if (c->attn) memcpy(c->attn + (int64_t)r * h, o, sizeof(double) * h);
        /* 6. h1 = fp16(x + o Wo^T + bo) */
        layer_linear(c, 1, o, h, h, c->bo, tmp, x16, q8);
        for (int i = 0; i < h; i++) h1[i] = round16(x[i] + tmp[i]);
        /* 7. y = h1 + fp16(relu(fp16(LN2(h1)) W1^T + b1)) W2^T + b2 */
        layernorm_row(h1, h, c->g2, c->be2, c->eps, a2);
        round16_vec(a2, h);
        layer_linear(c, 2, a2, F, h, c->b1, f, x16, q8);
        for (int i = 0; i < F; i++) f[i] = f[i] < 0.0 ? 0.0 : round16(f[i]);
        layer_linear(c, 3, f, h, F, c->b2, tmp, x16, q8);
        for (int i = 0; i < h; i++) y[i] = h1[i] + tmp[i];
        memcpy(c->out + (int64_t)r * h, y, sizeof(double) * h);
    }
    free(x); free(a); free(qkv); free(o); free(h1); free(a2); free(f); free(y); free(tmp); free(kb); free(sc);
    free(k16); free(v16); free(x16); free(q8);
    return NULL;
}

/* The rows of the layer over nthreads threads (rows of one sequence stay on one thread). */
static void run_layer_threads(layer_ctx *c, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    c->nthreads = nthreads;
    pthread_t *th = malloc(sizeof(pthread_t) * nthreads);
    layer_job *jobs = malloc(sizeof(layer_job) * nthreads);
    for (int t = 0; t < nthreads; t++) {
        jobs[t].c = c; jobs[t].tid = t;
        if (t > 0) pthread_create(&th[t], NULL, layer_worker, &jobs[t]);
    }
    layer_worker(&jobs[0]);
    for (int t = 1; t < nthreads; t++) pthread_join(th[t], NULL);
    free(th); free(jobs);
}

/*
 * dims = {hidden, heads, head_dim, ffn, group}.  Weights as packed 4-bit tensors
 * quantised along the input dim in groups of `group` (64 or 128; the KV cache
 * uses the same group along head_dim): wqkv [3h][h], wo [h][h], w1 [F][h],
 * w2 [h][F] (codes, mins, scales each); biases and LayerNorm parameters fp16
 * (NULL = 0, gamma NULL = 1).  The KV cache arrays are read and written in
 * place.  kv_only = 1 stops after step 3 (cache fill for prompts).
 */
int oracle_layer_rows(const int *dims, double eps,
                      const uint8_t *qkv_c, const uint16_t *qkv_m, const uint16_t *qkv_s, const uint16_t *bqkv,
                      const uint8_t *o_c, const uint16_t *o_m, const uint16_t *o_s, const uint16_t *bo,
                      const uint8_t *f1_c, const uint16_t *f1_m, const uint16_t *f1_s, const uint16_t *b1,
                      const uint8_t *f2_c, const uint16_t *f2_m, const uint16_t *f2_s, const uint16_t *b2,
                      const uint16_t *ln1_g, const uint16_t *ln1_b, const uint16_t *ln2_g, const uint16_t *ln2_b,
                      uint8_t *kc, uint16_t *km, uint16_t *ks, uint8_t *vc, uint16_t *vm, uint16_t *vs,
                      int S, int maxL,
                      const uint16_t *x, int R, const int *seq_of_row, const int *pos_of_row,
                      int kv_only, double *out, double *attn, int nthreads)
{
    layer_ctx c;
    memset(&c, 0, sizeof(c));
    c.h = dims[0]; c.H = dims[1]; c.d = dims[2]; c.F = dims[3]; c.eps = eps;
    int G = dims[4];
    if (!group_ok(G) || c.h != c.H * c.d || c.h % G || c.F % G || c.d % G) return -1;
    for (int r = 0; r < R; r++)
        if (seq_of_row[r] < 0 || seq_of_row[r] >= S || pos_of_row[r] < 0 || pos_of_row[r] >= maxL) return -2;
    c.Wqkv = dequant_weight(qkv_c, qkv_m, qkv_s, 3 * c.h, c.h, G);
    c.Wo = kv_only ? NULL : dequant_weight(o_c, o_m, o_s, c.h, c.h, G);
    c.W1 = kv_only ? NULL : dequant_weight(f1_c, f1_m, f1_s, c.F, c.h, G);
    c.W2 = kv_only ? NULL : dequant_weight(f2_c, f2_m, f2_s, c.h, c.F, G);
    c.bqkv = f16_vec(bqkv, 3 * c.h, 0.0); c.bo = f16_vec(bo, c.h, 0.0);
    c.b1 = f16_vec(b1, c.F, 0.0); c.b2 = f16_vec(b2, c.h, 0.0);
    c.g1 = f16_vec(ln1_g, c.h, 1.0); c.be1 = f16_vec(ln1_b, c.h, 0.0);
    c.g2 = f16_vec(ln2_g, c.h, 1.0); c.be2 = f16_vec(ln2_b, c.h, 0.0);
    kv_t kv = {kc, km, ks, vc, vm, vs, S, c.H, c.d, maxL, G, 0};
    c.kv = kv;
    c.x = x; c.seq_of_row = seq_of_row; c.pos_of_row = pos_of_row; c.R = R;
    c.kv_only = kv_only; c.out = out; c.attn = attn;
    run_layer_threads(&c, nthreads);
    free(c.Wqkv); free(c.Wo); free(c.W1); free(c.W2);
    free(c.bqkv); free(c.bo); free(c.b1); free(c.b2); free(c.g1); free(c.be1); free(c.g2); free(c.be2);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* W4A8: 4-bit weights, 8-bit activations, integer products                  */
/* ------------------------------------------------------------------------- */
/*
 * What it follows: the W4A8KV4 entry (QServe) in the PIPO paper's list of references,
 * by its title only; the "Optimizing LLM for low memory usage" page, section
 * "Quantization and Weight Compression" (weights mapped to INT8 or INT4); [G3] for the
 * groups of 64 along the input dimension.  The pages give no scheme, so this is the
 * reading (listed with the others in the design notes):
 *
 * Weights [N][K], two levels:
 *   1. per output row n: amax = max_k |w|; amax == 0 -> cscale = 0, every w8 = 0; else
 *      inv = 113 / amax and cscale = amax / 113 (each one fp32 division),
 *      w8 = clamp(round_half_even(w * inv), -113, 113)  (one fp32 multiply);
 *   2. per group of 64 along k, in the integer domain: mn = min w8, mx = max w8,
 *      step = max(1, ceil((mx - mn) / 15)), code = floor((2 (w8 - mn) + step) / (2 step))
 *      (nearest, halves up; at most 15 because mx - mn <= 15 step), two codes per byte,
 *      even element in the low nibble; gmin = mn (int8), gstep = step (uint8, 1..16).
 *   The 8-bit weight the product uses is mn + code * step.  113 is the largest bound for
 *   which that value stays in int8 whatever the group: mn + 15 step <= mx + 14 <= 127.
 * Activations [M][K], per row t: amax = max_k |x|; amax == 0 -> ascale = 0, a8 = 0; else
 *   inv = 127 / amax, ascale = amax / 127, a8 = clamp(round_half_even(x * inv), -127, 127),
 *   the same fp32 operations as level 1.
 * Product: acc[t][n] = sum_k a8[t][k] * (mn + code * step)[n][k], exact (int64 here);
 *   y = acc * (ascale[t] * cscale[n]) + bias[n], then the q-scale of the first qscale_cols
 *   outputs, ReLU and the fp16 residual as in oracle_linear, in float64.
 */
/* round-half-even of x * inv (fp32 multiply), clamped to [-bound, bound] */
static int q8_of(float x, float inv, int bound)
{
    float t = x * inv;
    int c = (int)nearbyintf(t);
    if (c < -bound) c = -bound;
    if (c > bound) c = bound;
    return c;
}

/* One row of n fp16 values -> symmetric 8-bit codes and the row's fp32 scale. */
static void quantize_row_sym8(const uint16_t *x, int64_t n, int bound, int *q, float *scale)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < n; k++) {
        float a = fabsf(oracle_f16_to_f32(x[k]));
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *scale = 0.0f;
        for (int64_t k = 0; k < n; k++) q[k] = 0;
        return;
    }
    float inv = (float)bound / amax;
    *scale = amax / (float)bound;
    for (int64_t k = 0; k < n; k++) q[k] = q8_of(oracle_f16_to_f32(x[k]), inv, bound);
}

int oracle_w4a8_quantize_weight(const uint16_t *w, int N, int K, uint8_t *codes, int8_t *gmin,
                                uint8_t *gstep, float *cscale)
{
    if (N < 0 || K <= 0 || K % OR_GROUP) return -1;
    int *w8 = (int *)malloc(sizeof(int) * (size_t)K);
    if (!w8) return -2;
    int ng = K / OR_GROUP;
    for (int64_t n = 0; n < N; n++) {
        quantize_row_sym8(w + n * K, K, OR_W8_BOUND, w8, &cscale[n]);
        for (int g = 0; g < ng; g++) {
            const int *v = w8 + g * OR_GROUP;
            int mn = v[0], mx = v[0];
            for (int i = 1; i < OR_GROUP; i++) {
                if (v[i] < mn) mn = v[i];
                if (v[i] > mx) mx = v[i];
            }
            int step = (mx - mn + 14) / 15;
            if (step < 1) step = 1;
            uint8_t *cp = codes + n * (K / 2) + g * (OR_GROUP / 2);
            for (int j = 0; j < OR_GROUP / 2; j++) {
                int c0 = (2 * (v[2 * j] - mn) + step) / (2 * step);
                int c1 = (2 * (v[2 * j + 1] - mn) + step) / (2 * step);
                cp[j] = (uint8_t)(c0 | (c1 << 4));
            }
            gmin[n * ng + g] = (int8_t)mn;
            gstep[n * ng + g] = (uint8_t)step;
        }
    }
    free(w8);
    return 0;
}

/* The 8-bit weights the product uses: w8[n][k] = gmin + code * gstep. */
int oracle_w4a8_weight_int8(const uint8_t *codes, const int8_t *gmin, const uint8_t *gstep, int N, int K,
                            int8_t *w8)
{
    if (N < 0 || K <= 0 || K % OR_GROUP) return -1;
    int ng = K / OR_GROUP;
    for (int64_t n = 0; n < N; n++)
        for (int k = 0; k < K; k++) {
            uint8_t byte = codes[n * (K / 2) + k / 2];
            int q = (k & 1) ? (byte >> 4) : (byte & 15);
            int64_t g = n * ng + k / OR_GROUP;
            int v = gmin[g] + q * gstep[g];
            if (v < -128 || v > 127) return -3;   /* cannot happen for weights quantised above */
            w8[n * K + k] = (int8_t)v;
        }
    return 0;
}

int oracle_act8_quantize(const uint16_t *x, int M, int K, int8_t *a8, float *ascale)
{
    if (M < 0 || K <= 0) return -1;
    int *q = (int *)malloc(sizeof(int) * (size_t)K);
    if (!q) return -2;
    for (int64_t t = 0; t < M; t++) {
        quantize_row_sym8(x + t * K, K, OR_A8_BOUND, q, &ascale[t]);
        for (int k = 0; k < K; k++) a8[t * K + k] = (int8_t)q[k];
    }
    free(q);
    return 0;
}

/* y[t][n] in float64; acc_out (optional) receives the exact integer sums [M][N]. */
int oracle_linear_w4a8(const int8_t *a8, const float *ascale, int M, int K,
                       const uint8_t *codes, const int8_t *gmin, const uint8_t *gstep, const float *cscale, int N,
                       const uint16_t *bias, const uint16_t *residual, int relu, int qscale_cols, double qscale,
                       double *y, int64_t *acc_out)
{
    if (M < 0 || N < 0 || K <= 0 || K % OR_GROUP) return -1;
    int8_t *W = (int8_t *)malloc((size_t)N * K + 1);
    if (!W) return -2;
    if (oracle_w4a8_weight_int8(codes, gmin, gstep, N, K, W)) { free(W); return -3; }
    for (int64_t t = 0; t < M; t++)
        for (int64_t n = 0; n < N; n++) {
            const int8_t *ar = a8 + t * K, *wr = W + n * K;
            int64_t acc = 0;
            for (int k = 0; k < K; k++) acc += (int64_t)ar[k] * (int64_t)wr[k];
            if (acc_out) acc_out[t * N + n] = acc;
            double v = (double)acc * ((double)ascale[t] * (double)cscale[n]);
            if (bias) v += oracle_f16_to_f64(bias[n]);
            if (n < qscale_cols) v *= qscale;
            if (relu && v < 0.0) v = 0.0;
            if (residual) v += oracle_f16_to_f64(residual[t * N + n]);
            y[t * N + n] = v;
        }
    free(W);
    return 0;
}

/*
 * The OPT layer with W4A8 products ([Q8] reading above): the layer of oracle_layer_rows with each
 * of its four products replaced by the W4A8 product of its fp16 input row (LayerNorm outputs, the
 * attention output, the ReLU output), everything else unchanged (the KV cache in groups of 64).
 * mats[4 * i + j], i = wqkv, wo, w1, w2: j = 0 codes [N][K/2], 1 gmin [N][K/64] (int8), 2 gstep
 * [N][K/64] (uint8), 3 cscale [N] (float).  dims = {hidden, heads, head_dim, ffn}.
 */
int oracle_layer_rows_w4a8(const int *dims, double eps, const void *const *mats,
                           const uint16_t *bqkv, const uint16_t *bo, const uint16_t *b1, const uint16_t *b2,
                           const uint16_t *ln1_g, const uint16_t *ln1_b, const uint16_t *ln2_g, const uint16_t *ln2_b,
                           uint8_t *kc, uint16_t *km, uint16_t *ks, uint8_t *vc, uint16_t *vm, uint16_t *vs,
                           int S, int maxL,
                           const uint16_t *x, int R, const int *seq_of_row, const int *pos_of_row,
                           int kv_only, double *out, double *attn, int nthreads)
{
    layer_ctx c;
    memset(&c, 0, sizeof(c));
    c.h = dims[0]; c.H = dims[1]; c.d = dims[2]; c.F = dims[3]; c.eps = eps;
    if (c.h != c.H * c.d || c.h % OR_GROUP || c.F % OR_GROUP || c.d % OR_GROUP) return -1;
    for (int r = 0; r < R; r++)
        if (seq_of_row[r] < 0 || seq_of_row[r] >= S || pos_of_row[r] < 0 || pos_of_row[r] >= maxL) return -2;
    const int NK[4][2] = {{3 * c.h, c.h}, {c.h, c.h}, {c.F, c.h}, {c.h, c.F}};
    c.w4a8 = 1;
    for (int i = 0; i < 4; i++) {
        c.Q[i] = (int8_t *)malloc((size_t)NK[i][0] * NK[i][1]);
        if (!c.Q[i]) return -3;
        if (oracle_w4a8_weight_int8((const uint8_t *)mats[4 * i], (const int8_t *)mats[4 * i + 1],
                                    (const uint8_t *)mats[4 * i + 2], NK[i][0], NK[i][1], c.Q[i]))
            return -4;
        c.cs[i] = (const float *)mats[4 * i + 3];
    }
    c.bqkv = f16_vec(bqkv, 3 * c.h, 0.0); c.bo = f16_vec(bo, c.h, 0.0);
    c.b1 = f16_vec(b1, c.F, 0.0); c.b2 = f16_vec(b2, c.h, 0.0);
    c.g1 = f16_vec(ln1_g, c.h, 1.0); c.be1 = f16_vec(ln1_b, c.h, 0.0);
    c.g2 = f16_vec(ln2_g, c.h, 1.0); c.be2 = f16_vec(ln2_b, c.h, 0.0);
    kv_t kv = {kc, km, ks, vc, vm, vs, S, c.H, c.d, maxL, OR_GROUP, 0};
    c.kv = kv;
    c.x = x; c.seq_of_row = seq_of_row; c.pos_of_row = pos_of_row; c.R = R;
    c.kv_only = kv_only; c.out = out; c.attn = attn;
    run_layer_threads(&c, nthreads);
    for (int i = 0; i < 4; i++) free(c.Q[i]);
    free(c.bqkv); free(c.bo); free(c.b1); free(c.b2); free(c.g1); free(c.be1); free(c.g2); free(c.be2);
    return 0;
}
