/*
 * awq_oracle.c -- plain, slow, obviously-correct CPU oracle for the AWQ
 * per-layer activation-aware scale search.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may load,
 * call or link this file.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA path.
 *
 * Sources (each function names the passage it follows):
 *   [P1] compassingai.com, "AWQ (Activation-aware Weight Quantization)" concept
 *        page: "quantisation math" section (absmax symmetric b-bit group
 *        quantiser), "statistical basis of salient channels" (activation_scale
 *        = mean|X| or max), "full scale-optimisation flow" steps 1-6.
 *   [P2] mudrobot.github.io, AWQ paper notes: "analysing the quantisation
 *        error" (Q(w) = delta * Round(w / delta)) and "searching the optimal
 *        scale" (L(s) = ||Q(W diag(s)) (diag(s)^-1 X) - W X||, s = s_X^alpha).
 *
 * Precision: the statistic and the loss are computed in fp64 (the loss via
 * explicit loops, no BLAS).  The quantiser is defined on fp32 values with
 * every operation correctly rounded (IEEE single, no contraction): that is the
 * only reading under which "identical INT4 codes" is well defined.  Build with
 * -O2 -fno-fast-math -ffp-contract=off.
 *
 * Readings taken where the pages are silent (see the design notes):
 *   - delta = max|w| / (2^(b-1) - 1) with the clamp to +-(2^(b-1) - 1) of P1;
 *     P2's max|w| / 2^(N-1) is a variant, not used here.
 *   - round = round-half-to-even (IEEE default).
 *   - an all-zero group has delta = 0 and all codes 0.
 *   - a_j is floored at 1e-6 * max_j a_j (fp32 product) so that a dead channel
 *     does not make S^-1 infinite; if every a_j is 0 the scales are all 1.
 *   - s_j = (float) pow((double) a_j, (double) alpha).
 *   - codes are stored offset-binary u = q + 2^(b-1), eight per 32-bit word,
 *     nibble i (bits 4i..4i+3) = row 8*k8 + i of the column.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_STAT_MEAN 0
#define ORACLE_STAT_MAX 1

static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* [P1] "statistical basis of salient channels": for every input channel j,
 * activation_scale[j] = mean_i |X[i, j]| (or max_i |X[i, j]|).  [P2] "searching
 * the optimal scale": s_X is the per-channel average activation magnitude. */
void oracle_act_stats(const uint16_t *X, int64_t N, int64_t D, int stat, double *a)
{
    for (int64_t j = 0; j < D; ++j)
        a[j] = 0.0;
    for (int64_t i = 0; i < N; ++i) {
        const uint16_t *row = X + i * D;
        for (int64_t j = 0; j < D; ++j) {
            double v = fabs(bf16_bits_to_double(row[j]));
            if (stat == ORACLE_STAT_MAX) {
                if (v > a[j])
                    a[j] = v;
            } else {
                a[j] += v;
            }
        }
    }
    if (stat != ORACLE_STAT_MAX && N > 0)
        for (int64_t j = 0; j < D; ++j)
            a[j] /= (double)N;
}

/* [P1] flow step 3: s_j(alpha) = activation_scale[j]^alpha.  [P2]: s = s_X^alpha.
 * Floor reading: see the header. */
void oracle_scales(const float *a, int64_t D, float alpha, float *s)
{
    float amax = 0.0f;
    for (int64_t j = 0; j < D; ++j)
        if (a[j] > amax)
            amax = a[j];
    const float floor_ = 1e-6f * amax;
    for (int64_t j = 0; j < D; ++j) {
        float aj;
        if (amax == 0.0f)
            aj = 1.0f;
        else
            aj = a[j] > floor_ ? a[j] : floor_;
        s[j] = (float)pow((double)aj, (double)alpha);
    }
}

/* The weight statistic of the balanced scale ([P3] "the scale per channel":
 * s_j = mean|X_j|^alpha / mean|W_j|^(1-alpha)): w_mean_j = (sum_n |W_jn|) / D_out
 * over input channel j's row of W, summed in fp64, rounded to fp32 once. */
void oracle_weight_mean(const float *W, int64_t D_in, int64_t D_out, float *w_mean)
{
    for (int64_t j = 0; j < D_in; ++j) {
        double acc = 0.0;
        for (int64_t n = 0; n < D_out; ++n)
            acc += fabs((double)W[j * D_out + n]);
        w_mean[j] = (float)(acc / (double)D_out);
    }
}

/* The balanced scale s_j = a_j^alpha / b_j^(1-alpha) ([P3], same passage), with
 * a and b each floored as in oracle_scales (1e-6 of its maximum; all zero ->
 * 1).  Computed in fp64, rounded to fp32 once. */
void oracle_scales_balanced(const float *a, const float *b, int64_t D, float alpha, float *s)
{
    float amax = 0.0f, bmax = 0.0f;
    for (int64_t j = 0; j < D; ++j) {
        if (a[j] > amax)
            amax = a[j];
        if (b[j] > bmax)
            bmax = b[j];
    }
    const float afl = 1e-6f * amax, bfl = 1e-6f * bmax;
    for (int64_t j = 0; j < D; ++j) {
        const float aj = amax == 0.0f ? 1.0f : (a[j] > afl ? a[j] : afl);
        const float bj = bmax == 0.0f ? 1.0f : (b[j] > bfl ? b[j] : bfl);
        s[j] = (float)(pow((double)aj, (double)alpha) / pow((double)bj, 1.0 - (double)alpha));
    }
}

/* Round a finite fp32 value to the nearest IEEE binary16 value (ties to
 * even), returned as a float: 11 significant bits in the normal range
 * (|x| >= 2^-14), a fixed step of 2^-24 below it, infinity from 65520 up
 * ([P2] "analysing the quantisation error": delta stored in FP16). */
static float round_to_fp16(float x)
{
    double ax = fabs((double)x);
    if (ax >= 65520.0)
        return x > 0 ? INFINITY : -INFINITY;
    if (ax == 0.0)
        return x;
    int e;
    frexp(ax, &e);                 /* ax = f * 2^e, f in [0.5, 1): the binade is 2^(e-1) */
    int ulp_exp = (e - 1) - 10;    /* 10 fraction bits */
    if (ulp_exp < -24)
        ulp_exp = -24;             /* subnormal step */
    const double ulp = ldexp(1.0, ulp_exp);
    const double r = nearbyint(ax / ulp) * ulp;   /* exact scaling; round half to even */
    return (float)(x < 0 ? -r : r);
}

/* [P1] "quantisation math", steps 1-3, applied to one group of one column of
 * W' = diag(s) W ([P1] flow step 4a):
 *   w'_k  = fl32(s_k * w_k)
 *   delta = fl32(max_k |w'_k| / (2^(b-1) - 1))
 *   q_k   = clamp(round(fl32(w'_k / delta)), -(2^(b-1)-1), 2^(b-1)-1)
 * s == NULL means s_k = 1 (no scaling).  clip is the weight-clipping ratio
 * ([P2] "searching the optimal scale": weight clipping to minimise the
 * quantisation MSE): the group maximum m is replaced by fl32(clip * m) before
 * delta is formed, and the clamp then bounds the codes of the clipped weights.
 * clip = 1 leaves m unchanged (fl32(1 * m) = m). */
/* qmode 2, the asymmetric (MinMax, zero-point) quantiser ([P1] "the AWQ
 * mechanism": absmax or MinMax uniform quantisation; "symmetric or asymmetric
 * both work"), with the plainest textbook reading of MinMax:
 *   lo = min(0, min_k w'_k),  hi = max(0, max_k w'_k)   (zero stays exact)
 *   delta = fl32(fl32(hi - lo) / (2^b - 1))
 *   z = clamp(round(fl32(-lo / delta)), 0, 2^b - 1)
 *   u_k = clamp(round(fl32(w'_k / delta)) + z, 0, 2^b - 1)
 * and the dequantised weight is (u_k - z) delta.  q receives the signed code
 * u_k - z (so that every loss below reads q * delta), *zero the point z.
 * An all-zero group has delta = 0, z = 0 and codes 0. */
static void quantize_group_asym(const float *W, const float *s, int64_t D_out, int64_t n, int64_t k0, int group,
                                int bits, int delta16, int8_t *q, float *delta, uint8_t *zero)
{
    const int umax = (1 << bits) - 1;
    float lo = 0.0f, hi = 0.0f;
    for (int k = 0; k < group; ++k) {
        float w = W[(k0 + k) * D_out + n];
        float wp = s ? s[k0 + k] * w : w;
        if (wp < lo)
            lo = wp;
        if (wp > hi)
            hi = wp;
    }
    float d = (hi - lo) / (float)umax;
    if (delta16)
        d = round_to_fp16(d);
    *delta = d;
    int z = 0;
    if (d != 0.0f) {
        float zr = nearbyintf(-lo / d);
        if (zr < 0.0f)
            zr = 0.0f;
        if (zr > (float)umax)
            zr = (float)umax;
        z = (int)zr;
    }
    *zero = (uint8_t)z;
    for (int k = 0; k < group; ++k) {
        int code = 0;
        if (d != 0.0f) {
            float w = W[(k0 + k) * D_out + n];
            float wp = s ? s[k0 + k] * w : w;
            float r = nearbyintf(wp / d) + (float)z;
            if (r < 0.0f)
                r = 0.0f;
            if (r > (float)umax)
                r = (float)umax;
            code = (int)r - z;
        }
        q[k] = (int8_t)code;
    }
}

static void quantize_group(const float *W, const float *s, int64_t D_out, int64_t n,
                           int64_t k0, int group, int bits, float clip, int delta16, int qmode, int8_t *q,
                           float *delta)
{
    if (qmode == 2) {
        uint8_t zdummy;
        quantize_group_asym(W, s, D_out, n, k0, group, bits, delta16, q, delta, &zdummy);
        return;
    }
    const int qmax = (1 << (bits - 1)) - 1;
    /* qmode 1 ([P2] "analysing the quantisation error"): delta = max / 2^(b-1)
     * (an exact power-of-two scaling), codes clamped to [-2^(b-1), 2^(b-1) - 1]
     * so that they fit b bits (the passage gives no clamp; +max would be 2^(b-1)). */
    const int qlo = qmode == 1 ? -(qmax + 1) : -qmax;
    float m = 0.0f;
    for (int k = 0; k < group; ++k) {
        float w = W[(k0 + k) * D_out + n];
        float wp = s ? s[k0 + k] * w : w;
        float am = fabsf(wp);
        if (am > m)
            m = am;
    }
    m = clip * m;
    float d = qmode == 1 ? ldexpf(m, -(bits - 1)) : m / (float)qmax;
    if (delta16)
        d = round_to_fp16(d);      /* the exported FP16 delta, which the codes then use */
    *delta = d;
    for (int k = 0; k < group; ++k) {
        int code = 0;
        if (d != 0.0f) {
            float w = W[(k0 + k) * D_out + n];
            float wp = s ? s[k0 + k] * w : w;
            float t = wp / d;
            float r = nearbyintf(t); /* round half to even in the default mode */
            if (r > (float)qmax)
                r = (float)qmax;
            if (r < (float)qlo)
                r = (float)qlo;
            code = (int)r;
        }
        q[k] = (int8_t)code;
    }
}

/* Quantise every (group, column) of diag(s) W.  q: [D_in][D_out] codes in
 * [-qmax, qmax]; delta: [D_in/group][D_out].  clip: [D_in/group][D_out] clip
 * ratios, or NULL for none.  delta16: delta is rounded to FP16 before the
 * codes are formed (the exported scale format). */
void oracle_quantize_mode(const float *W, const float *s, const float *clip, int64_t D_in, int64_t D_out,
                          int bits, int group, int delta16, int qmode, int8_t *q, float *delta)
{
    int8_t *col = (int8_t *)malloc((size_t)group);
    for (int64_t n = 0; n < D_out; ++n) {
        for (int64_t g = 0; g < D_in / group; ++g) {
            quantize_group(W, s, D_out, n, g * group, group, bits, clip ? clip[g * D_out + n] : 1.0f, delta16,
                           qmode, col, &delta[g * D_out + n]);
            for (int k = 0; k < group; ++k)
                q[(g * group + k) * D_out + n] = col[k];
        }
    }
    free(col);
}

/* The asymmetric quantiser over every (group, column): q [D_in][D_out] signed
 * codes u - z, delta and zeros [D_in/group][D_out]. */
void oracle_quantize_asym(const float *W, const float *s, int64_t D_in, int64_t D_out, int bits, int group,
                          int delta16, int8_t *q, float *delta, uint8_t *zeros)
{
    int8_t *col = (int8_t *)malloc((size_t)group);
    for (int64_t n = 0; n < D_out; ++n) {
        for (int64_t g = 0; g < D_in / group; ++g) {
            quantize_group_asym(W, s, D_out, n, g * group, group, bits, delta16, col, &delta[g * D_out + n],
                                &zeros[g * D_out + n]);
            for (int k = 0; k < group; ++k)
                q[(g * group + k) * D_out + n] = col[k];
        }
    }
    free(col);
}

void oracle_quantize_ex(const float *W, const float *s, const float *clip, int64_t D_in, int64_t D_out,
                        int bits, int group, int delta16, int8_t *q, float *delta)
{
    oracle_quantize_mode(W, s, clip, D_in, D_out, bits, group, delta16, 0, q, delta);
}

void oracle_quantize_clip(const float *W, const float *s, const float *clip, int64_t D_in, int64_t D_out,
                          int bits, int group, int8_t *q, float *delta)
{
    oracle_quantize_ex(W, s, clip, D_in, D_out, bits, group, 0, q, delta);
}

void oracle_quantize(const float *W, const float *s, int64_t D_in, int64_t D_out,
                     int bits, int group, int8_t *q, float *delta)
{
    oracle_quantize_ex(W, s, NULL, D_in, D_out, bits, group, 0, q, delta);
}

/* Pack codes: word (k8, n) holds rows 8*k8 .. 8*k8+7 of column n, row 8*k8+i in
 * bits 4i..4i+3 as u = q + 2^(b-1).  [P1] "inference-time equivalent":
 * W_quantized = Quantize(diag(s*) W) stored as INT4. */
void oracle_pack(const int8_t *q, int64_t D_in, int64_t D_out, int bits, uint32_t *packed)
{
    const int off = 1 << (bits - 1);
    for (int64_t k8 = 0; k8 < D_in / 8; ++k8) {
        for (int64_t n = 0; n < D_out; ++n) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i) {
                int u = (int)q[(8 * k8 + i) * D_out + n] + off;
                word |= ((uint32_t)u & 0xFu) << (4 * i);
            }
            packed[k8 * D_out + n] = word;
        }
    }
}

/* Dense 3-bit packing (an option of the pack): the 32 codes of rows 32j .. 32j+31 of column
 * n as one 96-bit little-endian string, code i (u = q + 4) at bits 3i .. 3i+2,
 * stored as words (3j, n), (3j+1, n), (3j+2, n) holding bits 0-31, 32-63 and
 * 64-95.  Codes 10 and 21 straddle two words.  D_in % 32 == 0. */
void oracle_pack3(const int8_t *q, int64_t D_in, int64_t D_out, uint32_t *packed)
{
    for (int64_t j = 0; j < D_in / 32; ++j) {
        for (int64_t n = 0; n < D_out; ++n) {
            uint32_t w[3] = {0u, 0u, 0u};
            for (int i = 0; i < 32; ++i) {
                const uint32_t u = (uint32_t)((int)q[(32 * j + i) * D_out + n] + 4) & 7u;
                for (int b = 0; b < 3; ++b) {
                    const int bit = 3 * i + b;
                    w[bit / 32] |= ((u >> b) & 1u) << (bit % 32);
                }
            }
            for (int t = 0; t < 3; ++t)
                packed[(3 * j + t) * D_out + n] = w[t];
        }
    }
}

/* [P1] flow step 4c for a set of output columns:
 *   L_n = sum_i ( sum_k x_ik * e_kn )^2,   e_kn = q_kn * delta_gn / s_k - w_kn
 * which is column n's share of ||X S^-1 Q(S W) - X W||^2 (exact algebra: the
 * k-th row of S^-1 Q(SW) is q_kn delta_gn / s_k).  All in fp64.
 * quantize == 0 replaces Q by the identity (w'_k itself), for the
 * cancellation check. */
static double column_loss(const double *Xd, const float *W, const float *s,
                          int64_t N, int64_t D_in, int64_t D_out, int64_t n,
                          int bits, int group, int quantize, int qmode, double *e, int8_t *qcol)
{
    for (int64_t g = 0; g < D_in / group; ++g) {
        const int64_t k0 = g * group;
        if (quantize) {
            float d;
            quantize_group(W, s, D_out, n, k0, group, bits, 1.0f, 0, qmode, qcol, &d);
            for (int k = 0; k < group; ++k) {
                double sk = s ? (double)s[k0 + k] : 1.0;
                e[k0 + k] = (double)qcol[k] * (double)d / sk - (double)W[(k0 + k) * D_out + n];
            }
        } else {
            for (int k = 0; k < group; ++k) {
                float w = W[(k0 + k) * D_out + n];
                float wp = s ? s[k0 + k] * w : w;
                double sk = s ? (double)s[k0 + k] : 1.0;
                e[k0 + k] = (double)wp / sk - (double)w;
            }
        }
    }
    double acc = 0.0;
    for (int64_t i = 0; i < N; ++i) {
        const double *xr = Xd + i * D_in;
        double y = 0.0;
        for (int64_t k = 0; k < D_in; ++k)
            y += xr[k] * e[k];
        acc += y * y;
    }
    return acc;
}

static double *x_to_double(const uint16_t *X, int64_t N, int64_t D_in)
{
    double *Xd = (double *)malloc((size_t)(N * D_in) * sizeof(double));
    for (int64_t i = 0; i < N * D_in; ++i)
        Xd[i] = bf16_bits_to_double(X[i]);
    return Xd;
}

/* Per-column losses for one scale vector s (NULL = all ones).  cols == NULL
 * means every column; otherwise L_col[c] is the loss of column cols[c]. */
void oracle_loss_cols_mode(const uint16_t *X, const float *W, const float *s,
                           int64_t N, int64_t D_in, int64_t D_out, int bits, int group,
                           int quantize, int qmode, const int64_t *cols, int64_t ncols, double *L_col)
{
    double *Xd = x_to_double(X, N, D_in);
    const int64_t nc = cols ? ncols : D_out;
#pragma omp parallel
    {
        double *e = (double *)malloc((size_t)D_in * sizeof(double));
        int8_t *qcol = (int8_t *)malloc((size_t)group);
#pragma omp for schedule(dynamic, 1)
        for (int64_t c = 0; c < nc; ++c) {
            int64_t n = cols ? cols[c] : c;
            L_col[c] = column_loss(Xd, W, s, N, D_in, D_out, n, bits, group, quantize, qmode, e, qcol);
        }
        free(e);
        free(qcol);
    }
    free(Xd);
}

void oracle_loss_cols(const uint16_t *X, const float *W, const float *s,
                      int64_t N, int64_t D_in, int64_t D_out, int bits, int group,
                      int quantize, const int64_t *cols, int64_t ncols, double *L_col)
{
    oracle_loss_cols_mode(X, W, s, N, D_in, D_out, bits, group, quantize, 0, cols, ncols, L_col);
}

/* [P1] flow steps 3-5 for one layer: for every alpha on the grid, s = a^alpha,
 * quantise diag(s) W per group, L(alpha) = ||X S^-1 Q(SW) - X W||^2, and
 * alpha* = argmin L (the smallest index among exact minima).
 * L: [n_alpha]; L_col: [n_alpha][ncols] (may be NULL); restricted to the
 * columns in cols when cols != NULL (L then sums those columns only).
 * Returns the argmin index. */
/* As oracle_search, with the quantiser mode (qmode, see quantize_group) and
 * the balanced scale when b != NULL (s = a^alpha / b^(1-alpha), [P3]). */
int oracle_search_mode(const uint16_t *X, const float *W, const float *a, const float *b,
                       int64_t N, int64_t D_in, int64_t D_out,
                       const float *alphas, int n_alpha, int bits, int group, int qmode,
                       const int64_t *cols, int64_t ncols, double *L, double *L_col)
{
    const int64_t nc = cols ? ncols : D_out;
    float *s = (float *)malloc((size_t)D_in * sizeof(float));
    double *lc = (double *)malloc((size_t)nc * sizeof(double));
    int best = 0;
    for (int ai = 0; ai < n_alpha; ++ai) {
        if (b)
            oracle_scales_balanced(a, b, D_in, alphas[ai], s);
        else
            oracle_scales(a, D_in, alphas[ai], s);
        oracle_loss_cols_mode(X, W, s, N, D_in, D_out, bits, group, 1, qmode, cols, ncols, lc);
        double sum = 0.0;
        for (int64_t c = 0; c < nc; ++c) {
            sum += lc[c];
            if (L_col)
                L_col[(int64_t)ai * nc + c] = lc[c];
        }
        L[ai] = sum;
        if (L[ai] < L[best])
            best = ai;
    }
    free(lc);
    free(s);
    return best;
}

int oracle_search(const uint16_t *X, const float *W, const float *a,
                  int64_t N, int64_t D_in, int64_t D_out,
                  const float *alphas, int n_alpha, int bits, int group,
                  const int64_t *cols, int64_t ncols, double *L, double *L_col)
{
    return oracle_search_mode(X, W, a, NULL, N, D_in, D_out, alphas, n_alpha, bits, group, 0, cols, ncols, L, L_col);
}

/* The literal two-product form of [P1] flow step 4c for tiny layers:
 * materialise S^-1 (D_in x D_in), W_hat' = Q(S W) (D_in x D_out, codes times
 * delta), then L = ||(X S^-1) W_hat' - X W||_F^2, all in long double. */
long double oracle_literal_loss(const uint16_t *X, const float *W, const float *s,
                                int64_t N, int64_t D_in, int64_t D_out, int bits, int group)
{
    long double *Sinv = (long double *)calloc((size_t)(D_in * D_in), sizeof(long double));
    long double *What = (long double *)malloc((size_t)(D_in * D_out) * sizeof(long double));
    long double *XS = (long double *)malloc((size_t)(N * D_in) * sizeof(long double));
    int8_t *q = (int8_t *)malloc((size_t)(D_in * D_out));
    float *delta = (float *)malloc((size_t)(D_in / group * D_out) * sizeof(float));
    for (int64_t k = 0; k < D_in; ++k)
        Sinv[k * D_in + k] = 1.0L / (long double)s[k];
    oracle_quantize(W, s, D_in, D_out, bits, group, q, delta);
    for (int64_t k = 0; k < D_in; ++k)
        for (int64_t n = 0; n < D_out; ++n)
            What[k * D_out + n] = (long double)q[k * D_out + n] * (long double)delta[(k / group) * D_out + n];
    for (int64_t i = 0; i < N; ++i)
        for (int64_t c = 0; c < D_in; ++c) {
            long double acc = 0.0L;
            for (int64_t k = 0; k < D_in; ++k)
                acc += (long double)bf16_bits_to_double(X[i * D_in + k]) * Sinv[k * D_in + c];
            XS[i * D_in + c] = acc;
        }
    long double L = 0.0L;
    for (int64_t i = 0; i < N; ++i)
        for (int64_t n = 0; n < D_out; ++n) {
            long double yq = 0.0L, y = 0.0L;
            for (int64_t k = 0; k < D_in; ++k) {
                yq += XS[i * D_in + k] * What[k * D_out + n];
                y += (long double)bf16_bits_to_double(X[i * D_in + k]) * (long double)W[k * D_out + n];
            }
            L += (yq - y) * (yq - y);
        }
    free(Sinv);
    free(What);
    free(XS);
    free(q);
    free(delta);
    return L;
}

/* Number of OpenMP threads the loss loops use (reported with CPU timings). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Weight clipping search ([P2] "searching the optimal scale": after the scale
 * search, weight clipping is applied to minimise the quantisation MSE).
 * Reading: per (group, column) and per clip ratio c_i of a given grid, the
 * mean squared error of that group's share of the layer output,
 *   loss[i][g][n] = sum_t ( sum_{k in g} x_tk e_k )^2,
 *   e_k = q_k * delta / s_k - w_kn,   q, delta from quantize_group(clip = c_i),
 * in fp64; best[g][n] = argmin_i loss[i][g][n], the lowest index on exact
 * ties.  cols == NULL means every column (else column cols[c] in slot c);
 * loss may be NULL. */
void oracle_clip_loss(const uint16_t *X, const float *W, const float *s, int64_t N, int64_t D_in, int64_t D_out,
                      const float *clip, int n_clip, int bits, int group, const int64_t *cols, int64_t ncols,
                      double *loss, int32_t *best)
{
    double *Xd = x_to_double(X, N, D_in);
    const int64_t nc = cols ? ncols : D_out;
    const int64_t G = D_in / group;
#pragma omp parallel
    {
        double *e = (double *)malloc((size_t)group * sizeof(double));
        int8_t *qg = (int8_t *)malloc((size_t)group);
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t c = 0; c < nc; ++c) {
            for (int64_t g = 0; g < G; ++g) {
                const int64_t n = cols ? cols[c] : c;
                const int64_t k0 = g * group;
                double lbest = 0.0;
                int ibest = 0;
                for (int i = 0; i < n_clip; ++i) {
                    float d;
                    quantize_group(W, s, D_out, n, k0, group, bits, clip[i], 0, 0, qg, &d);
                    for (int k = 0; k < group; ++k) {
                        double sk = s ? (double)s[k0 + k] : 1.0;
                        e[k] = (double)qg[k] * (double)d / sk - (double)W[(k0 + k) * D_out + n];
                    }
                    double acc = 0.0;
                    for (int64_t t = 0; t < N; ++t) {
                        const double *xr = Xd + t * D_in + k0;
                        double y = 0.0;
                        for (int k = 0; k < group; ++k)
                            y += xr[k] * e[k];
                        acc += y * y;
                    }
                    if (loss)
                        loss[((int64_t)i * G + g) * nc + c] = acc;
                    if (i == 0 || acc < lbest) {
                        lbest = acc;
                        ibest = i;
                    }
                }
                best[g * nc + c] = ibest;
            }
        }
        free(e);
        free(qg);
    }
    free(Xd);
}

/* The quantised layer applied to activations ([P1] "inference-time
 * equivalent": W_quantized = Quantize(diag(s*) W) with s* kept as metadata and
 * 1/s* folded into the input; [P2] "searching the optimal scale": the output
 * Q(W diag(s)) (diag(s)^-1 X)):
 *   Y[t][n] = sum_k x_tk / s_k * (u_kn - 2^(b-1)) * delta_{k/group, n}
 * with u the offset-binary nibble of row k, column n of the packed words
 * (row 8*k8+i in bits 4i..4i+3 of word (k8, n)).  fp64 throughout. */
void oracle_w4a16(const uint16_t *X, const float *s, const uint32_t *packed, const float *scales, int64_t N,
                  int64_t D_in, int64_t D_out, int bits, int group, double *Y)
{
    const int off = 1 << (bits - 1);
    double *wd = (double *)malloc((size_t)(D_in * D_out) * sizeof(double));
    for (int64_t k = 0; k < D_in; ++k)
        for (int64_t n = 0; n < D_out; ++n) {
            const uint32_t word = packed[(k / 8) * D_out + n];
            const int u = (int)((word >> (4 * (k % 8))) & 0xFu);
            wd[k * D_out + n] = (double)(u - off) * (double)scales[(k / group) * D_out + n] / (double)s[k];
        }
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        for (int64_t n = 0; n < D_out; ++n)
            Y[t * D_out + n] = 0.0;
        for (int64_t k = 0; k < D_in; ++k) {
            const double x = bf16_bits_to_double(X[t * D_in + k]);
            if (x == 0.0)
                continue;
            const double *wr = wd + k * D_out;
            double *yr = Y + t * D_out;
            for (int64_t n = 0; n < D_out; ++n)
                yr[n] += x * wr[n];
        }
    }
    free(wd);
}

/* The layer applied to activations from asymmetric (zero-point) codes (the
 * stored u = q + z of the MinMax quantiser): as oracle_w4a16 with each
 * group's zero point in place of 2^(b-1),
 *   Y[t][n] = sum_k x_tk / s_k * (u_kn - z_{k/group, n}) * delta_{k/group, n},
 * zeros [D_in/group][D_out] uint8.  fp64 throughout. */
void oracle_w4a16_zp(const uint16_t *X, const float *s, const uint32_t *packed, const float *scales,
                     const uint8_t *zeros, int64_t N, int64_t D_in, int64_t D_out, int group, double *Y)
{
    double *wd = (double *)malloc((size_t)(D_in * D_out) * sizeof(double));
    for (int64_t k = 0; k < D_in; ++k)
        for (int64_t n = 0; n < D_out; ++n) {
            const uint32_t word = packed[(k / 8) * D_out + n];
            const int u = (int)((word >> (4 * (k % 8))) & 0xFu);
            const int z = (int)zeros[(k / group) * D_out + n];
            wd[k * D_out + n] = (double)(u - z) * (double)scales[(k / group) * D_out + n] / (double)s[k];
        }
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        for (int64_t n = 0; n < D_out; ++n)
            Y[t * D_out + n] = 0.0;
        for (int64_t k = 0; k < D_in; ++k) {
            const double x = bf16_bits_to_double(X[t * D_in + k]);
            if (x == 0.0)
                continue;
            const double *wr = wd + k * D_out;
            double *yr = Y + t * D_out;
            for (int64_t n = 0; n < D_out; ++n)
                yr[n] += x * wr[n];
        }
    }
    free(wd);
}

