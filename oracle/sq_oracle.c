/*
 * sq_oracle.c -- plain, slow, obviously-correct CPU oracle for the SmoothQuant
 * W8A8 linear layer (per-token activation scales x per-output-channel weight
 * scales, int8 x int8 -> int32, dequantised epilogue).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this library.  The product
 * path (the CUDA library) never calls it and shares no code with it.
 *
 * Arithmetic contract (kept deliberately plain so it can be checked by eye):
 *   - every floating-point step is one IEEE-754 binary32 operation with
 *     round-to-nearest-even; the file is compiled with -ffp-contract=off so no
 *     multiply-add is fused, and without -ffast-math;
 *   - bf16 inputs are widened to fp32 exactly (the 16 bf16 bits become the
 *     high half of the fp32 word);
 *   - "round" is round-half-to-even (nearbyint under the default
 *     FE_TONEAREST mode), then clamp to the symmetric range [-127, 127];
 *   - a zero absolute maximum gives scale 0 and all-zero codes (no division);
 *   - inputs must be finite; non-finite inputs are outside the contract.
 *
 * Sources, by page and section:
 *   [W]  "Understanding W8A8 INT8 LLM Quantization", section "Why Naive
 *        Weight Quantization Doesn't Work, and How GPTQ Fixes It": the
 *        per-channel weight scale max|w|/127 and code round(w/scale).
 *   [A]  same page, section "Why Activation Quantization Is Hard, and How
 *        SmoothQuant Fixes It": one dynamic scale per token over all channels.
 *   [S]  same page, sections "Where the outlier actually comes from" and
 *        "How the smoothing factor is computed": per-input-channel absmax over
 *        calibration samples, smoothing factor s_j, activations divided by s,
 *        the matching weight input channel multiplied by s.
 *   [V]  "quant_llm_int8" (LLM.int8() architecture page), sections "The
 *        architecture: every piece explained" and "End-to-end flow": int8
 *        matmul accumulating in int32, dequantised by the outer product of the
 *        per-row activation scales and the per-column weight scales.
 *   [C]  "How does SmoothQuant int8 LLM calibration work...", section "The
 *        Technical Workflow for Int8 Quantization Deployment": calibration
 *        records the maximum absolute value of every channel.
 *   [R]  "Understanding W8A8 INT8 LLM Quantization", section "Where the
 *        outlier actually comes from": RMSNorm (divide by the vector's
 *        root-mean-square, multiply by gamma) and SmoothQuant's division of
 *        gamma by s.
 *   [F]  "Understanding W8A8 INT8 LLM Quantization", section "Inter-Token
 *        Latency (ITL)": per layer and token, the dynamic activation
 *        quantisation is memory-bound work; and "How does SmoothQuant int8
 *        LLM calibration work...", section "Hardware Acceleration and
 *        Inference Optimization Strategies": fusing the feed-forward network
 *        with its neighbours saves memory traffic.  The pages do not define
 *        the feed-forward network itself; the gated SiLU form below is the
 *        one of the Llama-3-8B layers whose shapes the workloads use.
 *
 *   [G]  "Understanding W8A8 INT8 LLM Quantization", section "How GPTQ
 *        improves on naive quantization": quantise the weights of a channel
 *        one at a time, and after each one push its rounding error onto the
 *        channel's not yet quantised weights, weighted by the Hessian computed
 *        from the calibration activations.
 *
 * The smoothing-factor equation itself did not survive the page's text
 * extraction; this oracle uses s_j = A_j^alpha / B_j^(1-alpha), with A_j the
 * calibration absmax of input channel j and B_j the absmax of input channel j
 * of the weight, evaluated in fp64 with libm pow and rounded once to fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes shared with the Python wrapper: 0 = fp32, 1 = bf16 */
#define SQO_F32 0
#define SQO_BF16 1

static float widen_bf16(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* element i of a row-major fp32 or bf16 buffer, widened to fp32 exactly */
static float elem(const void *p, int dt, size_t i)
{
    if (dt == SQO_BF16)
        return widen_bf16(((const uint16_t *)p)[i]);
    return ((const float *)p)[i];
}

/* round-half-to-even of an fp32 value to the nearest bf16 (16-bit pattern) */
uint16_t sqo_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u); /* keep NaN a NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* [C], [S]: A_j = max over calibration tokens t of |X[t, j]|.
 * x: [T, K] with row stride ldx elements.  ax: [K], overwritten. */
void sqo_calib_absmax(const void *x, int dt, int64_t T, int64_t K, int64_t ldx, float *ax)
{
    for (int64_t j = 0; j < K; ++j)
        ax[j] = 0.0f;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < K; ++j) {
            float v = fabsf(elem(x, dt, (size_t)(t * ldx + j)));
            if (v > ax[j])
                ax[j] = v;
        }
}

/* [S]: B_j = max over output channels n of |W[n, j]|, W stored [N, K]
 * (out x in), so input channel j is column j. */
void sqo_weight_in_absmax(const void *w, int dt, int64_t N, int64_t K, float *aw)
{
    for (int64_t j = 0; j < K; ++j)
        aw[j] = 0.0f;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K; ++j) {
            float v = fabsf(elem(w, dt, (size_t)(n * K + j)));
            if (v > aw[j])
                aw[j] = v;
        }
}

/* [S]: s_j = A_j^alpha / B_j^(1 - alpha) in fp64, rounded once to fp32.
 * alpha is the fp32 argument widened to fp64.  A channel with A_j == 0 or
 * B_j == 0 is left unmigrated (s_j = 1). */
void sqo_smooth_factors(const float *ax, const float *aw, int64_t K, float alpha, float *s)
{
    double a = (double)alpha;
    for (int64_t j = 0; j < K; ++j) {
        if (ax[j] == 0.0f || aw[j] == 0.0f) {
            s[j] = 1.0f;
            continue;
        }
        double num = pow((double)ax[j], a);
        double den = pow((double)aw[j], 1.0 - a);
        s[j] = (float)(num / den);
    }
}

/* [S] then [W]: W'[n, k] = W[n, k] * s[k] (the weight's input channel k is
 * scaled up by s_k); sw[n] = max_k |W'[n, k]| / 127;
 * wq[n, k] = clamp(round(W'[n, k] / sw[n]), -127, 127). */
void sqo_smooth_quant_weight(const void *w, int dt, int64_t N, int64_t K, const float *s,
                             int8_t *wq, float *sw)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(elem(w, dt, (size_t)(n * K + k)) * s[k]);
            if (v > amax)
                amax = v;
        }
        float scale = amax / 127.0f;
        sw[n] = scale;
        for (int64_t k = 0; k < K; ++k) {
            int8_t q = 0;
            if (amax != 0.0f) {
                float wp = elem(w, dt, (size_t)(n * K + k)) * s[k];
                float r = nearbyintf(wp / scale);
                if (r > 127.0f)
                    r = 127.0f;
                if (r < -127.0f)
                    r = -127.0f;
                q = (int8_t)r;
            }
            wq[n * K + k] = q;
        }
    }
}

/* [S] then [A]: x^[m, k] = X[m, k] / s[k]; sx[m] = max_k |x^[m, k]| / 127;
 * xq[m, k] = clamp(round(x^[m, k] / sx[m]), -127, 127).  Only the rows listed
 * in `rows` (or all M rows when rows == NULL) are computed; row i of the
 * outputs corresponds to rows[i].  x has row stride ldx elements. */
void sqo_quant_act_rows(const void *x, int dt, int64_t ldx, int64_t K, const float *s,
                        const int64_t *rows, int64_t nrows, int8_t *xq, float *sx)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = fabsf(elem(x, dt, (size_t)(m * ldx + k)) / s[k]);
            if (v > amax)
                amax = v;
        }
        float scale = amax / 127.0f;
        sx[i] = scale;
        for (int64_t k = 0; k < K; ++k) {
            int8_t q = 0;
            if (amax != 0.0f) {
                float xh = elem(x, dt, (size_t)(m * ldx + k)) / s[k];
                float r = nearbyintf(xh / scale);
                if (r > 127.0f)
                    r = 127.0f;
                if (r < -127.0f)
                    r = -127.0f;
                q = (int8_t)r;
            }
            xq[i * K + k] = q;
        }
    }
}

void sqo_quant_act(const void *x, int dt, int64_t M, int64_t K, const float *s, int8_t *xq,
                   float *sx)
{
    sqo_quant_act_rows(x, dt, K, K, s, NULL, M, xq, sx);
}

/* [V]: acc[m, n] = sum_k xq[m, k] * wq[n, k], exact in int32 (|acc| is at
 * most K * 127^2, below 2^31 for K <= 133144).  Both operands are K-major. */
void sqo_gemm_i32(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                  int32_t *acc)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int32_t a = 0;
            for (int64_t k = 0; k < K; ++k)
                a += (int32_t)xq[m * K + k] * (int32_t)wq[n * K + k];
            acc[m * N + n] = a;
        }
}

/* [V]: one accumulator for each listed (m, n) pair. */
void sqo_gemm_i32_pairs(const int8_t *xq, int64_t ldxq, const int8_t *wq, int64_t K,
                        const int64_t *ms, const int64_t *ns, int64_t npairs, int32_t *acc)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < npairs; ++i) {
        int32_t a = 0;
        for (int64_t k = 0; k < K; ++k)
            a += (int32_t)xq[ms[i] * ldxq + k] * (int32_t)wq[ns[i] * K + k];
        acc[i] = a;
    }
}

/* [V]: y = ((float)acc * sx[m]) * sw[n], two fp32 multiplies in this order.
 * y_f32 and/or y_bf16 may be NULL. */
void sqo_dequant(const int32_t *acc, const float *sx, const float *sw, int64_t M, int64_t N,
                 float *y_f32, uint16_t *y_bf16)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float t = (float)acc[m * N + n] * sx[m];
            float y = t * sw[n];
            if (y_f32)
                y_f32[m * N + n] = y;
            if (y_bf16)
                y_bf16[m * N + n] = sqo_f32_to_bf16(y);
        }
}

/* [V]: the dequantised value for each listed (m, n) pair, same arithmetic as
 * sqo_dequant; acc[i], sx[i] and sw[i] belong to pair i. */
void sqo_dequant_pairs(const int32_t *acc, const float *sx, const float *sw, int64_t npairs,
                       float *y_f32, uint16_t *y_bf16)
{
    for (int64_t i = 0; i < npairs; ++i) {
        float t = (float)acc[i] * sx[i];
        float y = t * sw[i];
        if (y_f32)
            y_f32[i] = y;
        if (y_bf16)
            y_bf16[i] = sqo_f32_to_bf16(y);
    }
}

/* [R] "Understanding W8A8 INT8 LLM Quantization", section "Where the
 * outlier actually comes from": RMSNorm divides every value of a token's
 * vector by the vector's root-mean-square, then multiplies channel j by the
 * trained gamma_j; SmoothQuant divides gamma by the smoothing factors s, so
 * the norm's output is already the smoothed activation.
 *   g[j] = gamma[j] / s[j]   (one IEEE fp32 division per channel, offline) */
void sqo_fold_gamma(const float *gamma, const float *s, int64_t K, float *g)
{
    for (int64_t j = 0; j < K; ++j)
        g[j] = gamma[j] / s[j];
}

/* [R] then [A], per token m:
 *   ms   = (sum_k h[m, k]^2) / K + eps in fp64 (every square is exact in
 *          fp64; the sum runs in index order);
 *   rinv = 1 / sqrt(ms) with IEEE fp64 sqrt and division, rounded once to
 *          fp32 (0 when ms is 0: a zero row stays zero);
 *   a    = (h[m, k] * rinv) * g[k], two fp32 multiplies;
 *   sx   = max_k |a| / 127;  xq = clamp(round(a / sx), -127, 127).
 * rinv_out (may be NULL) receives rinv per token.
 *
 * The pages fix no summation order for the squares.  Any order of the fp64
 * sum of K non-negative terms lies within (K - 1) 2^-53 (relative) of the
 * exact sum, so any implementation's fp64 value of 1 / sqrt(ms) lies within
 * about (K + 16) 2^-53 of this one's, and only where this one's lies that
 * close to an fp32 rounding midpoint can another order round rinv to the
 * other neighbour.  For such a token the oracle flags it (alt_flag[m] = 1)
 * and also computes the whole result for the neighbour on the far side of
 * that midpoint (alt_rinv, alt_sx, alt_xq); otherwise alt_flag[m] = 0 and the
 * alternate outputs repeat the primary ones.  `window` is the relative
 * distance to a midpoint that flags a token; window < 0 takes
 * (K + 16) 2^-52, twice the bound above.  The alt_* pointers may be NULL. */
static void rmsnorm_quant_row(const void *h, int dt, int64_t m, int64_t K, const float *g, float rinv,
                              int8_t *xq_row, float *sx_out)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf((elem(h, dt, (size_t)(m * K + k)) * rinv) * g[k]);
        if (a > amax)
            amax = a;
    }
    float scale = amax / 127.0f;
    *sx_out = scale;
    for (int64_t k = 0; k < K; ++k) {
        int8_t q = 0;
        if (amax != 0.0f) {
            float a = (elem(h, dt, (size_t)(m * K + k)) * rinv) * g[k];
            float r = nearbyintf(a / scale);
            if (r > 127.0f)
                r = 127.0f;
            if (r < -127.0f)
                r = -127.0f;
            q = (int8_t)r;
        }
        xq_row[k] = q;
    }
}

void sqo_rmsnorm_quant(const void *h, int dt, int64_t M, int64_t K, const float *g, float eps, double window,
                       int8_t *xq, float *sx, float *rinv_out, uint8_t *alt_flag, int8_t *alt_xq, float *alt_sx,
                       float *alt_rinv)
{
    const double win = window < 0.0 ? ((double)K + 16.0) * ldexp(1.0, -52) : window;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double v = (double)elem(h, dt, (size_t)(m * K + k));
            ss += v * v;
        }
        double ms = ss / (double)K + (double)eps;
        double r64 = ms > 0.0 ? 1.0 / sqrt(ms) : 0.0;
        float rinv = (float)r64;
        if (rinv_out)
            rinv_out[m] = rinv;
        rmsnorm_quant_row(h, dt, m, K, g, rinv, xq + m * K, sx + m);
        /* the neighbour across the midpoint on r64's side of rinv (the
         * nearer one), if that midpoint lies within the window */
        float other = rinv;
        if (r64 > 0.0) {
            const float nb = r64 >= (double)rinv ? nextafterf(rinv, INFINITY) : nextafterf(rinv, 0.0f);
            const double mid = ((double)rinv + (double)nb) / 2.0;
            if (fabs(r64 - mid) <= win * r64)
                other = nb;
        }
        if (alt_flag)
            alt_flag[m] = other != rinv;
        if (alt_rinv)
            alt_rinv[m] = other;
        if (alt_xq && alt_sx) {
            if (other != rinv) {
                rmsnorm_quant_row(h, dt, m, K, g, other, alt_xq + m * K, alt_sx + m);
            } else {
                memcpy(alt_xq + m * K, xq + m * K, (size_t)K);
                alt_sx[m] = sx[m];
            }
        }
    }
}

/* [F] e^x in binary32, as a fixed sequence of IEEE operations (fmaf is one
 * correctly rounded fused multiply-add), so that every implementation that
 * follows the same steps gets the same bits.  Method: Cody and Waite's
 * argument reduction, then the Taylor series of e^r to degree 7.
 *   x < -87: 0 (e^-87 is about 1.6e-38; below it the result would leave the
 *            normal range; for SiLU only 1 + e^x matters, which is then 1);
 *   x >  88: +infinity;
 *   else     n = the integer nearest to x * L2E (L2E = RN(log2 e)), taken
 *            from fmaf(x, L2E, 1.5 * 2^23) - 1.5 * 2^23;
 *            r = fmaf(-n, LN2_LO, fmaf(-n, LN2_HI, x)), with LN2_HI = RN(ln 2)
 *            and LN2_LO = RN(ln 2 - LN2_HI);
 *            p = 1 + r (1 + r (1/2! + r (1/3! + ... + r / 7!))) by Horner's
 *            rule, one fmaf per step, each coefficient RN(1/k!);
 *            e^x = p * 2^n (exact: the result is normal). */
float sqo_exp_f32(float x)
{
    if (x < -87.0f)
        return 0.0f;
    if (x > 88.0f)
        return INFINITY;
    const float magic = 12582912.0f; /* 1.5 * 2^23 */
    const float n = fmaf(x, 0x1.715476p+0f, magic) - magic;
    float r = fmaf(-n, 0x1.62e430p-1f, x);
    r = fmaf(-n, -0x1.05c610p-29f, r);
    float p = 0x1.a01a02p-13f;         /* 1/7! */
    p = fmaf(p, r, 0x1.6c16c2p-10f);   /* 1/6! */
    p = fmaf(p, r, 0x1.111112p-7f);    /* 1/5! */
    p = fmaf(p, r, 0x1.555556p-5f);    /* 1/4! */
    p = fmaf(p, r, 0x1.555556p-3f);    /* 1/3! */
    p = fmaf(p, r, 0.5f);              /* 1/2! */
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    return ldexpf(p, (int)n);
}

/* [F] SiLU(z) = z * sigmoid(z) = z / (1 + e^-z): one fp32 addition and one
 * IEEE fp32 division, e^-z from sqo_exp_f32. */
float sqo_silu_f32(float z)
{
    const float d = 1.0f + sqo_exp_f32(-z);
    return z / d;
}

/* elementwise over arrays (for the tests): y[i] = sqo_exp_f32(x[i]) when
 * which == 0, sqo_silu_f32(x[i]) when which == 1 */
void sqo_exp_silu_vec(const float *x, int64_t n, int which, float *y)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = which == 0 ? sqo_exp_f32(x[i]) : sqo_silu_f32(x[i]);
}

/* [F] then [S] then [A]: the gated feed-forward activation of token m,
 *   h[m, j] = SiLU(gu[m, j]) * gu[m, I + j]   (gate, then up, in one row of
 *             2I values), one fp32 multiply, then rounded to the storage type
 *             of gu (bf16 by round-half-to-even; fp32 unchanged) -- the value
 *             an unfused feed-forward step would store for the next layer;
 * then exactly sqo_quant_act on h: x^ = h / s, sx = max |x^| / 127, codes.
 * h_out (may be NULL) receives h as fp32 [M, I].  h must be finite (like
 * every input of the quantisers). */
void sqo_silu_mul_quant(const void *gu, int dt, int64_t M, int64_t I, const float *s, int8_t *xq,
                        float *sx, float *h_out)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float *h = (float *)malloc((size_t)I * sizeof(float));
        for (int64_t j = 0; j < I; ++j) {
            const float g = elem(gu, dt, (size_t)(m * 2 * I + j));
            const float u = elem(gu, dt, (size_t)(m * 2 * I + I + j));
            float v = sqo_silu_f32(g) * u;
            if (dt == SQO_BF16)
                v = widen_bf16(sqo_f32_to_bf16(v));
            h[j] = v;
            if (h_out)
                h_out[m * I + j] = v;
        }
        float amax = 0.0f;
        for (int64_t j = 0; j < I; ++j) {
            const float v = fabsf(h[j] / s[j]);
            if (v > amax)
                amax = v;
        }
        const float scale = amax / 127.0f;
        sx[m] = scale;
        for (int64_t j = 0; j < I; ++j) {
            int8_t q = 0;
            if (amax != 0.0f) {
                float r = nearbyintf((h[j] / s[j]) / scale);
                if (r > 127.0f)
                    r = 127.0f;
                if (r < -127.0f)
                    r = -127.0f;
                q = (int8_t)r;
            }
            xq[m * I + j] = q;
        }
        free(h);
    }
}

/* ------------------------------------------------------------------------
 * [G] GPTQ.  Every step below is a sequence of IEEE binary64 operations (fma
 * is one correctly rounded fused multiply-add), with every sum in plain index
 * order.  The page describes the algorithm, not an order of summation: an
 * implementation that sums in another order reaches the same values up to
 * rounding, and its codes may then differ where a quotient lies at a
 * rounding tie (the tests bound both).
 * ------------------------------------------------------------------------ */

/* [G] the Hessian of the layer's squared output error over the calibration
 * tokens, without the constant factor (which cancels in every use below):
 *   H[i][j] = sum over t = 0, 1, ... of xh[t][i] * xh[t][j],
 * with xh[t][k] = X[t][k] / s[k] (the smoothed activation, one fp32
 * division, as in sqo_quant_act) widened to fp64; each step
 * acc = fma(xh[t][i], xh[t][j], acc) from acc = 0. */
void sqo_gptq_hessian(const void *x, int dt, int64_t T, int64_t K, const float *s, double *H)
{
    /* xh stored channel by channel (xt[k][t]) so that each sum reads memory
     * in order; the arithmetic is as written above */
    float *xt = (float *)malloc((size_t)(T * K) * sizeof(float));
    for (int64_t t = 0; t < T; ++t)
        for (int64_t k = 0; k < K; ++k)
            xt[k * T + t] = elem(x, dt, (size_t)(t * K + k)) / s[k];
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < K; ++i)
        for (int64_t j = 0; j < K; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t)
                acc = fma((double)xt[i * T + t], (double)xt[j * T + t], acc);
            H[i * K + j] = acc;
        }
    free(xt);
}

/* [G] damping, in place: d = RN(RN(sum_i H[i][i] / K) * damp_frac), the sum
 * taken in index order; d = 1 when that sum is 0 (an all-zero Hessian);
 * then H[i][i] = H[i][i] + d. */
void sqo_gptq_damp(double *H, int64_t K, float damp_frac)
{
    double sum = 0.0;
    for (int64_t i = 0; i < K; ++i)
        sum = sum + H[i * K + i];
    double d = (sum / (double)K) * (double)damp_frac;
    if (sum == 0.0)
        d = 1.0;
    for (int64_t i = 0; i < K; ++i)
        H[i * K + i] = H[i * K + i] + d;
}

/* [G] U, the upper triangular Cholesky factor of H^-1 (H^-1 = U^T U), which
 * carries the error feedback: U[k][j] / U[k][k] is the share of weight k's
 * error that weight j > k takes.  It is computed through the identity
 * U = J L^-1 J, with J the index reversal and L the lower Cholesky factor of
 * J H J (so no inverse of H itself is formed).  Every sum below runs in index
 * order, one fma a term:
 *   G[a][b] = H[K-1-a][K-1-b];
 *   L, column by column (j = 0, 1, ...):
 *     p = G[j][j] - L[j][0]^2 - L[j][1]^2 - ... - L[j][j-1]^2;
 *       L[j][j] = sqrt(p)  (p <= 0: not positive definite, return -1);
 *     for i > j: L[i][j] = (G[i][j] - L[i][0] L[j][0] - ... - L[i][j-1] L[j][j-1]) / L[j][j];
 *   N = L^-1, row by row (forward substitution):
 *     N[i][i] = 1 / L[i][i];
 *     for c < i: N[i][c] = -((L[i][c] N[c][c] + L[i][c+1] N[c+1][c] + ... + L[i][i-1] N[i-1][c]) / L[i][i]);
 *   U[a][b] = N[K-1-a][K-1-b] for b >= a, 0 below the diagonal.
 * Returns 0, or -1 when a pivot is not positive. */
int sqo_gptq_factor(const double *H, int64_t K, double *U)
{
    double *L = (double *)calloc((size_t)(K * K), sizeof(double));
    double *N = (double *)calloc((size_t)(K * K), sizeof(double));
    int bad = 0;
    for (int64_t j = 0; j < K && !bad; ++j) {
        double p = H[(K - 1 - j) * K + (K - 1 - j)];
        for (int64_t k = 0; k < j; ++k)
            p = fma(-L[j * K + k], L[j * K + k], p);
        if (!(p > 0.0)) {
            bad = 1;
            break;
        }
        const double ljj = sqrt(p);
        L[j * K + j] = ljj;
#pragma omp parallel for schedule(static)
        for (int64_t i = j + 1; i < K; ++i) {
            double q = H[(K - 1 - i) * K + (K - 1 - j)];
            for (int64_t k = 0; k < j; ++k)
                q = fma(-L[i * K + k], L[j * K + k], q);
            L[i * K + j] = q / ljj;
        }
    }
    if (!bad) {
        /* N is stored column by column (Nt[c][k] = N[k][c]) so that each sum
         * reads memory in order; the arithmetic is as written above */
        double *Nt = N;
        for (int64_t i = 0; i < K; ++i) {
            Nt[i * K + i] = 1.0 / L[i * K + i];
#pragma omp parallel for schedule(static)
            for (int64_t c = 0; c < i; ++c) {
                double q = 0.0;
                for (int64_t k = c; k < i; ++k)
                    q = fma(L[i * K + k], Nt[c * K + k], q);
                Nt[c * K + i] = -(q / L[i * K + i]);
            }
        }
        for (int64_t a = 0; a < K; ++a)
            for (int64_t b = 0; b < K; ++b)
                U[a * K + b] = b >= a ? Nt[(K - 1 - b) * K + (K - 1 - a)] : 0.0;
    }
    free(L);
    free(N);
    return bad ? -1 : 0;
}

/* [G] then [W]: GPTQ rounding of the smoothed weight, one output channel
 * (row n) at a time:
 *   w[k]  = W[n][k] * s[k] (one fp32 multiply, as in
 *           sqo_smooth_quant_weight), widened to fp64;
 *   sw[n] = max_k |w[k]| / 127 in fp32: the same per-channel scale as the
 *           plain rounding, found once from the unmodified row;
 *   for k = 0..K-1 in order:
 *     q      = clamp(rint(w[k] / sw), -127, 127)  (fp64 division, rounding
 *              half to even; q = 0 throughout when sw = 0)
 *     e      = fma(-q, sw, w[k]) / U[k][k]
 *     w[j]   = fma(-e, U[k][j], w[j]) for every j > k.
 * tie_pos (may be NULL) receives, per row, the first k whose quotient
 * w[k] / sw lies within `tau` of a rounding tie (a half-integer of magnitude
 * below 127.5), or -1.  A U that differs from this one by rounding moves the
 * quotients slightly, so from such a k on another implementation's codes of
 * that row may differ. */
void sqo_gptq_quant_weight(const void *w, int dt, int64_t N, int64_t K, const float *s, const double *U,
                           double tau, int8_t *wq, float *sw, int64_t *tie_pos)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; ++n) {
        double *r = (double *)malloc((size_t)K * sizeof(double));
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            const float v = elem(w, dt, (size_t)(n * K + k)) * s[k];
            r[k] = (double)v;
            if (fabsf(v) > amax)
                amax = fabsf(v);
        }
        const float scale = amax / 127.0f;
        sw[n] = scale;
        const double sd = (double)scale;
        int64_t tie = -1;
        for (int64_t k = 0; k < K; ++k) {
            double q = 0.0;
            if (scale != 0.0f) {
                const double t = r[k] / sd;
                const double a = fabs(t);
                if (tie < 0 && a < 127.5 + tau && fabs(a - floor(a) - 0.5) <= tau)
                    tie = k;
                q = nearbyint(t);
                if (q > 127.0)
                    q = 127.0;
                if (q < -127.0)
                    q = -127.0;
                const double e = fma(-q, sd, r[k]) / U[k * K + k];
                for (int64_t j = k + 1; j < K; ++j)
                    r[j] = fma(-e, U[k * K + j], r[j]);
            }
            wq[n * K + k] = (int8_t)q;
        }
        if (tie_pos)
            tie_pos[n] = tie;
        free(r);
    }
}

int sqo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
