/*
 * zq_oracle.c -- plain, slow, CPU reference of the W8A8 linear hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or constant
 * with the CUDA library.
 *
 * Every function is the plain definition of one step, written as loops in
 * the order the sources state it.  Floating point runs in double except
 * where the method itself fixes fp32 (the quantizer: scale = absmax/127 and
 * the code rint(v * (127/absmax)) are fp32 operations by definition).
 *
 * Sources (web pages) and the passages each function follows:
 *   [ZQ]   "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
 *          Quantization for Large-Scale Transformers" -- group-wise weight
 *          quantization paragraph; token-wise activation quantization
 *          paragraph; the fused-kernel flowcharts (LN/GeLU + Quantize,
 *          GEMM + DeQuantize).
 *   [TS36] "探秘Transformer系列之（36）— 大模型量化方案" -- §1.1.2
 *          (absmax quantization to [-127,127]; vector-wise quantization,
 *          denormalisation by the outer product of row and column scales);
 *          §1.2.2 (dynamic per-token activation quantization fused with the
 *          preceding LayerNorm; INT32 accumulators scaled by the weight and
 *          activation scales before the FP16 write; group-wise weights).
 *   [IQ]   "Integer Quantization: Deep Dive" -- "如何进行量化？" (quantize
 *          with scale, zero-point, round-to-nearest and clamp); "量化模拟"
 *          (dequantize x = s * (x_int - z)); "量化误差" (rounding error is
 *          at most s/2).
 *   [TS36] §1.3 SmoothQuant -- per-channel smoothing factor s chosen
 *          offline; Y = (X diag(s)^-1)(diag(s) W): weights scaled up per
 *          input channel, activations scaled down, output unchanged.
 *   [TS36] §1.1 LLM.int8() -- mixed-precision decomposition: the columns
 *          of the input holding a value above the threshold alpha = 6.0
 *          form the outlier set O; X[:, O] times the matching weights run in
 *          FP16; the other columns are quantized (absmax per row of X and
 *          per output of W) for the INT8 product, dequantized, and the two
 *          results are added.
 *   [SQ]   "SmoothQuant技术解析：大模型INT8量化的突破与实践" §2.2 (the same
 *          identity; s chosen so the channels of X diag(s)^-1 have similar
 *          absolute maxima), §3 (calibration of per-channel max |X| over
 *          calibration batches; offline fold into the weights).
 *
 * Readings where the pages are silent (each one is a choice, stated once):
 *   R1 round-to-nearest ties go to even (rintf under the default mode);
 *   R2 symmetric codes are clamped to [-127, 127], zero-point z = 0;
 *   R3 the code is rint(v * (127/absmax)) with 127/absmax an fp32 division,
 *      never v / scale;
 *   R4 an all-zero vector gets scale 0 and all-zero codes;
 *   R5 weight groups are G contiguous output rows spanning all K columns;
 *   R6 LayerNorm uses the biased variance with eps inside the square root;
 *   R7 GeLU is the exact erf form 0.5 x (1 + erf(x / sqrt 2));
 *   R8 bias is added after dequantization, in floating point.
 *  R14 the smoothing factor is the SmoothQuant paper's balance rule (the
 *      pages name the paper but are cut off before its formula):
 *      s_j = amax_x[j]^alpha / amax_w[j]^(1 - alpha), alpha the migration
 *      strength (0.5 balances both maxima; 1 equalises the activation
 *      channels); computed in double, rounded to fp32, at least 1e-5; a
 *      channel whose activation or weight absmax is 0 keeps s_j = 1;
 *  R15 the activation diag(s)^-1 is folded into the preceding LayerNorm's
 *      gamma and beta (the normalised row is divided per channel), so the
 *      online path is unchanged.
 *  R16 LLM.int8() outliers are detected on the linear's input (after the
 *      LayerNorm) over the whole batch: column j is in O when some
 *      |a[t, j]| >= alpha; at most max_o columns (the lowest indices) are
 *      decomposed; the weights keep their offline group quantization over
 *      all input channels (the outlier channels see zero activation codes);
 *      the outlier operands are rounded to fp16 (round to nearest even) and
 *      multiplied exactly; the outlier product is added to the dequantized
 *      INT8 result before bias and activation.
 *  R17 K-axis weight groups (the other reading of the group-wise paragraph
 *      of [ZQ] and [TS36] §1.2.2, which split W into groups without naming
 *      the axis): a group is one output row o and Gk consecutive input
 *      columns j*Gk .. j*Gk+Gk-1, quantized as one span with scale
 *      s_w[o, j].  The linear then takes each group's exact integer
 *      partial product, scales it by s_w[o, j], sums over j, multiplies by
 *      the token scale and adds bias (all in double, one rounding to fp32).
 *
 * Status codes: 0 = ok, 1 = bad argument, 2 = int32 overflow in the GEMM.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#define ZQO_OK 0
#define ZQO_EARG 1
#define ZQO_EOVERFLOW 2

/* [TS36] §1.1.2 absmax rule + readings R1-R4.  One scale for the n values
 * v[0..n): scale = absmax/127 (fp32), q_i = clamp(rint(v_i * (127/absmax))). */
int zqo_quantize_span(const float* v, int64_t n, int8_t* q, float* scale)
{
    if (!v || !q || !scale || n <= 0) return ZQO_EARG;
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *scale = 0.0f;
        for (int64_t i = 0; i < n; ++i) q[i] = 0;
        return ZQO_OK;
    }
    float s = amax / 127.0f;
    float inv = 127.0f / amax;
    for (int64_t i = 0; i < n; ++i) {
        float t = v[i] * inv;      /* one fp32 rounding, no fused add */
        float r = rintf(t);        /* half-to-even under FE_TONEAREST */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[i] = (int8_t)r;
    }
    *scale = s;
    return ZQO_OK;
}

/* [ZQ] group-wise weight quantization, [TS36] §1.2.2, reading R5.
 * W is [N, K] row-major; group g holds rows g*G .. g*G+G-1 (all K columns)
 * and is quantized as one span.  Wq is [N, K], s_grp is [N/G]. */
int zqo_quantize_weights(const float* W, int64_t N, int64_t K, int64_t G,
                         int8_t* Wq, float* s_grp)
{
    if (!W || !Wq || !s_grp || N <= 0 || K <= 0 || G <= 0 || N % G != 0)
        return ZQO_EARG;
    for (int64_t g = 0; g < N / G; ++g) {
        int rc = zqo_quantize_span(W + g * G * K, G * K, Wq + g * G * K, &s_grp[g]);
        if (rc) return rc;
    }
    return ZQO_OK;
}

/* Dynamic per-token quantization ([ZQ] token-wise paragraph, [TS36] §1.2.2):
 * every row of Y [T, H] gets its own scale. */
int zqo_quantize_rows(const float* Y, int64_t T, int64_t H, int8_t* q, float* s_tok)
{
    if (!Y || !q || !s_tok || T <= 0 || H <= 0) return ZQO_EARG;
    for (int64_t t = 0; t < T; ++t) {
        int rc = zqo_quantize_span(Y + t * H, H, q + t * H, &s_tok[t]);
        if (rc) return rc;
    }
    return ZQO_OK;
}

/* LayerNorm over each row of x [T, H] in double (reading R6), result rounded
 * once to fp32.  mean = sum/H; var = sum (x-mean)^2 / H (two passes);
 * y = (x - mean) / sqrt(var + eps) * gamma + beta. */
int zqo_layernorm(const float* x, int64_t T, int64_t H, const float* gamma,
                  const float* beta, float eps, float* y)
{
    if (!x || !gamma || !beta || !y || T <= 0 || H <= 0) return ZQO_EARG;
    for (int64_t t = 0; t < T; ++t) {
        const float* r = x + t * H;
        double mean = 0.0;
        for (int64_t h = 0; h < H; ++h) mean += (double)r[h];
        mean /= (double)H;
        double var = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            double d = (double)r[h] - mean;
            var += d * d;
        }
        var /= (double)H;
        double denom = sqrt(var + (double)eps);
        for (int64_t h = 0; h < H; ++h) {
            double v = ((double)r[h] - mean) / denom * (double)gamma[h] + (double)beta[h];
            y[t * H + h] = (float)v;
        }
    }
    return ZQO_OK;
}

/* Reading R7: exact GeLU in double. */
static double gelu_d(double v) { return 0.5 * v * (1.0 + erf(v / sqrt(2.0))); }

/* Element-wise activation step before token quantization ([ZQ] fused
 * "LN/GeLU + Quantize" flowchart): y = act(x + bias), bias optional
 * (length H, broadcast over rows), act 0 = identity, 1 = GeLU. */
int zqo_bias_act(const float* x, int64_t T, int64_t H, const float* bias, int act, float* y)
{
    if (!x || !y || T <= 0 || H <= 0 || (act != 0 && act != 1)) return ZQO_EARG;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t h = 0; h < H; ++h) {
            double v = (double)x[t * H + h];
            if (bias) v += (double)bias[h];
            if (act == 1) v = gelu_d(v);
            y[t * H + h] = (float)v;
        }
    return ZQO_OK;
}

/* INT8 x INT8 -> INT32 contraction ([TS36] §1.2.2 "INT32 accumulation";
 * [IQ] MAC unit): acc[t, o] = sum_k xq[t, k] * Wq[o, k].  Accumulated in
 * int64; a sum outside the int32 range is reported, not wrapped. */
int zqo_gemm_i32(const int8_t* xq, int64_t T, int64_t K, const int8_t* Wq, int64_t N,
                 int32_t* acc)
{
    if (!xq || !Wq || !acc || T <= 0 || K <= 0 || N <= 0) return ZQO_EARG;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t o = 0; o < N; ++o) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)xq[t * K + k] * (int64_t)Wq[o * K + k];
            if (s > INT32_MAX || s < INT32_MIN) return ZQO_EOVERFLOW;
            acc[t * N + o] = (int32_t)s;
        }
    return ZQO_OK;
}

/* Dequantize the accumulators ([TS36] §1.2.2: scale the INT32 accumulation
 * by the activation and weight scales; §1.1.2: denormalise by the outer
 * product of the row and column scales; [IQ] "量化模拟" with z = 0), then add
 * bias (reading R8) and apply the optional activation, all in double:
 *   y[t, o] = act(s_tok[t] * s_grp[o / G] * acc[t, o] + bias[o]). */
int zqo_dequant(const int32_t* acc, int64_t T, int64_t N, const float* s_tok,
                const float* s_grp, int64_t G, const float* bias, int act, float* y)
{
    if (!acc || !s_tok || !s_grp || !y || T <= 0 || N <= 0 || G <= 0 || N % G != 0 ||
        (act != 0 && act != 1))
        return ZQO_EARG;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t o = 0; o < N; ++o) {
            double v = (double)s_tok[t] * (double)s_grp[o / G] * (double)acc[t * N + o];
            if (bias) v += (double)bias[o];
            if (act == 1) v = gelu_d(v);
            y[t * N + o] = (float)v;
        }
    return ZQO_OK;
}

/* [SQ] §3 calibration: running per-channel absmax of an activation a [T, H]
 * (the input of the linear): amax[j] = max(amax[j], max_t |a[t, j]|).
 * Max is exact, so no rounding enters. */
int zqo_channel_absmax(const float* a, int64_t T, int64_t H, float* amax)
{
    if (!a || !amax || T <= 0 || H <= 0) return ZQO_EARG;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < H; ++j) {
            float v = fabsf(a[t * H + j]);
            if (v > amax[j]) amax[j] = v;
        }
    return ZQO_OK;
}

/* Per input channel (column j of W [N, K]) absmax: wmax[j] = max_o |W[o, j]|. */
int zqo_weight_col_absmax(const float* W, int64_t N, int64_t K, float* wmax)
{
    if (!W || !wmax || N <= 0 || K <= 0) return ZQO_EARG;
    for (int64_t j = 0; j < K; ++j) wmax[j] = 0.0f;
    for (int64_t o = 0; o < N; ++o)
        for (int64_t j = 0; j < K; ++j) {
            float v = fabsf(W[o * K + j]);
            if (v > wmax[j]) wmax[j] = v;
        }
    return ZQO_OK;
}

/* [TS36] §1.3 / [SQ] §2.2, reading R14: s_j = amax_j^alpha / wmax_j^(1-alpha).
 * alpha is an fp32 parameter (the migration strength as the library's
 * interface passes it); the powers use its exact value in double. */
int zqo_smooth_factors(const float* amax, const float* wmax, int64_t K, float alpha_f, float* s)
{
    const double alpha = (double)alpha_f;
    if (!amax || !wmax || !s || K <= 0 || !(alpha >= 0.0 && alpha <= 1.0)) return ZQO_EARG;
    for (int64_t j = 0; j < K; ++j) {
        if (amax[j] == 0.0f || wmax[j] == 0.0f) {
            s[j] = 1.0f;
            continue;
        }
        double v = pow((double)amax[j], alpha) / pow((double)wmax[j], 1.0 - alpha);
        float f = (float)v;
        s[j] = f < 1e-5f ? 1e-5f : f;
    }
    return ZQO_OK;
}

/* [TS36] §1.3 identity, reading R15: W_out[o, j] = W[o, j] * s_j (each
 * output row scaled per input channel), gamma_out[j] = gamma[j] / s_j,
 * beta_out[j] = beta[j] / s_j; each computed in double and rounded once to
 * fp32 (gamma or beta may be NULL: not folded). */
int zqo_smooth_fold(const float* W, int64_t N, int64_t K, const float* gamma, const float* beta,
                    const float* s, float* W_out, float* gamma_out, float* beta_out)
{
    if (!W || !s || !W_out || N <= 0 || K <= 0) return ZQO_EARG;
    if ((gamma && !gamma_out) || (beta && !beta_out)) return ZQO_EARG;
    for (int64_t o = 0; o < N; ++o)
        for (int64_t j = 0; j < K; ++j) W_out[o * K + j] = (float)((double)W[o * K + j] * (double)s[j]);
    for (int64_t j = 0; j < K; ++j) {
        if (gamma) gamma_out[j] = (float)((double)gamma[j] / (double)s[j]);
        if (beta) beta_out[j] = (float)((double)beta[j] / (double)s[j]);
    }
    return ZQO_OK;
}

/* [TS36] §1.1 outlier detection, reading R16: the columns j with
 * amax[j] >= threshold in ascending order, at most max_o of them written;
 * returns the total count. */
int64_t zqo_outlier_columns(const float* amax, int64_t K, float threshold, int32_t* idx, int64_t max_o)
{
    if (!amax || K <= 0 || max_o < 0 || (max_o > 0 && !idx)) return -1;
    int64_t n = 0;
    for (int64_t j = 0; j < K; ++j)
        if (amax[j] >= threshold) {
            if (n < max_o) idx[n] = (int32_t)j;
            ++n;
        }
    return n;
}

/* IEEE binary16 value nearest to v (ties to even), as a double; overflow
 * goes to infinity, values below the subnormal range to zero. */
static double fp16_round(float v)
{
    double a = fabs((double)v);
    if (a == 0.0 || v != v) return (double)v;
    double r;
    if (a >= 65520.0) {                 /* at or past the midpoint above 65504 */
        r = INFINITY;
    } else {
        int e;
        frexp(a, &e);                   /* a = m * 2^e, m in [0.5, 1) */
        int q = e - 11;                 /* spacing 2^(e-11) for normal halves */
        if (q < -24) q = -24;           /* subnormal spacing 2^-24 */
        double step = ldexp(1.0, q);
        r = nearbyint(a / step) * step; /* exact quotient; default mode is to nearest even */
    }
    return v < 0 ? -r : r;
}

/* [TS36] §1.1 the FP16 part of the decomposition, reading R16:
 * out[t, o] = sum over the first min(cnt, max) listed columns j of
 * fp16(a[t, j]) * fp16(W[o, j]), exact products summed in double. */
int zqo_outlier_product(const float* a, int64_t T, int64_t K, const float* W, int64_t N,
                        const int32_t* idx, int64_t cnt, double* out)
{
    if (!a || !W || !out || T <= 0 || K <= 0 || N <= 0 || cnt < 0 || (cnt > 0 && !idx)) return ZQO_EARG;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t o = 0; o < N; ++o) {
            double acc = 0.0;
            for (int64_t k = 0; k < cnt; ++k) {
                int64_t j = idx[k];
                acc += fp16_round(a[t * K + j]) * fp16_round(W[o * K + j]);
            }
            out[t * N + o] = acc;
        }
    return ZQO_OK;
}

/* The INT8 part dequantized with an extra addend before bias and activation
 * (the decomposition's sum, reading R16): y = act(s_tok s_grp acc + add + b). */
int zqo_dequant_add(const int32_t* acc, int64_t T, int64_t N, const float* s_tok, const float* s_grp,
                    int64_t G, const double* add, const float* bias, int act, float* y)
{
    if (!acc || !s_tok || !s_grp || !y || T <= 0 || N <= 0 || G <= 0 || N % G != 0 ||
        (act != 0 && act != 1))
        return ZQO_EARG;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t o = 0; o < N; ++o) {
            double v = (double)s_tok[t] * (double)s_grp[o / G] * (double)acc[t * N + o];
            if (add) v += add[t * N + o];
            if (bias) v += (double)bias[o];
            if (act == 1) v = gelu_d(v);
            y[t * N + o] = (float)v;
        }
    return ZQO_OK;
}

/* [ZQ] group-wise weight quantization along the input axis, reading R17.
 * W is [N, K] row-major; group (o, j) is W[o, j*Gk .. j*Gk+Gk-1], quantized
 * as one span.  Wq is [N, K]; s_w is [N, K/Gk] row-major. */
int zqo_quantize_weights_kgroups(const float* W, int64_t N, int64_t K, int64_t Gk, int8_t* Wq,
                                 float* s_w)
{
    if (!W || !Wq || !s_w || N <= 0 || K <= 0 || Gk <= 0 || K % Gk != 0) return ZQO_EARG;
    const int64_t ng = K / Gk;
    for (int64_t o = 0; o < N; ++o)
        for (int64_t j = 0; j < ng; ++j) {
            int rc = zqo_quantize_span(W + o * K + j * Gk, Gk, Wq + o * K + j * Gk, &s_w[o * ng + j]);
            if (rc) return rc;
        }
    return ZQO_OK;
}

/* The W8A8 linear with K-axis weight groups (reading R17; the dequantization
 * of [TS36] §1.2.2 applied per group, bias per reading R8):
 *   acc_j[t, o] = sum over k in group j of xq[t, k] * Wq[o, k]   (exact)
 *   y[t, o] = act(s_tok[t] * sum_j s_w[o, j] * acc_j[t, o] + bias[o]). */
int zqo_linear_kgroups(const int8_t* xq, int64_t T, int64_t K, const int8_t* Wq, int64_t N, int64_t Gk,
                       const float* s_tok, const float* s_w, const float* bias, int act, float* y)
{
    if (!xq || !Wq || !s_tok || !s_w || !y || T <= 0 || K <= 0 || N <= 0 || Gk <= 0 || K % Gk != 0 ||
        (act != 0 && act != 1))
        return ZQO_EARG;
    const int64_t ng = K / Gk;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t o = 0; o < N; ++o) {
            double v = 0.0;
            for (int64_t j = 0; j < ng; ++j) {
                int64_t acc = 0;
                for (int64_t k = j * Gk; k < (j + 1) * Gk; ++k)
                    acc += (int64_t)xq[t * K + k] * (int64_t)Wq[o * K + k];
                v += (double)s_w[o * ng + j] * (double)acc;
            }
            v *= (double)s_tok[t];
            if (bias) v += (double)bias[o];
            if (act == 1) v = gelu_d(v);
            y[t * N + o] = (float)v;
        }
    return ZQO_OK;
}
