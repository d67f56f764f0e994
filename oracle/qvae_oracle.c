/*
 * qvae_oracle.c -- plain CPU definition of the W8A8 CausalConv3d layer.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA path and must stay slow and
 * obviously correct: every function is the definition written out, with no
 * blocking, fusion or reordering.
 *
 * What it follows (ComfyUI-Qwen-VAE-Triton v0.2.0 release note, sd114.wiki):
 *   - section "three presets": weights are symmetric INT8 with one scale per
 *     output channel; activations are dynamic symmetric INT8; products are
 *     INT8 x INT8 accumulated in INT32, rescaled in FP32, and the output keeps
 *     the activation's original precision (bf16 here);
 *   - same section, "fixed internal parameters": activation and weight clip
 *     ratios are 1.0, channels_last layout;
 *   - opening paragraph: the layer is a CausalConv3d (implicit-GEMM lowering
 *     is only how the kernel evaluates it; the result is the plain sum below).
 * Readings where the page is silent:
 *   - activation scale is per tensor; scale = absmax / 127 (IEEE fp32 divide);
 *   - code = clamp(rint(v / scale), -127, 127), rint = round half to even,
 *     v / scale an IEEE fp32 divide; absmax == 0 gives scale 0 and all codes 0;
 *   - causal padding is two leading zero frames (kernel slice kt = 2 meets
 *     frame t, kt = 0 meets frame t - 2), spatial padding 1, stride 1, 3x3x3;
 *   - epilogue: y = float(acc) * (s_a * s_w[co]), then y + float(bias[co]) as
 *     a separate add (no fused multiply-add), then bf16 round-to-nearest-even;
 *   - streamed temporal decode (the release note names the Wan VAE; chunking
 *     is a reading): a chunk's input carries the previous chunk's last two
 *     input frames in place of the zero frames, quantised with the chunk;
 *   - row bands: codes of every band are taken with the whole image's
 *     maximum (oracle_act_quant_amax), so bands reproduce the whole image;
 *   - native-precision layers (the two the Aggressive preset keeps): the
 *     exact convolution of the bf16 values plus bias, rounded once to bf16
 *     (oracle_conv_bf16, oracle_f64_to_bf16).
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -shared -fPIC (see build.py).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_NONFINITE 1
#define ORC_ERR_OVERFLOW 2
#define ORC_ERR_ARG 3

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even (inputs are finite). */
static uint16_t float_to_bf16_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) /* NaN: keep it quiet */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

uint16_t oracle_f32_to_bf16(float f) { return float_to_bf16_bits(f); }

/* One INT8 code: clamp(rint(v / s), -127, 127); s == 0 maps to code 0. */
static int8_t quantize_one(float v, float s)
{
    if (s == 0.0f)
        return 0;
    float r = rintf(v / s);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/*
 * Weight quantisation, per output channel.
 * w: bf16 bits, PyTorch Conv3d weight [Cout][Cin][3][3][3] (contiguous).
 * qw: INT8 codes in the same layout.  s_w: [Cout] fp32 scales.
 */
int oracle_quantize_weights(const uint16_t *w, int32_t Cout, int32_t Cin,
                            int8_t *qw, float *s_w)
{
    if (Cout <= 0 || Cin <= 0) return ORC_ERR_ARG;
    const int64_t per_co = (int64_t)Cin * 27;
    for (int32_t co = 0; co < Cout; ++co) {
        const uint16_t *wc = w + (int64_t)co * per_co;
        float amax = 0.0f;
        for (int64_t i = 0; i < per_co; ++i) {
            float v = bf16_bits_to_float(wc[i]);
            if (!isfinite(v)) return ORC_ERR_NONFINITE;
            float a = fabsf(v);
            if (a > amax) amax = a;
        }
        amax = amax * 1.0f;          /* weight clip ratio 1.0 */
        float s = amax / 127.0f;
        s_w[co] = s;
        for (int64_t i = 0; i < per_co; ++i)
            qw[(int64_t)co * per_co + i] = quantize_one(bf16_bits_to_float(wc[i]), s);
    }
    return ORC_OK;
}

/* Per-tensor absmax of a bf16 tensor (any layout; every element counts). */
int oracle_act_absmax(const uint16_t *x, int64_t numel, float *amax_out)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < numel; ++i) {
        float v = bf16_bits_to_float(x[i]);
        if (!isfinite(v)) return ORC_ERR_NONFINITE;
        float a = fabsf(v);
        if (a > amax) amax = a;
    }
    *amax_out = amax;
    return ORC_OK;
}

/*
 * Dynamic per-tensor activation quantisation.
 * x: bf16 bits, numel elements.  qx: INT8 codes, same order.  s_a: scale.
 * oracle_act_quant_amax takes the maximum |x| from the caller: the maximum
 * over a larger tensor of which x is a part (the row bands of one image);
 * the codes of every part then equal those of the whole tensor.
 */
int oracle_act_quant_amax(const uint16_t *x, int64_t numel, float amax, int8_t *qx, float *s_a)
{
    amax = amax * 1.0f;              /* activation clip ratio 1.0 */
    float s = amax / 127.0f;
    *s_a = s;
    for (int64_t i = 0; i < numel; ++i) {
        float v = bf16_bits_to_float(x[i]);
        if (!isfinite(v)) return ORC_ERR_NONFINITE;
        qx[i] = quantize_one(v, s);
    }
    return ORC_OK;
}

int oracle_act_quant(const uint16_t *x, int64_t numel, int8_t *qx, float *s_a)
{
    float amax;
    int rc = oracle_act_absmax(x, numel, &amax);
    if (rc != ORC_OK) return rc;
    return oracle_act_quant_amax(x, numel, amax, qx, s_a);
}

/*
 * The causal 3x3x3 convolution of the codes, accumulated exactly.
 * One output point (n, t, h, w, co):
 *   acc = sum over kt, kh, kw in {0,1,2} and ci of
 *         qx[n, t + kt - 2, h + kh - 1, w + kw - 1, ci] * qw[co, ci, kt, kh, kw]
 * where any input index outside the tensor contributes zero (two leading
 * zero frames in time, one zero pixel on each spatial side).
 * qx: [N][T][H][W][Cin] (channels_last); qw: [Cout][Cin][3][3][3].
 */
static int conv_point(const int8_t *qx, const int8_t *qw, int64_t T, int64_t hist,
                      int64_t H, int64_t W, int32_t Cin, int64_t n, int64_t t, int64_t h,
                      int64_t w, int32_t co, int32_t *out)
{
    /* The input holds hist + T frames: hist carried frames, then the T frames
     * of this call.  Output frame t reads input frames t + kt - 2 + hist for
     * kt = 0, 1, 2; a frame before the first one is a causal zero frame. */
    const int64_t Tin = T + hist;
    int64_t acc = 0;
    for (int kt = 0; kt < 3; ++kt) {
        int64_t ti = t + kt - 2 + hist;
        if (ti < 0 || ti >= Tin) continue;
        for (int kh = 0; kh < 3; ++kh) {
            int64_t hi = h + kh - 1;
            if (hi < 0 || hi >= H) continue;
            for (int kw = 0; kw < 3; ++kw) {
                int64_t wi = w + kw - 1;
                if (wi < 0 || wi >= W) continue;
                const int8_t *xp = qx + ((((n * Tin + ti) * H + hi) * W + wi) * Cin);
                for (int32_t ci = 0; ci < Cin; ++ci) {
                    int64_t widx = ((((int64_t)co * Cin + ci) * 3 + kt) * 3 + kh) * 3 + kw;
                    acc += (int64_t)xp[ci] * (int64_t)qw[widx];
                }
            }
        }
    }
    if (acc > INT32_MAX || acc < INT32_MIN) return ORC_ERR_OVERFLOW;
    *out = (int32_t)acc;
    return ORC_OK;
}

/* Every output point of a call whose input carries `hist` frames of history
 * (qx: [N][hist + T][H][W][Cin]); acc: [N][T][H][W][Cout]. */
static int conv_acc_hist(const int8_t *qx, const int8_t *qw, int64_t N, int64_t T, int64_t hist,
                         int64_t H, int64_t W, int32_t Cin, int32_t Cout, int32_t *acc)
{
    if (N <= 0 || T <= 0 || H <= 0 || W <= 0 || Cin <= 0 || Cout <= 0) return ORC_ERR_ARG;
    int rc_all = ORC_OK;
    const int64_t rows = N * T * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t n = r / (T * H), t = (r / H) % T, h = r % H;
        for (int64_t w = 0; w < W; ++w)
            for (int32_t co = 0; co < Cout; ++co) {
                int32_t v = 0;
                int rc = conv_point(qx, qw, T, hist, H, W, Cin, n, t, h, w, co, &v);
                if (rc != ORC_OK) {
#pragma omp atomic write
                    rc_all = rc;
                }
                acc[(((n * T + t) * H + h) * W + w) * Cout + co] = v;
            }
    }
    return rc_all;
}

/* Every output point of the causal conv (two zero frames before frame 0);
 * qx: [N][T][H][W][Cin], acc: [N][T][H][W][Cout]. */
int oracle_conv_acc(const int8_t *qx, const int8_t *qw, int64_t N, int64_t T,
                    int64_t H, int64_t W, int32_t Cin, int32_t Cout, int32_t *acc)
{
    return conv_acc_hist(qx, qw, N, T, 0, H, W, Cin, Cout, acc);
}

/* Streaming decode of a chunk of T frames: the two frames before it are the
 * last two input frames of the previous chunk (carried), not zeros.
 * qx_ext: [N][T + 2][H][W][Cin] (carried frames first), acc: [N][T][H][W][Cout]. */
int oracle_conv_acc_carry(const int8_t *qx_ext, const int8_t *qw, int64_t N, int64_t T,
                          int64_t H, int64_t W, int32_t Cin, int32_t Cout, int32_t *acc)
{
    return conv_acc_hist(qx_ext, qw, N, T, 2, H, W, Cin, Cout, acc);
}

/* Selected output pixels only; pts: [npts][4] = (n, t, h, w); acc: [npts][Cout]. */
int oracle_conv_acc_points(const int8_t *qx, const int8_t *qw, int64_t N, int64_t T,
                           int64_t H, int64_t W, int32_t Cin, int32_t Cout,
                           const int64_t *pts, int64_t npts, int32_t *acc)
{
    int rc_all = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npts; ++p) {
        const int64_t *q = pts + 4 * p;
        int bad = q[0] < 0 || q[0] >= N || q[1] < 0 || q[1] >= T || q[2] < 0 ||
                  q[2] >= H || q[3] < 0 || q[3] >= W;
        for (int32_t co = 0; co < Cout; ++co) {
            int32_t v = 0;
            int rc = bad ? ORC_ERR_ARG
                         : conv_point(qx, qw, T, 0, H, W, Cin, q[0], q[1], q[2], q[3], co, &v);
            if (rc != ORC_OK) {
#pragma omp atomic write
                rc_all = rc;
            }
            acc[p * Cout + co] = v;
        }
    }
    return rc_all;
}

/*
 * FP32 rescale, bias, cast back to bf16.
 * acc: [M][Cout]; s_w: [Cout]; bias: bf16 bits [Cout] or NULL (zero bias).
 */
void oracle_epilogue(const int32_t *acc, int64_t M, int32_t Cout, float s_a,
                     const float *s_w, const uint16_t *bias, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int32_t co = 0; co < Cout; ++co) {
            float scale = s_a * s_w[co];
            float y = (float)acc[m * Cout + co] * scale;
            float b = bias ? bf16_bits_to_float(bias[co]) : 0.0f;
            y = y + b;
            out[m * Cout + co] = float_to_bf16_bits(y);
        }
}

/*
 * Native-precision layer.  The release note's Aggressive preset quantises 26
 * of the 28 decoder convolutions and keeps two (decoder.upsamples.14.residual.2
 * and .residual.6, the full-resolution 96-channel stage) in their original
 * precision: the same causal 3x3x3 convolution evaluated on the bf16 values
 * themselves.  Written out exactly:
 *   y[n,t,h,w,co] = bias[co] + sum over kt,kh,kw,ci of
 *                   x[n, t+kt-2, h+kh-1, w+kw-1, ci] * w[co, ci, kt, kh, kw]
 * with zero outside the tensor, as for the quantised layer.  Each bf16 x bf16
 * product has at most 16 significant bits, so it is exact in binary64, and
 * the sum of at most 27*Cin + 1 such terms is kept in binary64 (its own
 * rounding is below 2^-40 of the magnitudes involved).  s_abs receives the
 * sum of the magnitudes of the same terms, bias included: the scale of the
 * error that any binary32 evaluation of the sum can make.
 * x: bf16 bits [N][T][H][W][Cin]; w: bf16 bits [Cout][Cin][3][3][3];
 * bias: bf16 bits [Cout] or NULL; y, s_abs: [N][T][H][W][Cout].
 */
int oracle_conv_bf16(const uint16_t *x, const uint16_t *w, const uint16_t *bias, int64_t N,
                     int64_t T, int64_t H, int64_t W, int32_t Cin, int32_t Cout, double *y,
                     double *s_abs)
{
    if (N <= 0 || T <= 0 || H <= 0 || W <= 0 || Cin <= 0 || Cout <= 0) return ORC_ERR_ARG;
    const int64_t rows = N * T * H;
    int rc_all = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t n = r / (T * H), t = (r / H) % T, h = r % H;
        for (int64_t wo = 0; wo < W; ++wo)
            for (int32_t co = 0; co < Cout; ++co) {
                double b = bias ? (double)bf16_bits_to_float(bias[co]) : 0.0;
                double sum = b, mag = fabs(b);
                for (int kt = 0; kt < 3; ++kt) {
                    int64_t ti = t + kt - 2;
                    if (ti < 0) continue;
                    for (int kh = 0; kh < 3; ++kh) {
                        int64_t hi = h + kh - 1;
                        if (hi < 0 || hi >= H) continue;
                        for (int kw = 0; kw < 3; ++kw) {
                            int64_t wi = wo + kw - 1;
                            if (wi < 0 || wi >= W) continue;
                            const uint16_t *xp = x + (((n * T + ti) * H + hi) * W + wi) * Cin;
                            for (int32_t ci = 0; ci < Cin; ++ci) {
                                int64_t widx = ((((int64_t)co * Cin + ci) * 3 + kt) * 3 + kh) * 3 + kw;
                                double xv = (double)bf16_bits_to_float(xp[ci]);
                                double wv = (double)bf16_bits_to_float(w[widx]);
                                if (!isfinite(xv) || !isfinite(wv)) {
#pragma omp atomic write
                                    rc_all = ORC_ERR_NONFINITE;
                                }
                                sum += xv * wv;
                                mag += fabs(xv * wv);
                            }
                        }
                    }
                }
                int64_t o = (((n * T + t) * H + h) * W + wo) * Cout + co;
                y[o] = sum;
                s_abs[o] = mag;
            }
    }
    return rc_all;
}

/*
 * binary64 -> bf16, round to nearest, ties to even, in one rounding (going
 * through binary32 first could round twice).  v finite and below the bf16
 * overflow threshold.  The two bf16 neighbours of |v| are found by scaling
 * with the spacing of bf16 values at that magnitude (8 significant bits, or
 * the subnormal spacing 2^-133), both exact operations in binary64.
 */
static uint16_t double_to_bf16_bits(double v)
{
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    int e;
    frexp(a, &e);                       /* a in [2^(e-1), 2^e) */
    int q = e - 8;
    if (q < -133) q = -133;
    double ulp = ldexp(1.0, q);
    double k = floor(a / ulp);          /* a / ulp is exact (a power-of-two scaling) */
    double lo = k * ulp, rem = a - lo;  /* both exact */
    double pick;
    if (rem < ulp / 2) pick = lo;
    else if (rem > ulp / 2) pick = lo + ulp;
    else pick = (fmod(k, 2.0) == 0.0) ? lo : lo + ulp;
    float f = (float)pick;              /* exact: pick has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)((u >> 16) | (signbit(v) ? 0x8000u : 0u));
}

void oracle_f64_to_bf16(const double *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16_bits(v[i]);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
