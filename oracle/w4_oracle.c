/*
 * w4_oracle.c -- plain, slow, obviously-correct CPU reference for weight-only
 * per-group INT4 (W4A16) quantize / pack / dequantize / matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code with the CUDA library.
 *
 * Sources (cited by page and section):
 *   [Accel 2.1]  discosf.com "LLM inference acceleration" article, section 2.1
 *                "what quantization actually does": an affine map of a float
 *                range onto integers through a scale and a zero point, with
 *                per-group granularity (e.g. 128 elements per group).
 *   [Accel 2.2]  same article, section 2.2: INT4 cuts a 70B model from about
 *                140 GB (FP16) to about 35 GB.
 *   [Accel 2.3]  same article, section 2.3: scale and zero_point are loaded
 *                together with the weights ("dequantize mapping").
 *   [Ch22 22.3]  aiwing.uk chapter 22 "Advanced inference optimisation",
 *                section 22.3 "Model quantization": bytes-per-parameter table
 *                (INT4 = 0.5 B), weight-only quantization (dequantize back to
 *                FP16 then matmul), and the AWQ equation W^ = quant(W/s) * s.
 *
 *   [Notes 2.1]  mhpq.cn practitioner's article, section 2.1: INT4 weights take
 *                values in the symmetric set {-7, ..., 7} (the symmetric variant).
 *
 * Readings taken where the pages are silent (each one is exercised by a test):
 *   - codes are asymmetric uint4 in [0,15]; one fp16 scale and one fp16 zero
 *     point per group of G = 128 consecutive input channels (k) of a row n;
 *   - every step runs in IEEE fp32 with round-to-nearest-even; rint() is
 *     round-half-to-even; scale = fp16((max - min) / 15), and z and q are
 *     computed with that fp16-rounded scale widened back to fp32, so the
 *     stored (scale, zero) describe exactly the grid that was used;
 *   - z = clamp(rint(-min / scale), 0, 15); q = clamp(rint(w / scale) + z, 0, 15)
 *     (rint first, then add z);
 *   - degenerate group: if the fp16 scale is 0 (max == min, or fp16
 *     underflow) the scale is taken as 1.0;
 *   - packing: two codes per byte, low nibble = even k, high nibble = odd k;
 *   - dequant: w^ = ((float)q - z) * scale * s[k], fp32, left to right;
 *   - matmul: y[m][n] = sum_k x[m][k] * w^[n][k], accumulated in fp64 in
 *     increasing k; bound[m][n] = sum_k |x[m][k] * w^[n][k]|.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* fp32 -> IEEE binary16, round-to-nearest-even (compiler conversion). */
static uint16_t f32_to_f16_bits(float v) {
    _Float16 h = (_Float16)v;
    uint16_t b;
    memcpy(&b, &h, sizeof b);
    return b;
}

static float f16_bits_to_f32(uint16_t b) {
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return (float)h;
}

/* Exposed so the tests can pin the conversion against an independent one. */
uint16_t w4o_f32_to_f16(float v) { return f32_to_f16_bits(v); }
float w4o_f16_to_f32(uint16_t b) { return f16_bits_to_f32(b); }

/* clamp to [0, 15]; codes and zero points are integers, so -0 clamps to +0
 * (IEEE 754-2019 maximum orders -0 below +0). */
static float clamp_0_15(float v) {
    if (!(v > 0.0f)) return 0.0f;
    if (v > 15.0f) return 15.0f;
    return v;
}

/*
 * Quantize W [N][K] (fp32, row-major) group by group [Accel 2.1], with the
 * optional AWQ per-input-channel scale s [K] applied as W / s first
 * [Ch22 22.3, AWQ equation].  Outputs: codes [N][K] (one code per byte),
 * scales [N][K/G] and zeros [N][K/G] as fp16 bit patterns.
 * Returns 0, or -1 for arguments it cannot serve.
 */
int w4o_quantize(const float *W, const float *awq_s, int64_t N, int64_t K,
                 int group, uint8_t *codes, uint16_t *scales, uint16_t *zeros) {
    if (N < 0 || K < 0 || group <= 0 || K % group != 0) return -1;
    fesetround(FE_TONEAREST);
    const int64_t Kg = K / group;
    float wp[1024];
    if (group > 1024) return -1;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < Kg; ++g) {
            const int64_t k0 = g * group;
            /* step 1: AWQ prescale w' = w / s[k] (IEEE division) */
            for (int i = 0; i < group; ++i) {
                float w = W[n * K + k0 + i];
                wp[i] = awq_s ? w / awq_s[k0 + i] : w;
            }
            /* step 2: group min and max */
            float mn = wp[0], mx = wp[0];
            for (int i = 1; i < group; ++i) {
                if (wp[i] < mn) mn = wp[i];
                if (wp[i] > mx) mx = wp[i];
            }
            /* step 3: scale = fp16((max - min) / 15); degenerate -> 1.0 */
            float sc32 = (mx - mn) / 15.0f;
            uint16_t sc_bits = f32_to_f16_bits(sc32);
            float sc = f16_bits_to_f32(sc_bits);
            if (sc == 0.0f) {
                sc = 1.0f;
                sc_bits = f32_to_f16_bits(1.0f);
            }
            /* step 4: zero point z = clamp(rint(-min / scale), 0, 15) */
            float z = clamp_0_15(rintf(-mn / sc));
            scales[n * Kg + g] = sc_bits;
            zeros[n * Kg + g] = f32_to_f16_bits(z);
            /* step 5: codes q = clamp(rint(w' / scale) + z, 0, 15) */
            for (int i = 0; i < group; ++i) {
                float q = clamp_0_15(rintf(wp[i] / sc) + z);
                codes[n * K + k0 + i] = (uint8_t)q;
            }
        }
    }
    return 0;
}

/* clamp to [-7, 7] */
static float clamp_pm7(float v) {
    if (v < -7.0f) return -7.0f;
    if (v > 7.0f) return 7.0f;
    return v;
}

/*
 * Symmetric variant: INT4 as the symmetric value set {-7, ..., 7} ([Notes 2.1]:
 * mhpq.cn practitioner's article, section 2.1).  The page gives the value set
 * only; the scale rule taken here is the plain symmetric one:
 *   amax  = max |w'| over the group
 *   scale = fp16(amax / 7), taken as 1.0 if that is 0
 *   q     = clamp(rint(w' / scale), -7, 7)
 * and the code stored is q + 8 (1..15) with zero point 8, so the asymmetric
 * dequantization ((float)code - z) * scale gives q * scale unchanged.
 */
int w4o_quantize_sym(const float *W, const float *awq_s, int64_t N, int64_t K,
                     int group, uint8_t *codes, uint16_t *scales, uint16_t *zeros) {
    if (N < 0 || K < 0 || group <= 0 || K % group != 0) return -1;
    fesetround(FE_TONEAREST);
    const int64_t Kg = K / group;
    float wp[1024];
    if (group > 1024) return -1;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < Kg; ++g) {
            const int64_t k0 = g * group;
            for (int i = 0; i < group; ++i) {
                float w = W[n * K + k0 + i];
                wp[i] = awq_s ? w / awq_s[k0 + i] : w;
            }
            float amax = 0.0f;
            for (int i = 0; i < group; ++i) {
                float a = fabsf(wp[i]);
                if (a > amax) amax = a;
            }
            float sc32 = amax / 7.0f;
            uint16_t sc_bits = f32_to_f16_bits(sc32);
            float sc = f16_bits_to_f32(sc_bits);
            if (sc == 0.0f) {
                sc = 1.0f;
                sc_bits = f32_to_f16_bits(1.0f);
            }
            scales[n * Kg + g] = sc_bits;
            zeros[n * Kg + g] = f32_to_f16_bits(8.0f);
            for (int i = 0; i < group; ++i) {
                float q = clamp_pm7(rintf(wp[i] / sc));
                codes[n * K + k0 + i] = (uint8_t)(q + 8.0f);
            }
        }
    }
    return 0;
}

/*
 * Pack codes [N][K] into bytes [N][K/2]: byte j of a row holds the code of
 * k = 2j in its low nibble and of k = 2j+1 in its high nibble (0.5 byte per
 * parameter, [Ch22 22.3] table).  Codes above 15 are masked to 4 bits.
 */
int w4o_pack(const uint8_t *codes, int64_t N, int64_t K, uint8_t *packed) {
    if (N < 0 || K < 0 || K % 2 != 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 2; ++j) {
            uint8_t lo = codes[n * K + 2 * j] & 0x0F;
            uint8_t hi = codes[n * K + 2 * j + 1] & 0x0F;
            packed[n * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
    return 0;
}

/* Inverse of w4o_pack. */
int w4o_unpack(const uint8_t *packed, int64_t N, int64_t K, uint8_t *codes) {
    if (N < 0 || K < 0 || K % 2 != 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 2; ++j) {
            uint8_t b = packed[n * (K / 2) + j];
            codes[n * K + 2 * j] = b & 0x0F;
            codes[n * K + 2 * j + 1] = b >> 4;
        }
    return 0;
}

/*
 * Dequantize: w^[n][k] = ((float)q - z) * scale * s[k] in fp32, left to
 * right (weight-only path, [Ch22 22.3]; AWQ re-multiplies by s).
 */
int w4o_dequant(const uint8_t *codes, const uint16_t *scales,
                const uint16_t *zeros, const float *awq_s, int64_t N,
                int64_t K, int group, float *What) {
    if (N < 0 || K < 0 || group <= 0 || K % group != 0) return -1;
    fesetround(FE_TONEAREST);
    const int64_t Kg = K / group;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float sc = f16_bits_to_f32(scales[n * Kg + k / group]);
            float z = f16_bits_to_f32(zeros[n * Kg + k / group]);
            float t = (float)codes[n * K + k] - z;
            float w = t * sc;
            if (awq_s) w = w * awq_s[k];
            What[n * K + k] = w;
        }
    return 0;
}

/*
 * Y = X . W^T with X [M][K] and W^ [N][K] given as fp32 (fp16/bf16 inputs
 * widen exactly), accumulated in fp64 in increasing k.  bound[m][n] receives
 * sum_k |x * w^| (the scale of the tolerance).  Either output may be NULL.
 */
int w4o_gemm(const float *X, const float *What, int64_t M, int64_t N,
             int64_t K, double *Y, double *bound) {
    if (M < 0 || N < 0 || K < 0) return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, abs_acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)X[m * K + k] * (double)What[n * K + k];
                acc += p;
                abs_acc += fabs(p);
            }
            if (Y) Y[m * N + n] = acc;
            if (bound) bound[m * N + n] = abs_acc;
        }
    return 0;
}

/*
 * AWQ scale search.  AWQ takes a per-input-channel activation magnitude s from
 * calibration data and quantizes W / s ([Ch22 22.3], AWQ); the quality
 * measure of a quantized layer is its output error on calibration activations,
 * || X W^T - X W^^T ||_F^2 ([Ch22 22.3], the objective stated for GPTQ).
 * Reading taken (the page gives no formula for s): s_k = m_k^a with
 * m_k = mean over the calibration rows of |x_k| (fp64), rounded to fp32 (1 where
 * m_k = 0), and the exponent a is the one of the given grid with the smallest
 * error (the first one on ties).
 *
 * X [Mc][K] holds the calibration activations as floats; W [N][K] fp32.
 * Outputs: errors [n_alpha] (fp64), s_out [K] for the best exponent, *best.
 * Plain loops: the error of each exponent is the fp64 sum of squared
 * differences between the fp64 products X W^T and X W^^T.
 */
int w4o_awq_search(const float *W, int64_t N, int64_t K, int group,
                   const float *X, int64_t Mc, const double *alphas,
                   int n_alpha, double *errors, float *s_out, int *best) {
    if (N < 1 || K < 1 || Mc < 1 || n_alpha < 1 || group <= 0 || K % group != 0) return -1;
    double *m = (double *)malloc(sizeof(double) * (size_t)K);
    float *s = (float *)malloc(sizeof(float) * (size_t)K);
    uint8_t *codes = (uint8_t *)malloc((size_t)(N * K));
    uint16_t *sc = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(N * (K / group)));
    uint16_t *zp = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(N * (K / group)));
    float *What = (float *)malloc(sizeof(float) * (size_t)(N * K));
    double *Yref = (double *)malloc(sizeof(double) * (size_t)(Mc * N));
    double *Yq = (double *)malloc(sizeof(double) * (size_t)(Mc * N));
    int rc = -1;
    if (!m || !s || !codes || !sc || !zp || !What || !Yref || !Yq) goto done;
    for (int64_t k = 0; k < K; ++k) {
        double acc = 0.0;
        for (int64_t r = 0; r < Mc; ++r) acc += fabs((double)X[r * K + k]);
        m[k] = acc / (double)Mc;
    }
    w4o_gemm(X, W, Mc, N, K, Yref, NULL);
    int arg = 0;
    for (int i = 0; i < n_alpha; ++i) {
        for (int64_t k = 0; k < K; ++k) s[k] = m[k] > 0.0 ? (float)pow(m[k], alphas[i]) : 1.0f;
        w4o_quantize(W, s, N, K, group, codes, sc, zp);
        w4o_dequant(codes, sc, zp, s, N, K, group, What);
        w4o_gemm(X, What, Mc, N, K, Yq, NULL);
        double e = 0.0;
        for (int64_t j = 0; j < Mc * N; ++j) {
            double d = Yref[j] - Yq[j];
            e += d * d;
        }
        errors[i] = e;
        if (e < errors[arg]) arg = i;
    }
    for (int64_t k = 0; k < K; ++k) s_out[k] = m[k] > 0.0 ? (float)pow(m[k], alphas[arg]) : 1.0f;
    *best = arg;
    rc = 0;
done:
    free(m); free(s); free(codes); free(sc); free(zp); free(What); free(Yref); free(Yq);
    return rc;
}

/*
 * GPTQ ([Ch22 22.3]: a layer's weights are quantized so as to minimize
 * || W X - W^ X ||_F^2 on calibration inputs X, using the Hessian H = 2 X X^T to
 * order the work and to compensate each weight's quantization error on the
 * weights not yet quantized -- the Optimal Brain Compression idea).  The page
 * gives no algorithm beyond that; the reading taken is the standard column
 * sweep, in plain fp64 loops (no fused multiply-add):
 *   H[a][b] = 2 sum_m x[m][a] x[m][b]  (m increasing);  H[a][a] += damp,
 *   damp = damp_frac * (sum_a H[a][a]) / K  (a increasing);
 *   U = the upper Cholesky factor of H^-1, computed as P inv(L') P with
 *   L' the lower Cholesky factor of P H P (P reverses the order of k);
 *   for each row, for k = 0..K-1 in order: at the start of each group, its
 *   scale and zero point come from the current (updated) weights by the rule of
 *   w4o_quantize (in fp32); q = the rounded code of the current weight,
 *   err = (w - w^) / U[k][k], and every later weight of the row moves by
 *   w[k'] -= err * U[k][k'].
 * X [Mc][K] floats (the calibration activations), W [N][K] fp32.
 * Outputs as for w4o_quantize.  Returns 0, -1 on bad arguments, -2 if H is not
 * positive definite.
 */
int w4o_gptq(const float *W, int64_t N, int64_t K, int group, const float *X,
             int64_t Mc, double damp_frac, uint8_t *codes, uint16_t *scales,
             uint16_t *zeros) {
    if (N < 1 || K < 1 || Mc < 1 || group <= 0 || K % group != 0 || group > 1024) return -1;
    fesetround(FE_TONEAREST);
    const int64_t Kg = K / group;
    double *H = (double *)malloc(sizeof(double) * (size_t)(K * K));
    double *L = (double *)calloc((size_t)(K * K), sizeof(double));
    double *Li = (double *)calloc((size_t)(K * K), sizeof(double));
    double *w = (double *)malloc(sizeof(double) * (size_t)K);
    int rc = -1;
    if (!H || !L || !Li || !w) goto out;
    /* H = 2 X^T X, then damping */
    for (int64_t a = 0; a < K; ++a)
        for (int64_t b = 0; b < K; ++b) {
            double acc = 0.0;
            for (int64_t m = 0; m < Mc; ++m) acc = acc + (double)X[m * K + a] * (double)X[m * K + b];
            H[a * K + b] = 2.0 * acc;
        }
    {
        double tr = 0.0;
        for (int64_t a = 0; a < K; ++a) tr = tr + H[a * K + a];
        const double damp = damp_frac * (tr / (double)K);
        for (int64_t a = 0; a < K; ++a) H[a * K + a] = H[a * K + a] + damp;
    }
    /* L = lower Cholesky factor of R = P H P, R[i][j] = H[K-1-i][K-1-j] (left-looking) */
    for (int64_t j = 0; j < K; ++j) {
        double d = H[(K - 1 - j) * K + (K - 1 - j)];
        for (int64_t k = 0; k < j; ++k) d = d - L[j * K + k] * L[j * K + k];
        if (!(d > 0.0)) { rc = -2; goto out; }
        const double ljj = sqrt(d);
        L[j * K + j] = ljj;
        for (int64_t i = j + 1; i < K; ++i) {
            double acc = H[(K - 1 - i) * K + (K - 1 - j)];
            for (int64_t k = 0; k < j; ++k) acc = acc - L[i * K + k] * L[j * K + k];
            L[i * K + j] = acc / ljj;
        }
    }
    /* Li = inverse of L (lower), column by column */
    for (int64_t c = 0; c < K; ++c) {
        Li[c * K + c] = 1.0 / L[c * K + c];
        for (int64_t i = c + 1; i < K; ++i) {
            double acc = 0.0;
            for (int64_t k = c; k < i; ++k) acc = acc + L[i * K + k] * Li[k * K + c];
            Li[i * K + c] = -acc / L[i * K + i];
        }
    }
    /* U[j][k] = Li[K-1-j][K-1-k]; sweep each row */
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) w[k] = (double)W[n * K + k];
        float sc = 1.0f, z = 0.0f;
        for (int64_t j = 0; j < K; ++j) {
            if (j % group == 0) {
                float mn = (float)w[j], mx = (float)w[j];
                for (int64_t i = 1; i < group; ++i) {
                    const float v = (float)w[j + i];
                    if (v < mn) mn = v;
                    if (v > mx) mx = v;
                }
                uint16_t sc_bits = f32_to_f16_bits((mx - mn) / 15.0f);
                sc = f16_bits_to_f32(sc_bits);
                if (sc == 0.0f) {
                    sc = 1.0f;
                    sc_bits = f32_to_f16_bits(1.0f);
                }
                z = clamp_0_15(rintf(-mn / sc));
                scales[n * Kg + j / group] = sc_bits;
                zeros[n * Kg + j / group] = f32_to_f16_bits(z);
            }
            const float q = clamp_0_15(rintf((float)w[j] / sc) + z);
            codes[n * K + j] = (uint8_t)q;
            const float wq = (q - z) * sc;
            const double ujj = Li[(K - 1 - j) * K + (K - 1 - j)];
            const double err = (w[j] - (double)wq) / ujj;
            for (int64_t k = j + 1; k < K; ++k) w[k] = w[k] - err * Li[(K - 1 - j) * K + (K - 1 - k)];
        }
    }
    rc = 0;
out:
    free(H); free(L); free(Li); free(w);
    return rc;
}
