/*
 * oracle.c -- plain, slow CPU reference for the quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may link,
 * load or call this file.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library: every routine here is written out from the
 * definitions on the source pages, with plain loops, fp32 where the pages fix
 * the arithmetic of a quantisation decision and double accumulation for every
 * dot product.
 *
 * Sources (cited by page title and section):
 *   [QL]  docs.rs nuvec-nn 0.1.0, "Struct QuantizedLinear" -- fields weight /
 *         scales / biases / bias / group_size / bits, and the methods
 *         from_linear, dequantized_weight, forward.
 *   [PG]  cider/ops.py, pergroup_linear docstring -- the affine quantize and
 *         dequantize formulas  q = clip(round((w - bias)/scale), 0, 2^b - 1),
 *         w = q*scale + bias.
 *   [BL]  mlx_lm/models/bitlinear_layers.py, make_bitlinear_kernel (kernel
 *         source) and class BitLinear (__init__, execute_matmul_kernel,
 *         __call__).
 *   [Q8]  cider/ops.py, quantize_weight_int8.
 *   [P4]  cider/ops.py, pack_weight_int4.
 *   [PC]  cider/ops.py, perchannel_linear (W8A8).
 *   [W4]  cider/ops.py, w4a8_linear (W4A8).
 *   [I8]  cider/ops.py, int8_matmul_int32.
 *   [PG]  also: cider/ops.py, pergroup_linear (Args and Dispatches
 *         paragraphs) -- per-group symmetric INT8 weights w [N, K], scales
 *         scale_w [num_groups, N] indexed scale_w[g * N + n], group size 64 /
 *         128 / 256, and the dispatch M > 1 -> activation quantize + INT8
 *         GEMM, M == 1 -> FP activation with the weights dequantised.
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes): round() is round-half-to-even (numpy's rule, and rintf under the
 * default rounding mode); scale and bias of an affine group are chosen by
 * min-max (scale = (max-min)/(2^b-1), bias = min); a zero scale becomes 1.0
 * (the rule the cider helpers use); the stored (possibly bf16-rounded) scale
 * and bias are the ones the codes are computed from; codes are packed
 * LSB-first into uint32 words, element k of a row at bit b*(k mod 32/b) of
 * word k*b/32; the undefined activation quantiser quant_a is the per-row
 * int8 rule of quantize_weight_int8 applied to each token row of x.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 * Return values: 0 on success, a negative number for an invalid argument.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define ORC_EINVAL (-1)
#define ORC_EOVERFLOW (-2)

/* ------------------------------------------------------------------ */
/* bf16: the upper 16 bits of an IEEE binary32, rounded to nearest even. */
/* ------------------------------------------------------------------ */

static uint16_t orc_f32_to_bf16_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    /* Round to nearest, ties to even, on the 16 discarded bits. */
    uint32_t discarded = u & 0xffffu;
    uint32_t kept = u >> 16;
    if (discarded > 0x8000u || (discarded == 0x8000u && (kept & 1u)))
        kept += 1u;
    return (uint16_t)kept;
}

static float orc_bf16_bits_to_f32(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round an fp32 value to the nearest bf16 value and return it as fp32. */
static float orc_round_bf16(float f)
{
    return orc_bf16_bits_to_f32(orc_f32_to_bf16_bits(f));
}

void orc_f32_to_bf16(const float* in, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_f32_to_bf16_bits(in[i]);
}

void orc_bf16_to_f32(const uint16_t* in, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_bf16_bits_to_f32(in[i]);
}

/* ------------------------------------------------------------------ */
/* fp16: IEEE binary16, rounded to nearest even from binary32.           */
/* ------------------------------------------------------------------ */

/* Nearest binary16 value (ties to even) of a finite float, returned as a
 * float; overflow past the largest binary16 gives +-inf, and values below the
 * smallest normal round on the subnormal grid (multiples of 2^-24). */
static float orc_round_f16(float f)
{
    if (f != f)
        return f;
    const double a = fabs((double)f);
    if (a >= 65520.0)  /* rounds past 65504 (the tie at 65520 goes to the even, infinite side) */
        return copysignf(INFINITY, f);
    int e;
    frexp(a, &e);             /* a = m 2^e, m in [0.5, 1) */
    int q = e - 11;           /* spacing 2^q for 11 significant bits */
    if (q < -24)
        q = -24;              /* subnormal spacing */
    const double step = ldexp(1.0, q);
    double r = a / step;      /* exact: a has at most 24 bits */
    double fl = floor(r);
    const double frac = r - fl;
    if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0))
        fl += 1.0;
    return (float)copysign(fl * step, (double)f);  /* keeps the sign of a zero result */
}

void orc_round_f16_array(const float* in, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_round_f16(in[i]);
}

/* ------------------------------------------------------------------ */
/* [QL] weight field: b-bit codes packed into uint32, shape [N, K*b/32].  */
/* ------------------------------------------------------------------ */

/* [QL] from_linear: 1 to 6 or 8 bits per weight. */
static int orc_bits_ok(int bits)
{
    return (bits >= 1 && bits <= 6) || bits == 8;
}

/*
 * q: one code per byte, [N, K], each < 2^bits.  out: [N, K*bits/32].  A row
 * is one LSB-first bitstream: code k occupies bits k*bits .. k*bits+bits-1 of
 * the row read as a little-endian integer of 32-bit words, so for 3, 5 and 6
 * bits a code may continue in the next word (a reading: the pages do not
 * show how such widths straddle words).
 */
int orc_pack(const uint8_t* q, int64_t N, int64_t K, int bits, uint32_t* out)
{
    if (!orc_bits_ok(bits) || N < 0 || K < 0 || (K * bits) % 32 != 0)
        return ORC_EINVAL;
    const int64_t words = K * bits / 32;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t w = 0; w < words; ++w)
            out[n * words + w] = 0u;
        for (int64_t k = 0; k < K; ++k) {
            uint32_t code = q[n * K + k];
            if (code >= (1u << bits))
                return ORC_EINVAL;
            int64_t bitpos = k * bits;
            out[n * words + bitpos / 32] |= code << (bitpos % 32);
            if (bitpos % 32 + bits > 32)  /* the high bits continue in the next word */
                out[n * words + bitpos / 32 + 1] |= code >> (32 - bitpos % 32);
        }
    }
    return 0;
}

/* Inverse of orc_pack. */
int orc_unpack(const uint32_t* packed, int64_t N, int64_t K, int bits, uint8_t* q)
{
    if (!orc_bits_ok(bits) || N < 0 || K < 0 || (K * bits) % 32 != 0)
        return ORC_EINVAL;
    const int64_t words = K * bits / 32;
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int64_t bitpos = k * bits;
            uint32_t v = packed[n * words + bitpos / 32] >> (bitpos % 32);
            if (bitpos % 32 + bits > 32)
                v |= packed[n * words + bitpos / 32 + 1] << (32 - bitpos % 32);
            q[n * K + k] = (uint8_t)(v & mask);
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* [QL] from_linear + [PG] quantize formula: affine group quantisation.  */
/* ------------------------------------------------------------------ */

static int orc_group_ok(int g)
{
    return g == 32 || g == 64 || g == 128;
}

/*
 * w: [N, K] values (fp32, or the fp32 value of a bf16 / fp16 input).
 * bf16_params: 0 -> scales/biases stored as fp32; 1 -> stored as bf16;
 * 2 -> stored as fp16.
 * codes: [N, K*bits/32]; scales, biases: [N, K/g], the STORED values written
 * as fp32 (a bf16-stored parameter is written as its exact fp32 value).
 *
 * Per group of g consecutive inputs of one output row:
 *   mn, mx   = min, max of the group
 *   scale    = (mx - mn) / (2^b - 1)       fp32 subtract, fp32 IEEE divide
 *   bias     = mn
 *   stored   = scale, bias rounded to the parameter dtype; a stored scale of
 *              0 (constant group) is replaced by 1.0
 *   q        = clip(round((w - bias_s) / scale_s), 0, 2^b - 1)
 *              fp32 subtract, fp32 IEEE divide, round half to even
 */
int orc_affine_quantize(const float* w, int64_t N, int64_t K, int bits, int g,
                        int bf16_params, uint32_t* codes, float* scales, float* biases)
{
    if (!orc_bits_ok(bits) || !orc_group_ok(g) || N <= 0 || K <= 0 || K % g != 0)
        return ORC_EINVAL;
    const int64_t G = K / g;
    const float qmax = (float)((1 << bits) - 1);
    uint8_t* q = (uint8_t*)malloc((size_t)(N * K));
    if (!q)
        return ORC_EINVAL;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t gi = 0; gi < G; ++gi) {
            const float* wg = w + n * K + gi * g;
            float mn = wg[0], mx = wg[0];
            for (int i = 1; i < g; ++i) {
                if (wg[i] < mn) mn = wg[i];
                if (wg[i] > mx) mx = wg[i];
            }
            float scale = (mx - mn) / qmax;
            float bias = mn;
            if (bf16_params == 1) {
                scale = orc_round_bf16(scale);
                bias = orc_round_bf16(bias);
            } else if (bf16_params == 2) {
                scale = orc_round_f16(scale);
                bias = orc_round_f16(bias);
            }
            if (scale == 0.0f)
                scale = 1.0f;
            scales[n * G + gi] = scale;
            biases[n * G + gi] = bias;
            for (int i = 0; i < g; ++i) {
                float t = (wg[i] - bias) / scale;
                float r = rintf(t);
                if (r < 0.0f) r = 0.0f;
                if (r > qmax) r = qmax;
                q[n * K + gi * g + i] = (uint8_t)r;
            }
        }
    }
    int rc = orc_pack(q, N, K, bits, codes);
    free(q);
    return rc;
}

/*
 * [QL] dequantized_weight, [PG] dequantize formula:  w = q*scale + bias,
 * evaluated as one fused multiply-add in fp32.  w_hat: [N, K] fp32.
 */
int orc_affine_dequantize(const uint32_t* codes, const float* scales, const float* biases,
                          int64_t N, int64_t K, int bits, int g, float* w_hat)
{
    if (!orc_bits_ok(bits) || !orc_group_ok(g) || N <= 0 || K <= 0 || K % g != 0)
        return ORC_EINVAL;
    const int64_t G = K / g;
    uint8_t* q = (uint8_t*)malloc((size_t)(N * K));
    if (!q)
        return ORC_EINVAL;
    int rc = orc_unpack(codes, N, K, bits, q);
    if (rc == 0) {
        for (int64_t n = 0; n < N; ++n)
            for (int64_t k = 0; k < K; ++k)
                w_hat[n * K + k] = fmaf((float)q[n * K + k], scales[n * G + k / g], biases[n * G + k / g]);
    }
    free(q);
    return rc;
}

/*
 * [QL] forward: y = x W^T + bias over the last axis of x, W the dequantized
 * weight.  x: [M, K] fp32 values; bias: [N] or NULL.  y, absdot: [M, N]
 * doubles, y unrounded; absdot[m,n] = sum_k |x[m,k] * w_hat[n,k]|, the scale
 * of the floating-point tolerance.
 */
int orc_affine_matmul(const float* x, int64_t M, int64_t K, const uint32_t* codes,
                      const float* scales, const float* biases, int64_t N, int bits, int g,
                      const float* bias, double* y, double* absdot)
{
    if (M <= 0 || N <= 0)
        return ORC_EINVAL;
    float* w_hat = (float*)malloc((size_t)(N * K) * sizeof(float));
    if (!w_hat)
        return ORC_EINVAL;
    int rc = orc_affine_dequantize(codes, scales, biases, N, K, bits, g, w_hat);
    if (rc == 0) {
#pragma omp parallel for collapse(2) schedule(static)
        for (int64_t m = 0; m < M; ++m)
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0, mag = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double p = (double)x[m * K + k] * (double)w_hat[n * K + k];
                    acc += p;
                    mag += fabs(p);
                }
                if (bias)
                    acc += (double)bias[n];
                y[m * N + n] = acc;
                absdot[m * N + n] = mag;
            }
    }
    free(w_hat);
    return rc;
}

/* ------------------------------------------------------------------ */
/* [BL] BitLinear ternary weights.                                        */
/* ------------------------------------------------------------------ */

/*
 * Inverse of the kernel's unpacking: codes [N, K] in {0,1,2,3}; P [N/4, K].
 * Code of output row n = r + j*(N/4) sits in bits 2j..2j+1 of byte P[r, k].
 */
int orc_pack_ternary(const uint8_t* codes, int64_t N, int64_t K, uint8_t* P)
{
    if (N <= 0 || K <= 0 || N % 4 != 0)
        return ORC_EINVAL;
    const int64_t R = N / 4;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) {
            unsigned byte = 0;
            for (int j = 0; j < 4; ++j) {
                unsigned c = codes[(r + j * R) * K + k];
                if (c > 3u)
                    return ORC_EINVAL;
                byte |= c << (2 * j);
            }
            P[r * K + k] = (uint8_t)byte;
        }
    return 0;
}

/*
 * [BL] kernel source:  out[m, r + j*N/4] = scale * sum_k x[m,k] * (((P[r,k] >> 2j) & 3) - 1)
 * with scale = invert ? 1/ws : ws (an fp32 reciprocal, as the kernel takes
 * it), then [BL] __call__ adds the layer bias.  The sum is kept in double.
 * x: [M, K]; P: [N/4, K]; bias: [N] or NULL; y, absdot: [M, N].
 */
int orc_bitlinear(const float* x, int64_t M, int64_t K, const uint8_t* P, int64_t N,
                  float ws, int invert, const float* bias, double* y, double* absdot)
{
    if (M <= 0 || K <= 0 || N <= 0 || N % 4 != 0)
        return ORC_EINVAL;
    const int64_t R = N / 4;
    const float scale = invert ? 1.0f / ws : ws;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            const int64_t r = n % R;
            const int j = (int)(n / R);
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                int v = (int)((P[r * K + k] >> (2 * j)) & 3u) - 1;
                double p = (double)x[m * K + k] * (double)v;
                acc += p;
                mag += fabs(p);
            }
            double out = acc * (double)scale;
            if (bias)
                out += (double)bias[n];
            y[m * N + n] = out;
            absdot[m * N + n] = mag * fabs((double)scale);
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* [Q8] per-row symmetric int8; the same rule quantises activations.      */
/* ------------------------------------------------------------------ */

/*
 * w: [R, C].  Per row: scale = max|w| / 127 (fp32); a zero scale becomes 1;
 * q = clip(round(w / scale), -128, 127) with an fp32 IEEE divide and round
 * half to even.  q: [R, C] int8; scale: [R] fp32.
 */
int orc_quantize_int8_rows(const float* w, int64_t R, int64_t C, int8_t* q, float* scale)
{
    if (R <= 0 || C <= 0)
        return ORC_EINVAL;
    for (int64_t r = 0; r < R; ++r) {
        float amax = 0.0f;
        for (int64_t c = 0; c < C; ++c) {
            float a = fabsf(w[r * C + c]);
            if (a > amax) amax = a;
        }
        float s = amax / 127.0f;
        if (s == 0.0f)
            s = 1.0f;
        scale[r] = s;
        for (int64_t c = 0; c < C; ++c) {
            float t = rintf(w[r * C + c] / s);
            if (t < -128.0f) t = -128.0f;
            if (t > 127.0f) t = 127.0f;
            q[r * C + c] = (int8_t)t;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* [Q8] with clip_percentile: a per-row percentile of |w| as the clip.   */
/* ------------------------------------------------------------------ */

static int orc_cmp_f32(const void* a, const void* b)
{
    const float x = *(const float*)a, y = *(const float*)b;
    return (x > y) - (x < y);
}

/*
 * The p-th percentile of v[0..n) (0 <= p <= 100) by linear interpolation
 * between the order statistics around (n - 1) p / 100 -- numpy's default
 * ("linear", Hyndman and Fan's type 7), which [Q8] calls through
 * np.percentile -- with numpy's float32 arithmetic for a float32 row:
 * q = f32(p) / 100, h = (n - 1) q, j = floor(h), t = h - j, a = v_(j),
 * b = v_(j+1), and  a + (b - a) t  when t < 1/2, else  b - (b - a)(1 - t);
 * h >= n - 1 gives the largest value.  Each step rounded to float32.
 */
float orc_percentile_linear(const float* v, int64_t n, double p)
{
    float* s = (float*)malloc((size_t)n * sizeof(float));
    if (!s)
        return NAN;
    memcpy(s, v, (size_t)n * sizeof(float));
    qsort(s, (size_t)n, sizeof(float), orc_cmp_f32);
    const float q = (float)p / 100.0f;
    const float h = (float)(n - 1) * q;
    float r;
    if (h >= (float)(n - 1)) {
        r = s[n - 1];
    } else {
        const float j = floorf(h);
        const float t = h - j;
        const float a = s[(int64_t)j], b = s[(int64_t)j + 1];
        const float d = b - a;
        r = t < 0.5f ? a + d * t : b - d * (1.0f - t);
    }
    free(s);
    return r;
}

/*
 * [Q8] quantize_weight_int8 with clip_percentile set: per row, row_clip =
 * percentile(|w_row|, clip_percentile) (above), replaced by max |w_row| when
 * it is 0; scale = row_clip / 127 (fp32), zero -> 1; w clipped to
 * [-row_clip, row_clip]; q = clip(round(w / scale), -128, 127).
 * w: [R, C]; q: [R, C] int8; scale: [R] fp32.
 */
int orc_quantize_weight_int8_clip(const float* w, int64_t R, int64_t C, double clip_percentile, int8_t* q,
                                  float* scale)
{
    if (R <= 0 || C <= 0 || !(clip_percentile >= 0.0 && clip_percentile <= 100.0))
        return ORC_EINVAL;
    float* a = (float*)malloc((size_t)C * sizeof(float));
    if (!a)
        return ORC_EINVAL;
    for (int64_t r = 0; r < R; ++r) {
        float amax = 0.0f;
        for (int64_t c = 0; c < C; ++c) {
            a[c] = fabsf(w[r * C + c]);
            if (a[c] > amax) amax = a[c];
        }
        float row_clip = orc_percentile_linear(a, C, clip_percentile);
        if (row_clip == 0.0f)
            row_clip = amax;
        float s = row_clip / 127.0f;
        if (s == 0.0f)
            s = 1.0f;
        scale[r] = s;
        for (int64_t c = 0; c < C; ++c) {
            float v = w[r * C + c];
            if (v < -row_clip) v = -row_clip;
            if (v > row_clip) v = row_clip;
            float t = rintf(v / s);
            if (t < -128.0f) t = -128.0f;
            if (t > 127.0f) t = 127.0f;
            q[r * C + c] = (int8_t)t;
        }
    }
    free(a);
    return 0;
}

/* ------------------------------------------------------------------ */
/* [P4] per-column int4, zero point 8, two codes per byte.               */
/* ------------------------------------------------------------------ */

/*
 * w: [K, N] (K even).  Per column n: scale = max_k |w[k,n]| / 7 (fp32), zero
 * -> 1; c = clip(round(w / scale) + 8, 0, 15).  P[i, n] holds c[2i, n] in the
 * high nibble and c[2i+1, n] in the low nibble.  P: [K/2, N]; scale: [N].
 */
int orc_pack_int4_cols(const float* w, int64_t K, int64_t N, uint8_t* P, float* scale)
{
    if (K <= 0 || N <= 0 || K % 2 != 0)
        return ORC_EINVAL;
    for (int64_t n = 0; n < N; ++n) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(w[k * N + n]);
            if (a > amax) amax = a;
        }
        float s = amax / 7.0f;
        if (s == 0.0f)
            s = 1.0f;
        scale[n] = s;
    }
    for (int64_t i = 0; i < K / 2; ++i)
        for (int64_t n = 0; n < N; ++n) {
            unsigned c[2];
            for (int h = 0; h < 2; ++h) {
                float t = rintf(w[(2 * i + h) * N + n] / scale[n]) + 8.0f;
                if (t < 0.0f) t = 0.0f;
                if (t > 15.0f) t = 15.0f;
                c[h] = (unsigned)t;
            }
            P[i * N + n] = (uint8_t)((c[0] << 4) | c[1]);
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* [I8] raw int8 x int8 -> int32, exact.                                 */
/* ------------------------------------------------------------------ */

/* a: [M, K], b: [N, K]; c = a b^T: [M, N].  int64 sums, checked to fit int32. */
int orc_int8_matmul(const int8_t* a, const int8_t* b, int64_t M, int64_t N, int64_t K, int32_t* c)
{
    if (M <= 0 || N <= 0 || K <= 0)
        return ORC_EINVAL;
    int overflow = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(| : overflow)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k)
                acc += (int64_t)a[m * K + k] * (int64_t)b[n * K + k];
            if (acc > INT32_MAX || acc < INT32_MIN)
                overflow = 1;
            c[m * N + n] = (int32_t)acc;
        }
    return overflow ? ORC_EOVERFLOW : 0;
}

/* ------------------------------------------------------------------ */
/* [PC] W8A8 and [W4] W4A8 linear layers.                                 */
/* ------------------------------------------------------------------ */

/*
 * [PC]: y = dequant(quant_a(x) @ w_int8^T) + bias.  quant_a is the per-row
 * int8 rule above applied to each token of x.  The int32 accumulator is
 * exact; dequant multiplies it by s_x[m] * s_w[n] (done in double here).
 * x: [M, K]; w: [N, K] int8; scale_w: [N]; bias: [N] or NULL.
 * qx, s_x (outputs, for inspection): [M, K] int8, [M] fp32.
 * y, absdot: [M, N], absdot = s_x s_w sum_k |qx qw|.
 */
int orc_w8a8_linear(const float* x, int64_t M, int64_t K, const int8_t* w, const float* scale_w,
                    int64_t N, const float* bias, int8_t* qx, float* s_x, double* y, double* absdot)
{
    int rc = orc_quantize_int8_rows(x, M, K, qx, s_x);
    if (rc != 0)
        return rc;
    if (N <= 0)
        return ORC_EINVAL;
    int overflow = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(| : overflow)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0, mag = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t p = (int64_t)qx[m * K + k] * (int64_t)w[n * K + k];
                acc += p;
                mag += p < 0 ? -p : p;
            }
            if (acc > INT32_MAX || acc < INT32_MIN)
                overflow = 1;
            double sc = (double)s_x[m] * (double)scale_w[n];
            double out = (double)acc * sc;
            if (bias)
                out += (double)bias[n];
            y[m * N + n] = out;
            absdot[m * N + n] = (double)mag * sc;
        }
    return overflow ? ORC_EOVERFLOW : 0;
}

/*
 * [W4]: y = dequant(quant_a(x) @ unpack4(w)).  unpack4 reads code
 * c[k, n] from P[k/2, n] (high nibble for even k, low nibble for odd k) and
 * the signed weight is c - 8 (zero point 8, [P4]).  scale_w: [N]; P: [K/2, N].
 */
int orc_w4a8_linear(const float* x, int64_t M, int64_t K, const uint8_t* P, const float* scale_w,
                    int64_t N, const float* bias, int8_t* qx, float* s_x, double* y, double* absdot)
{
    if (K % 2 != 0)
        return ORC_EINVAL;
    int rc = orc_quantize_int8_rows(x, M, K, qx, s_x);
    if (rc != 0)
        return rc;
    if (N <= 0)
        return ORC_EINVAL;
    int overflow = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(| : overflow)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0, mag = 0;
            for (int64_t k = 0; k < K; ++k) {
                uint8_t byte = P[(k / 2) * N + n];
                int c = (k % 2 == 0) ? (byte >> 4) : (byte & 15);
                int64_t p = (int64_t)qx[m * K + k] * (int64_t)(c - 8);
                acc += p;
                mag += p < 0 ? -p : p;
            }
            if (acc > INT32_MAX || acc < INT32_MIN)
                overflow = 1;
            double sc = (double)s_x[m] * (double)scale_w[n];
            double out = (double)acc * sc;
            if (bias)
                out += (double)bias[n];
            y[m * N + n] = out;
            absdot[m * N + n] = (double)mag * sc;
        }
    return overflow ? ORC_EOVERFLOW : 0;
}

/* ------------------------------------------------------------------ */
/* [PG] per-group symmetric INT8 linear (pergroup_linear).              */
/* ------------------------------------------------------------------ */

static int orc_pg_group_ok(int g) { return g == 64 || g == 128 || g == 256; }

/*
 * The weight quantiser of the per-group format (the page prints none; its
 * Args say "per-group symmetric quantized"): the rule of [Q8] applied to each
 * group of g consecutive inputs of a row -- scale = max |w| / 127 (fp32), zero
 * -> 1, q = clip(round(w / scale), -128, 127).  w: [N, K]; q: [N, K] int8;
 * scale_w: [K/g, N], stored transposed as the page's Args give it (group grp,
 * output n at scale_w[grp * N + n]).
 */
int orc_quantize_int8_groups(const float* w, int64_t N, int64_t K, int g, int8_t* q, float* scale_w)
{
    if (N <= 0 || K <= 0 || !orc_pg_group_ok(g) || K % g != 0)
        return ORC_EINVAL;
    const int64_t G = K / g;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t grp = 0; grp < G; ++grp) {
            const float* wg = w + n * K + grp * g;
            float amax = 0.0f;
            for (int k = 0; k < g; ++k) {
                float a = fabsf(wg[k]);
                if (a > amax) amax = a;
            }
            float s = amax / 127.0f;
            if (s == 0.0f)
                s = 1.0f;
            scale_w[grp * N + n] = s;
            for (int k = 0; k < g; ++k) {
                float t = rintf(wg[k] / s);
                if (t < -128.0f) t = -128.0f;
                if (t > 127.0f) t = 127.0f;
                q[n * K + grp * g + k] = (int8_t)t;
            }
        }
    return 0;
}

/*
 * [PG] y = pergroup_linear(x, w, scale_w, g, bias), with the page's dispatch:
 *   M == 1: FP activation, weights dequantised per group:
 *       y[n] = sum_grp scale_w[grp, n] * sum_{k in grp} x[k] * w[n, k] + bias[n]
 *   M > 1:  quant_a(x) (the per-token int8 rule of [PC]), exact integer sums
 *       per group, then y[m, n] = s_x[m] * sum_grp scale_w[grp, n] * acc_grp + bias[n]
 *       with acc_grp = sum_{k in grp} qx[m, k] * w[n, k].
 * Double accumulation.  x: [M, K]; w: [N, K] int8; scale_w: [K/g, N]; bias: [N]
 * or NULL.  qx, s_x (outputs, M > 1 only): [M, K], [M].  y, absdot: [M, N],
 * absdot = the same sums over |products|.
 */
int orc_pergroup_linear(const float* x, int64_t M, int64_t K, const int8_t* w, const float* scale_w,
                        int64_t N, int g, const float* bias, int8_t* qx, float* s_x, double* y, double* absdot)
{
    if (M <= 0 || N <= 0 || K <= 0 || !orc_pg_group_ok(g) || K % g != 0)
        return ORC_EINVAL;
    const int64_t G = K / g;
    const int fp_act = M == 1;  /* the page's dispatch: FP activation only for a single token */
    if (!fp_act) {
        int rc = orc_quantize_int8_rows(x, M, K, qx, s_x);
        if (rc != 0)
            return rc;
    }
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double out = 0.0, mag = 0.0;
            for (int64_t grp = 0; grp < G; ++grp) {
                const double sw = (double)scale_w[grp * N + n];
                if (fp_act) {
                    double acc = 0.0, am = 0.0;
                    for (int k = 0; k < g; ++k) {
                        const double p = (double)x[grp * g + k] * (double)w[n * K + grp * g + k];
                        acc += p;
                        am += fabs(p);
                    }
                    out += sw * acc;
                    mag += sw * am;
                } else {
                    int64_t acc = 0, am = 0;
                    for (int k = 0; k < g; ++k) {
                        const int64_t p = (int64_t)qx[m * K + grp * g + k] * (int64_t)w[n * K + grp * g + k];
                        acc += p;
                        am += p < 0 ? -p : p;
                    }
                    out += sw * (double)acc;
                    mag += sw * (double)am;
                }
            }
            if (!fp_act) {
                out *= (double)s_x[m];
                mag *= (double)s_x[m];
            }
            if (bias)
                out += (double)bias[n];
            y[m * N + n] = out;
            absdot[m * N + n] = mag;
        }
    return 0;
}
