/*
 * convrot_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * ConvRot-quantized linear layer (W8A8 / W4A4).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: it exists so that tests/, the smoke check and the CPU
 * baseline leg of bench.py can compare the CUDA library against an
 * independent statement of the method.  It shares no code, header, table or
 * constant with the CUDA sources.
 *
 * What the method computes (source pages):
 *   - civarchive.com, "SAM 3.1 Multiplex ConvRot" release, section
 *     "Quantization recipe": for each eligible linear weight the converter
 *     (1) upcasts the source weight to FP32, (2) applies a block-Hadamard
 *     ConvRot transform, (3) chooses an MSE-optimized clipping scale,
 *     (4) stores per-row quantization scales.  The runtime uses W8A8 (or
 *     W4A4) operations with online, dynamic activation quantization.
 *   - trellis3d.app, "TRELLIS.2 INT8 ConvRot in ComfyUI", section
 *     "What ConvRot changes": a grouped, normalized Hadamard rotation is
 *     applied before per-row weight quantization and the matching rotation
 *     is applied to the activations at runtime, to spread channel outliers.
 *   - salahadawi.com, "Explanation of INT8 ConvRot", tables "8-bit INT type
 *     models": INT8 encoding, Row-wise scaling, ConvRot quantization method.
 *
 * Readings taken where the pages are silent (none of these pages fixes the
 * block order, the signs, the clip grid or the rounding of the steps below):
 *   R      = blockdiag(R_b, ..., R_b),  R_b = H_b / sqrt(b), H_b the Sylvester
 *            Hadamard matrix in natural order, no random signs, disjoint blocks.
 *   X~     = fp32( X . R ) evaluated as a dense fp64 product per block.
 *   s      = fp32( fp32(alpha * amax) / qmax ),  alpha = 1 for absmax mode,
 *            alpha in {100/100, 99/100, ..., 50/100} for the MSE clip search
 *            (first strict minimum of the fp64 squared error, largest alpha
 *            first, so a tie keeps the larger alpha).
 *   q      = clamp( rne( x * fp32(1/s) ), qmin, qmax ), the product taken
 *            exactly (one rounding, to the integer grid; ties to even),
 *            int8: [-127, 127], int4: [-8, 7].  s == 0 gives q == 0.
 *   int4   : two codes per byte, element 2j in bits 0..3, 2j+1 in bits 4..7.
 *   acc    = sum_k qx[m,k] * qw[n,k]   (exact integer, must fit int32)
 *   y      = fp16_rne( fma_fp32( fp32(float(acc) * s_x[m]), s_w[n], bias[n] ) ),
 *            the last multiply-add rounded once (bias 0 when absent)
 *
 * Compile with -ffp-contract=off so that no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_OVERFLOW 2

#define ORACLE_DTYPE_F16 0
#define ORACLE_DTYPE_BF16 1
#define ORACLE_DTYPE_F32 2

#define ORACLE_CLIP_ABSMAX 0
#define ORACLE_CLIP_MSE 1
#define ORACLE_MSE_GRID 51

/* ------------------------------------------------------------------ */
/* Number formats (IEEE 754 binary16 / bfloat16 / binary32 definitions) */
/* ------------------------------------------------------------------ */

/* binary16 -> double, exactly: sign, 5-bit biased exponent, 10-bit fraction. */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
    } else if (e == 31) {
        v = m ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16 -> double, exactly: the upper half of a binary32. */
double oracle_bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* binary32 -> binary16, round to nearest, ties to even; overflow -> inf. */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
    double a = fabs((double)f);
    /* The largest finite binary16 is 65504; halfway to the next power
     * 65536 is 65520, and that tie rounds to the even neighbour (inf). */
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: value = q * 2^-24, q in [0, 1024] */
        double q = nearbyint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)q); /* q == 1024 is the smallest normal */
    }
    int ex;
    frexp(a, &ex);   /* a = fr * 2^ex, fr in [0.5, 1) */
    int E = ex - 1;  /* a in [2^E, 2^(E+1)) */
    double q = nearbyint(ldexp(a, 10 - E)); /* in [1024, 2048] */
    if (q >= 2048.0) {
        q = 1024.0;
        E += 1;
    }
    if (E + 15 >= 31) return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)((int)q - 1024));
}

/* Decode n source values of the given dtype to double (the "upcast"). */
int oracle_decode(const void *src, int dtype, int64_t n, double *out)
{
    if (!src || !out || n < 0) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        if (dtype == ORACLE_DTYPE_F16)
            out[i] = oracle_f16_to_f64(((const uint16_t *)src)[i]);
        else if (dtype == ORACLE_DTYPE_BF16)
            out[i] = oracle_bf16_to_f64(((const uint16_t *)src)[i]);
        else if (dtype == ORACLE_DTYPE_F32)
            out[i] = (double)((const float *)src)[i];
        else
            return ORACLE_ERR_ARG;
    }
    return ORACLE_OK;
}

void oracle_f32_to_f16_array(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_f16(in[i]);
}

/* ------------------------------------------------------------------ */
/* The rotation                                                         */
/* ------------------------------------------------------------------ */

static int is_pow2(int b) { return b >= 1 && (b & (b - 1)) == 0; }

/* R_b = H_b / sqrt(b), with H_1 = [1] and H_2n = [[H_n, H_n], [H_n, -H_n]]
 * (Sylvester).  R is written row-major, b x b, as float64. */
int oracle_hadamard(int b, double *R)
{
    if (!is_pow2(b) || !R) return ORACLE_ERR_ARG;
    R[0] = 1.0;
    for (int n = 1; n < b; n *= 2) {
        for (int i = 0; i < n; ++i) {
            for (int j = 0; j < n; ++j) {
                double h = R[(int64_t)i * b + j];
                R[(int64_t)i * b + (j + n)] = h;
                R[(int64_t)(i + n) * b + j] = h;
                R[(int64_t)(i + n) * b + (j + n)] = -h;
            }
        }
    }
    double c = 1.0 / sqrt((double)b);
    for (int64_t i = 0; i < (int64_t)b * b; ++i) R[i] *= c;
    return ORACLE_OK;
}

/* One row x (K values, float64) times blockdiag(R_b): for every block t,
 * out[t*b + k] = sum_j x[t*b + j] * R_b[j][k], accumulated in float64. */
static void rotate_row(const double *x, int64_t K, int b, const double *Rb, double *out)
{
    for (int64_t t = 0; t < K / b; ++t) {
        const double *xb = x + t * b;
        for (int k = 0; k < b; ++k) {
            double acc = 0.0;
            for (int j = 0; j < b; ++j) acc += xb[j] * Rb[(int64_t)j * b + k];
            out[t * b + k] = acc;
        }
    }
}

/* X (rows x K, float64) -> X.R in float64 (out64, nullable) and rounded to
 * fp32 (out32, nullable).  Requires K % b == 0. */
int oracle_rotate(const double *X, int64_t rows, int64_t K, int b, double *out64, float *out32)
{
    if (!X || rows < 0 || K <= 0 || !is_pow2(b) || K % b) return ORACLE_ERR_ARG;
    double *Rb = (double *)malloc(sizeof(double) * (size_t)b * b);
    if (!Rb) return ORACLE_ERR_ARG;
    oracle_hadamard(b, Rb);
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        double *tmp = (double *)malloc(sizeof(double) * (size_t)K);
        rotate_row(X + r * K, K, b, Rb, tmp);
        for (int64_t k = 0; k < K; ++k) {
            if (out64) out64[r * K + k] = tmp[k];
            if (out32) out32[r * K + k] = (float)tmp[k];
        }
        free(tmp);
    }
    free(Rb);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Symmetric round-to-nearest quantization                              */
/* ------------------------------------------------------------------ */

int oracle_qmax(int bits) { return bits == 8 ? 127 : 7; }
int oracle_qmin(int bits) { return bits == 8 ? -127 : -8; }

/* s = fp32( fp32(alpha * amax) / qmax ) */
float oracle_scale(float amax, float alpha, int bits)
{
    float clipped = alpha * amax;
    return clipped / (float)oracle_qmax(bits);
}

/* fp32(1/s); a zero scale maps every value to code 0. */
float oracle_inv_scale(float s) { return s == 0.0f ? 0.0f : 1.0f / s; }

/* q = clamp(rne(x * inv), qmin, qmax) with the product exact: two 24-bit
 * significands multiply exactly in float64, and nearbyint rounds that exact
 * value to the nearest integer, ties to even. */
int oracle_quantize_value(float x, float inv, int bits)
{
    double t = (double)x * (double)inv;
    double r = nearbyint(t); /* default rounding mode: nearest, ties to even */
    double lo = (double)oracle_qmin(bits), hi = (double)oracle_qmax(bits);
    if (r < lo) r = lo;
    if (r > hi) r = hi;
    return (int)r;
}

/* Squared reconstruction error of one row under scale s, in float64:
 * sum_k (x_k - s * q_k)^2. */
double oracle_quant_error(const float *x, int64_t K, float s, int bits)
{
    float inv = oracle_inv_scale(s);
    double err = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        int q = oracle_quantize_value(x[k], inv, bits);
        double d = (double)x[k] - (double)s * (double)q;
        err += d * d;
    }
    return err;
}

/* The clip factor of grid point i: alpha_i = fp32((100 - i) / 100). */
float oracle_alpha(int i) { return (float)(100 - i) / 100.0f; }

static float row_absmax(const float *x, int64_t K)
{
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float v = fabsf(x[k]);
        if (v > a) a = v;
    }
    return a;
}

/* Offline weight path (steps 1-4 of the converter):
 * W (N x K, dtype) -> upcast -> X.R rounded to fp32 -> per-row clip search ->
 * per-row scale s_w[n] and codes (one int8 per element, unpacked).
 * alpha_idx (nullable) receives the chosen grid index per row; errs
 * (nullable, N x 51) receives the squared error of every grid point. */
int oracle_quantize_weight(const void *W, int dtype, int64_t N, int64_t K, int b, int bits,
                           int clip_mode, int8_t *codes, float *scales, int32_t *alpha_idx,
                           double *errs)
{
    if (!W || !codes || !scales || N < 0 || K <= 0 || !is_pow2(b) || K % b) return ORACLE_ERR_ARG;
    if (bits != 8 && bits != 4) return ORACLE_ERR_ARG;
    if (clip_mode != ORACLE_CLIP_ABSMAX && clip_mode != ORACLE_CLIP_MSE) return ORACLE_ERR_ARG;
    double *Rb = (double *)malloc(sizeof(double) * (size_t)b * b);
    oracle_hadamard(b, Rb);
    int n_alpha = clip_mode == ORACLE_CLIP_MSE ? ORACLE_MSE_GRID : 1;
    int64_t n;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
    for (n = 0; n < N; ++n) {
        double *src = (double *)malloc(sizeof(double) * (size_t)K);
        double *rot = (double *)malloc(sizeof(double) * (size_t)K);
        float *w = (float *)malloc(sizeof(float) * (size_t)K);
        if (dtype == ORACLE_DTYPE_F32)
            bad |= oracle_decode((const float *)W + n * K, dtype, K, src);
        else
            bad |= oracle_decode((const uint16_t *)W + n * K, dtype, K, src);
        rotate_row(src, K, b, Rb, rot);
        for (int64_t k = 0; k < K; ++k) w[k] = (float)rot[k];
        float a = row_absmax(w, K);
        int best = 0;
        double best_err = INFINITY;
        for (int i = 0; i < n_alpha; ++i) {
            float s = oracle_scale(a, oracle_alpha(i), bits);
            double e = oracle_quant_error(w, K, s, bits);
            if (errs) errs[n * ORACLE_MSE_GRID + i] = e;
            if (e < best_err) {
                best_err = e;
                best = i;
            }
        }
        float s = oracle_scale(a, oracle_alpha(best), bits);
        float inv = oracle_inv_scale(s);
        for (int64_t k = 0; k < K; ++k) codes[n * K + k] = (int8_t)oracle_quantize_value(w[k], inv, bits);
        scales[n] = s;
        if (alpha_idx) alpha_idx[n] = best;
        free(src);
        free(rot);
        free(w);
    }
    free(Rb);
    return bad ? ORACLE_ERR_ARG : ORACLE_OK;
}

/* Tensor-wise variant of the converter (salahadawi.com "Explanation of INT8
 * ConvRot", "8-bit INT type models" table: Tensor-wise scaling, one scale per
 * weight tensor; civarchive.com release, downloads table: an int8_tensorwise
 * ConvRot file).  Same rotation and code rule as oracle_quantize_weight, but
 * one scale for all rows: s = fp32(fp32(alpha * max over the tensor of |W~|) /
 * qmax), with alpha from the same grid.  In MSE mode alpha minimises the
 * total squared error of the tensor, the rows' float64 errors summed in row
 * order (first strict minimum from alpha = 1).  `scales` receives s for every
 * row, `errs` (if given) the tensor's error for each grid point. */
int oracle_quantize_weight_tensorwise(const void *W, int dtype, int64_t N, int64_t K, int b, int bits,
                                      int clip_mode, int8_t *codes, float *scales, int32_t *alpha_idx,
                                      double *errs)
{
    if (!W || !codes || !scales || N < 0 || K <= 0 || !is_pow2(b) || K % b) return ORACLE_ERR_ARG;
    if (bits != 8 && bits != 4) return ORACLE_ERR_ARG;
    if (clip_mode != ORACLE_CLIP_ABSMAX && clip_mode != ORACLE_CLIP_MSE) return ORACLE_ERR_ARG;
    double *Rb = (double *)malloc(sizeof(double) * (size_t)b * b);
    float *w = (float *)malloc(sizeof(float) * (size_t)(N > 0 ? N : 1) * (size_t)K);
    float *row_max = (float *)malloc(sizeof(float) * (size_t)(N > 0 ? N : 1));
    oracle_hadamard(b, Rb);
    int64_t n;
    int bad = 0;
    /* step 1: every row rotated and rounded to fp32, and its absmax */
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
    for (n = 0; n < N; ++n) {
        double *src = (double *)malloc(sizeof(double) * (size_t)K);
        double *rot = (double *)malloc(sizeof(double) * (size_t)K);
        if (dtype == ORACLE_DTYPE_F32)
            bad |= oracle_decode((const float *)W + n * K, dtype, K, src);
        else
            bad |= oracle_decode((const uint16_t *)W + n * K, dtype, K, src);
        rotate_row(src, K, b, Rb, rot);
        for (int64_t k = 0; k < K; ++k) w[n * K + k] = (float)rot[k];
        row_max[n] = row_absmax(w + n * K, K);
        free(src);
        free(rot);
    }
    /* step 2: the tensor's absmax */
    float a = 0.0f;
    for (n = 0; n < N; ++n) a = row_max[n] > a ? row_max[n] : a;
    /* step 3: the clip choice */
    int n_alpha = clip_mode == ORACLE_CLIP_MSE ? ORACLE_MSE_GRID : 1;
    double *row_err = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1) * ORACLE_MSE_GRID);
#pragma omp parallel for schedule(dynamic, 4)
    for (n = 0; n < N; ++n)
        for (int i = 0; i < n_alpha; ++i)
            row_err[n * ORACLE_MSE_GRID + i] = oracle_quant_error(w + n * K, K, oracle_scale(a, oracle_alpha(i), bits), bits);
    int best = 0;
    double best_err = INFINITY;
    for (int i = 0; i < n_alpha; ++i) {
        double e = 0.0;
        for (n = 0; n < N; ++n) e += row_err[n * ORACLE_MSE_GRID + i];
        if (errs) errs[i] = e;
        if (e < best_err) {
            best_err = e;
            best = i;
        }
    }
    /* step 4: every row quantized with the one scale */
    float s = oracle_scale(a, oracle_alpha(best), bits);
    float inv = oracle_inv_scale(s);
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) codes[n * K + k] = (int8_t)oracle_quantize_value(w[n * K + k], inv, bits);
        scales[n] = s;
    }
    if (alpha_idx) *alpha_idx = best;
    free(row_err);
    free(row_max);
    free(w);
    free(Rb);
    return bad ? ORACLE_ERR_ARG : ORACLE_OK;
}

/* Online activation path: X (M x K fp16) -> X.R rounded to fp32 -> per-token
 * absmax scale s_x[m] = fp32(amax / qmax) -> codes (unpacked int8). */
int oracle_rotate_quant_act(const uint16_t *X, int64_t M, int64_t K, int b, int bits, int8_t *codes,
                            float *scales)
{
    if (!X || !codes || !scales || M < 0 || K <= 0 || !is_pow2(b) || K % b) return ORACLE_ERR_ARG;
    if (bits != 8 && bits != 4) return ORACLE_ERR_ARG;
    double *Rb = (double *)malloc(sizeof(double) * (size_t)b * b);
    oracle_hadamard(b, Rb);
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        double *src = (double *)malloc(sizeof(double) * (size_t)K);
        double *rot = (double *)malloc(sizeof(double) * (size_t)K);
        float *x = (float *)malloc(sizeof(float) * (size_t)K);
        for (int64_t k = 0; k < K; ++k) src[k] = oracle_f16_to_f64(X[m * K + k]);
        rotate_row(src, K, b, Rb, rot);
        for (int64_t k = 0; k < K; ++k) x[k] = (float)rot[k];
        float s = oracle_scale(row_absmax(x, K), 1.0f, bits);
        float inv = oracle_inv_scale(s);
        for (int64_t k = 0; k < K; ++k) codes[m * K + k] = (int8_t)oracle_quantize_value(x[k], inv, bits);
        scales[m] = s;
        free(src);
        free(rot);
        free(x);
    }
    free(Rb);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Int4 storage                                                         */
/* ------------------------------------------------------------------ */

/* Two codes per byte: element 2j in the low nibble, 2j+1 in the high
 * nibble, each in 4-bit two's complement. */
int oracle_pack_int4(const int8_t *codes, int64_t count, uint8_t *packed)
{
    if (!codes || !packed || count < 0 || (count & 1)) return ORACLE_ERR_ARG;
    for (int64_t j = 0; j < count / 2; ++j) {
        int lo = codes[2 * j], hi = codes[2 * j + 1];
        if (lo < -8 || lo > 7 || hi < -8 || hi > 7) return ORACLE_ERR_ARG;
        packed[j] = (uint8_t)((lo & 0xf) | ((hi & 0xf) << 4));
    }
    return ORACLE_OK;
}

int oracle_unpack_int4(const uint8_t *packed, int64_t count, int8_t *codes)
{
    if (!codes || !packed || count < 0 || (count & 1)) return ORACLE_ERR_ARG;
    for (int64_t j = 0; j < count / 2; ++j) {
        int lo = packed[j] & 0xf, hi = (packed[j] >> 4) & 0xf;
        codes[2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
        codes[2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
    }
    return ORACLE_OK;
}

/* Stored bytes of one quantized N x K weight: the codes plus one fp32 scale
 * per output row. */
int64_t oracle_weight_bytes(int64_t N, int64_t K, int bits) { return N * K * bits / 8 + 4 * N; }

/* ------------------------------------------------------------------ */
/* Integer GEMM and dequantizing epilogue                               */
/* ------------------------------------------------------------------ */

/* acc[m,n] = sum_k qx[m,k] * qw[n,k]; y[m,n] as in the header comment.
 * acc_out (nullable) receives the int32 accumulators.  bias is nullable
 * (fp16 bit patterns).  Fails if an accumulator leaves the int32 range. */
int oracle_gemm_dequant(const int8_t *qx, const float *sx, int64_t M, const int8_t *qw, const float *sw,
                        int64_t N, int64_t K, const uint16_t *bias, int32_t *acc_out, uint16_t *y)
{
    if (!qx || !sx || !qw || !sw || !y || M < 0 || N < 0 || K <= 0) return ORACLE_ERR_ARG;
    int64_t m;
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k) acc += (int64_t)qx[m * K + k] * (int64_t)qw[n * K + k];
            if (acc > INT32_MAX || acc < INT32_MIN) {
                overflow = 1;
                acc = 0;
            }
            if (acc_out) acc_out[m * N + n] = (int32_t)acc;
            float f = (float)(int32_t)acc;
            float t = f * sx[m];
            float b = bias ? (float)oracle_f16_to_f64(bias[n]) : 0.0f;
            y[m * N + n] = oracle_f32_to_f16(fmaf(t, sw[n], b)); /* C99 fmaf: one rounding */
        }
    }
    return overflow ? ORACLE_ERR_OVERFLOW : ORACLE_OK;
}

/* fp32 value of one output before its fp16 conversion (for pinning the
 * single-rounding multiply-add). */
float oracle_epilogue_value(int32_t acc, float sx, float sw, float bias)
{
    float t = (float)acc * sx;
    return fmaf(t, sw, bias);
}

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
