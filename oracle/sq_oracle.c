/*
 * CPU oracle for the dual-path sparse-quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this file.  It shares no code, header,
 * table or helper with the CUDA library and must never be linked into it.
 *
 * What it computes (a plain, slow, literal statement of the layer):
 *
 *   Y[m,n] = s_x[m] * s_w[n] * sum_{k not in O} q(X)[m,k] * q(W)[n,k]
 *          +                   sum_{k in O}     X[m,k]   * W[n,k]
 *
 * Sources:
 *   - OSC: Hardware Efficient W4A4 Quantization via Outlier Separation in
 *     Channel Dimension (arXiv:2604.12782), abstract and "technical framework"
 *     paragraph: a static set O of outlier input channels is chosen offline;
 *     at inference the scattered outlier channels are coalesced into a compact
 *     dense tensor and run through a 16-bit branch GEMM while every other
 *     channel runs through a 4-bit GEMM; the two results are fused (summed).
 *   - SQ-format write-up of arXiv:2512.05409, section 9 (technical details):
 *     the low-precision part uses symmetric quantization, which leaves the
 *     most negative two's-complement code unused (INT2 keeps {-1,0,1}); for
 *     INT4 that is the range [-7, 7].  Section 9 also reorders weight columns
 *     by the static mask; here the compact normal part keeps the channels in
 *     ascending order and the compact outlier part keeps O in ascending order.
 *   - Scale granularity (not fixed by the pages; the layer's formula above):
 *     one scale per token row of X (computed online) and one per output
 *     channel (row) of W (computed offline), each the absolute maximum over
 *     the NON-outlier channels divided by 7.
 *
 * Readings taken where the pages are silent:
 *   - s = a / 7 with a = max |x| over k not in O, both fp32 (bf16 widens to
 *     fp32 exactly) with IEEE round-to-nearest division.
 *   - code = clamp(rint(x / s), -7, 7) where x / s is the IEEE fp32 quotient
 *     and rint rounds half to even (FE_TONEAREST).  The integer decision is
 *     made in fp32, the same precision as the CUDA kernels.
 *   - a == 0 (all normal channels zero, or no normal channels): s = 0 and
 *     every code is 0.
 *   - Integer products are summed exactly in int64; the 16-bit branch and the
 *     final Y are computed in fp64 without any final rounding.
 *
 * The `omp parallel for` pragmas only distribute independent output rows over
 * host threads; they do not change any arithmetic or its order.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_QMAX 7

static float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* O must be strictly increasing inside [0, K).  Returns 0 when valid. */
int orc_validate_outliers(const int32_t *O, int64_t nO, int64_t K)
{
    if (K <= 0 || nO < 0 || nO > K) return -1;
    for (int64_t j = 0; j < nO; ++j) {
        if (O[j] < 0 || O[j] >= K) return -1;
        if (j > 0 && O[j] <= O[j - 1]) return -1;
    }
    return 0;
}

/*
 * Quantize-and-gather of `rows` rows of a bf16 matrix (row stride `ld`
 * elements).  Used for activations (rows = tokens, online) and for weights
 * (rows = output channels, offline): the pages apply the same symmetric
 * quantizer to both operands of the 4-bit path.
 *
 * Outputs (caller-allocated, dense):
 *   codes [rows, K - nO]  int8 codes of the normal channels, ascending order
 *   scale [rows]          fp32 scales
 *   outl  [rows, nO]      bf16 bit copies of the outlier channels, O order
 * Returns 0, or -1 when O is invalid.
 */
int orc_quantize_rows(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                      const int32_t *O, int64_t nO,
                      int8_t *codes, float *scale, uint16_t *outl)
{
    if (orc_validate_outliers(O, nO, K) != 0 || ld < K) return -1;
    char *is_outlier = (char *)calloc((size_t)K, 1);
    if (!is_outlier) return -1;
    for (int64_t j = 0; j < nO; ++j) is_outlier[O[j]] = 1;
    const int64_t KN = K - nO;

#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *row = src + r * ld;

        /* a = absolute maximum over the normal channels only. */
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (is_outlier[k]) continue;
            float v = fabsf(orc_bf16_to_f32(row[k]));
            if (v > a) a = v;
        }
        float s = a / 7.0f;
        if (a == 0.0f) s = 0.0f;
        scale[r] = s;

        /* Codes of the normal channels, in ascending channel order. */
        int64_t j = 0;
        for (int64_t k = 0; k < K; ++k) {
            if (is_outlier[k]) continue;
            int q = 0;
            if (a != 0.0f) {
                float x = orc_bf16_to_f32(row[k]);
                float t = x / s;
                q = (int)nearbyintf(t); /* default mode: nearest, ties to even */
                if (q > ORC_QMAX) q = ORC_QMAX;
                if (q < -ORC_QMAX) q = -ORC_QMAX;
            }
            codes[r * KN + j] = (int8_t)q;
            ++j;
        }

        /* Compact outlier tensor: bit copies of the channels in O. */
        for (int64_t jo = 0; jo < nO; ++jo) outl[r * nO + jo] = row[O[jo]];
    }
    free(is_outlier);
    return 0;
}

/*
 * Storage layout of the packed 4-bit normal part: row r occupies `row_bytes`
 * bytes; byte j holds code 2j in its low nibble and code 2j+1 in its high
 * nibble, each as 4-bit two's complement; bytes past the codes are zero.
 */
int orc_pack_int4(const int8_t *codes, int64_t rows, int64_t KN, int64_t row_bytes,
                  uint8_t *packed)
{
    if (row_bytes * 2 < KN) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        uint8_t *dst = packed + r * row_bytes;
        memset(dst, 0, (size_t)row_bytes);
        for (int64_t j = 0; j < KN; ++j) {
            uint8_t nib = (uint8_t)(codes[r * KN + j]) & 0x0F;
            if (j % 2 == 0)
                dst[j / 2] |= nib;
            else
                dst[j / 2] |= (uint8_t)(nib << 4);
        }
    }
    return 0;
}

/*
 * Static channel table (the pages' "static mask", one word per 8 channels):
 * word c = (number of outlier channels below 8c) << 8 | bit e set when
 * channel 8c+e is an outlier.  K must be a multiple of 8.
 */
int orc_chan_table(const int32_t *O, int64_t nO, int64_t K, uint32_t *table)
{
    if (orc_validate_outliers(O, nO, K) != 0 || K % 8 != 0) return -1;
    for (int64_t c = 0; c < K / 8; ++c) {
        uint32_t below = 0, mask = 0;
        for (int64_t j = 0; j < nO; ++j) {
            if (O[j] < 8 * c) ++below;
            else if (O[j] < 8 * c + 8) mask |= 1u << (O[j] - 8 * c);
        }
        table[c] = (below << 8) | mask;
    }
    return 0;
}

/*
 * Dual-path products for `Mr` activation rows against all N weight rows.
 * Inputs are the outputs of orc_quantize_rows for X and for W.
 *   acc_i [Mr, N]  exact integer dot product of the codes (int64)
 *   acc_o [Mr, N]  16-bit branch: sum of X_O * W_O in fp64
 *   y     [Mr, N]  acc_i * s_x * s_w + acc_o in fp64 (no final rounding)
 */
int orc_dual_linear_rows(const int8_t *qx, const float *sx, const uint16_t *xo, int64_t Mr,
                         const int8_t *qw, const float *sw, const uint16_t *wo, int64_t N,
                         int64_t KN, int64_t nO,
                         int64_t *acc_i, double *acc_o, double *y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < Mr; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t ai = 0;
            for (int64_t j = 0; j < KN; ++j)
                ai += (int64_t)qx[m * KN + j] * (int64_t)qw[n * KN + j];
            double ao = 0.0;
            for (int64_t j = 0; j < nO; ++j)
                ao += (double)orc_bf16_to_f32(xo[m * nO + j]) *
                      (double)orc_bf16_to_f32(wo[n * nO + j]);
            acc_i[m * N + n] = ai;
            acc_o[m * N + n] = ao;
            y[m * N + n] = (double)ai * (double)sx[m] * (double)sw[n] + ao;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ FP8 low path
 * OSC (arXiv:2604.12782), abstract and "technical framework": for the inputs
 * of W2 (the down projection), where outlier clustering is less pronounced,
 * the 4-bit path falls back to FP8.  The pages fix nothing further; the
 * reading taken here keeps the rest of the layer unchanged:
 *   - format E4M3 (4 exponent bits, bias 7, 3 mantissa bits, subnormals
 *     m * 2^-9, largest finite value 448, no infinities);
 *   - s = a / 448 with a the absolute maximum over the normal channels (fp32,
 *     IEEE division), one scale per token row of X and per output row of W;
 *   - code = E4M3 nearest to the fp32 quotient t = x / s, ties to the even
 *     code, magnitudes above 448 saturate to 448 (t can exceed 448 by a
 *     rounding error at the absolute-maximum element);
 *   - the sign follows the quotient, as in any IEEE-style conversion: a
 *     negative t that rounds to zero gives -0 (0x80);
 *   - a == 0: s = 0 and every code is 0x00;
 *   - the outlier channels still run through the 16-bit branch (nO = 0 gives
 *     a plain FP8 GEMM).
 */
#define ORC_E4M3_MAX 448.0

/* Value of an E4M3 code (sign bit 7, exponent bits 6..3, mantissa bits 2..0). */
double orc_e4m3_decode(uint8_t code)
{
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Nearest E4M3 code to t (finite), ties to the even code, saturating at
 * 448.  The non-negative finite codes 0x00..0x7E are increasing in value, so
 * the neighbours of |t| are found by bisection over them. */
uint8_t orc_e4m3_encode(float t)
{
    const uint8_t sign = signbit(t) ? 0x80 : 0x00;
    const double v = fabs((double)t);
    if (v >= ORC_E4M3_MAX) return (uint8_t)(sign | 0x7E);
    int lo = 0, hi = 0x7E; /* decode(lo) <= v < decode(hi) */
    while (hi - lo > 1) {
        const int mid = (lo + hi) / 2;
        if (orc_e4m3_decode((uint8_t)mid) <= v) lo = mid; else hi = mid;
    }
    const double dl = v - orc_e4m3_decode((uint8_t)lo), dh = orc_e4m3_decode((uint8_t)hi) - v;
    const int code = (dl < dh) ? lo : (dh < dl) ? hi : ((lo % 2 == 0) ? lo : hi);
    return (uint8_t)(sign | code); /* a negative value that rounds to zero gives -0 (0x80) */
}

int orc_e4m3_encode_array(const float *t, int64_t n, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i) codes[i] = orc_e4m3_encode(t[i]);
    return 0;
}

int orc_e4m3_decode_array(const uint8_t *codes, int64_t n, double *v)
{
    for (int64_t i = 0; i < n; ++i) v[i] = orc_e4m3_decode(codes[i]);
    return 0;
}

/* Quantize-and-gather with the FP8 low path; outputs as orc_quantize_rows,
 * with E4M3 codes (uint8) in place of the INT4 codes. */
int orc_quantize_rows_fp8(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                          const int32_t *O, int64_t nO,
                          uint8_t *codes, float *scale, uint16_t *outl)
{
    if (orc_validate_outliers(O, nO, K) != 0 || ld < K) return -1;
    char *is_outlier = (char *)calloc((size_t)K, 1);
    if (!is_outlier) return -1;
    for (int64_t j = 0; j < nO; ++j) is_outlier[O[j]] = 1;
    const int64_t KN = K - nO;

#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *row = src + r * ld;
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (is_outlier[k]) continue;
            float v = fabsf(orc_bf16_to_f32(row[k]));
            if (v > a) a = v;
        }
        float s = a / 448.0f;
        if (a == 0.0f) s = 0.0f;
        scale[r] = s;
        int64_t j = 0;
        for (int64_t k = 0; k < K; ++k) {
            if (is_outlier[k]) continue;
            uint8_t q = 0;
            if (a != 0.0f) {
                float t = orc_bf16_to_f32(row[k]) / s;
                q = orc_e4m3_encode(t);
            }
            codes[r * KN + j] = q;
            ++j;
        }
        for (int64_t jo = 0; jo < nO; ++jo) outl[r * nO + jo] = row[O[jo]];
    }
    free(is_outlier);
    return 0;
}

/* Dual-path products with the FP8 low path:
 *   acc_8 [Mr, N]  sum of decoded E4M3 products, fp64 (each product exact)
 *   acc_o [Mr, N]  16-bit branch, fp64
 *   y     [Mr, N]  acc_8 * s_x * s_w + acc_o, fp64 */
int orc_dual_linear_rows_fp8(const uint8_t *qx, const float *sx, const uint16_t *xo, int64_t Mr,
                             const uint8_t *qw, const float *sw, const uint16_t *wo, int64_t N,
                             int64_t KN, int64_t nO,
                             double *acc_8, double *acc_o, double *y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < Mr; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double a8 = 0.0;
            for (int64_t j = 0; j < KN; ++j)
                a8 += orc_e4m3_decode(qx[m * KN + j]) * orc_e4m3_decode(qw[n * KN + j]);
            double ao = 0.0;
            for (int64_t j = 0; j < nO; ++j)
                ao += (double)orc_bf16_to_f32(xo[m * nO + j]) *
                      (double)orc_bf16_to_f32(wo[n * nO + j]);
            acc_8[m * N + n] = a8;
            acc_o[m * N + n] = ao;
            y[m * N + n] = a8 * (double)sx[m] * (double)sw[n] + ao;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ micro-scaling FP4 low path
 * OSC (arXiv:2604.12782), abstract: the channel split fits 4-bit
 * micro-scaling hardware; SQ-format write-up of arXiv:2512.05409, section 8:
 * the format also works with FP8/FP4 data types.  The pages name no block
 * format, so the reading taken is the open MX definition of FP4 (MXFP4):
 *   - the normal channels of a row, in ascending channel order, are cut into
 *     blocks of 32 consecutive entries (j = 32b .. 32b+31; the last block may
 *     be partial, the missing entries count as zero);
 *   - every block has one power-of-two scale 2^E stored as an E8M0 byte
 *     e8 = E + 127: E = floor(log2(a)) - 2 with a the block's absolute
 *     maximum (2 is the largest exponent of E2M1), clamped to [-127, 127];
 *     a == 0 gives E = -127 (byte 0);
 *   - every entry becomes the E2M1 code (sign bit 3, exponent bits 2..1, bias
 *     1, mantissa bit 0: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) nearest to
 *     t = x / 2^E (exact), ties to the even code, magnitudes above 6
 *     saturated to 6, the sign bit copied from x (so -0 and negative values
 *     that round to zero give code 8);
 *   - the outlier channels still run through the 16-bit branch, and
 *     Y = sum_b 2^(Ex + Ew) * sum_{j in b} e(x_j) e(w_j) + sum_{k in O} X W.
 * No per-row fp32 scale remains: both operands carry their block scales. */
#define ORC_MX_BLOCK 32
#define ORC_E2M1_MAX 6.0

/* Value of an E2M1 code. */
double orc_e2m1_decode(uint8_t code)
{
    const int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -v : v;
}

/* Nearest E2M1 code to t, ties to the even code (mantissa bit 0),
 * saturating at 6; sign bit from t.  Codes 0..7 increase in value, so the
 * neighbours of |t| are found by a linear scan. */
uint8_t orc_e2m1_encode(double t)
{
    const uint8_t sign = signbit(t) ? 8 : 0;
    const double v = fabs(t);
    if (v >= ORC_E2M1_MAX) return (uint8_t)(sign | 7);
    int lo = 0;
    while (lo < 6 && orc_e2m1_decode((uint8_t)(lo + 1)) <= v) ++lo;
    const int hi = lo + 1; /* decode(lo) <= v < decode(hi) */
    const double dl = v - orc_e2m1_decode((uint8_t)lo), dh = orc_e2m1_decode((uint8_t)hi) - v;
    const int code = (dl < dh) ? lo : (dh < dl) ? hi : ((lo % 2 == 0) ? lo : hi);
    return (uint8_t)(sign | code);
}

int orc_e2m1_encode_array(const double *t, int64_t n, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i) codes[i] = orc_e2m1_encode(t[i]);
    return 0;
}

/* Block exponent E (before the E8M0 bias) of a block with absolute maximum a. */
int orc_mx_block_exponent(double a)
{
    if (a == 0.0) return -127;
    int e2;
    frexp(a, &e2); /* a = f * 2^e2, f in [0.5, 1): floor(log2 a) = e2 - 1 */
    int E = (e2 - 1) - 2;
    if (E < -127) E = -127;
    if (E > 127) E = 127;
    return E;
}

/* Quantize-and-gather with the MXFP4 low path.
 * Outputs (dense, caller-allocated):
 *   codes [rows, K - nO]          one E2M1 code per byte (unpacked)
 *   e8    [rows, ceil((K-nO)/32)] E8M0 block-scale bytes
 *   outl  [rows, nO]              bf16 bit copies of the outlier channels */
int orc_quantize_rows_mx(const uint16_t *src, int64_t rows, int64_t K, int64_t ld,
                         const int32_t *O, int64_t nO,
                         uint8_t *codes, uint8_t *e8, uint16_t *outl)
{
    if (orc_validate_outliers(O, nO, K) != 0 || ld < K) return -1;
    const int64_t KN = K - nO, NB = (KN + ORC_MX_BLOCK - 1) / ORC_MX_BLOCK;
    int64_t *normal = (int64_t *)malloc((size_t)(KN > 0 ? KN : 1) * sizeof(int64_t));
    char *is_outlier = (char *)calloc((size_t)K, 1);
    if (!normal || !is_outlier) { free(normal); free(is_outlier); return -1; }
    for (int64_t j = 0; j < nO; ++j) is_outlier[O[j]] = 1;
    for (int64_t k = 0, j = 0; k < K; ++k)
        if (!is_outlier[k]) normal[j++] = k;

#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *row = src + r * ld;
        for (int64_t b = 0; b < NB; ++b) {
            const int64_t j0 = b * ORC_MX_BLOCK;
            const int64_t j1 = (j0 + ORC_MX_BLOCK < KN) ? j0 + ORC_MX_BLOCK : KN;
            double a = 0.0;
            for (int64_t j = j0; j < j1; ++j) {
                const double v = fabs((double)orc_bf16_to_f32(row[normal[j]]));
                if (v > a) a = v;
            }
            const int E = orc_mx_block_exponent(a);
            e8[r * NB + b] = (uint8_t)(E + 127);
            for (int64_t j = j0; j < j1; ++j) {
                const double x = (double)orc_bf16_to_f32(row[normal[j]]);
                codes[r * KN + j] = orc_e2m1_encode(ldexp(x, -E)); /* exact: a power-of-two rescale */
            }
        }
        for (int64_t jo = 0; jo < nO; ++jo) outl[r * nO + jo] = row[O[jo]];
    }
    free(normal);
    free(is_outlier);
    return 0;
}

/* Dual-path products with the MXFP4 low path:
 *   acc_mx [Mr, N]  sum over blocks of 2^(Ex+Ew) * (exact block sum of decoded
 *                   E2M1 products), fp64, blocks in order
 *   acc_o  [Mr, N]  16-bit branch, fp64
 *   y      [Mr, N]  acc_mx + acc_o, fp64 */
int orc_dual_linear_rows_mx(const uint8_t *qx, const uint8_t *ex, const uint16_t *xo, int64_t Mr,
                            const uint8_t *qw, const uint8_t *ew, const uint16_t *wo, int64_t N,
                            int64_t KN, int64_t nO,
                            double *acc_mx, double *acc_o, double *y)
{
    const int64_t NB = (KN + ORC_MX_BLOCK - 1) / ORC_MX_BLOCK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < Mr; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double amx = 0.0;
            for (int64_t b = 0; b < NB; ++b) {
                const int64_t j0 = b * ORC_MX_BLOCK;
                const int64_t j1 = (j0 + ORC_MX_BLOCK < KN) ? j0 + ORC_MX_BLOCK : KN;
                double s = 0.0;
                for (int64_t j = j0; j < j1; ++j) s += orc_e2m1_decode(qx[m * KN + j]) * orc_e2m1_decode(qw[n * KN + j]);
                amx += ldexp(s, ((int)ex[m * NB + b] - 127) + ((int)ew[n * NB + b] - 127));
            }
            double ao = 0.0;
            for (int64_t j = 0; j < nO; ++j)
                ao += (double)orc_bf16_to_f32(xo[m * nO + j]) * (double)orc_bf16_to_f32(wo[n * nO + j]);
            acc_mx[m * N + n] = amx;
            acc_o[m * N + n] = ao;
            y[m * N + n] = amx + ao;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ element-level SQ-format weights
 * SQ-format write-up of arXiv:2512.05409: section 3 (the low-precision part
 * keeps its storage format with a mask value marking the positions that need
 * high precision, which a gather unit handles as sparse data), section 7
 * (banks with a fixed sparsity pattern each), section 9 (symmetric
 * quantization, the unused top code is the mask; in each bank the top (1-s)
 * fraction by importance is high precision), section 8 (FP8/FP4 combination);
 * the abstract (the sparse part is accelerated in high precision).  Readings
 * taken where the pages leave it open:
 *   - a bank is `bank` consecutive input channels of one weight row; its `h`
 *     channels with the largest |w| are high precision (importance without
 *     calibration Hessians reduces to the magnitude), ties to the lower index;
 *   - low part: symmetric INT4 over the row's low channels, s_lo = a/7 (fp32),
 *     code = clamp(rint(fl(w/s_lo)), -7, 7), and the mask code -8 at every
 *     high position; a == 0 gives s_lo = 0 and zero codes (the mask stays);
 *   - high part: FP8 E4M3 with s_hi = (absmax over the row's high channels) /
 *     448, code = E4M3 nearest to fl(w/s_hi) as for the FP8 path;
 *   - activations: per token, INT4 over all K channels for the low part and
 *     E4M3 over all K channels for the high part (the two row quantizers of
 *     this file with an empty outlier set);
 *   - Y = s_x4 s_lo sum_{k low} qx4 qw + s_x8 s_hi sum_{k high} e(x) e(w).
 */

/* One weight row: in each bank, mark the h channels with the largest |w|
 * (ties to the lower index) in hi[k] (1 high, 0 low). */
static void orc_bank_select(const uint16_t *row, int64_t K, int bank, int h, char *hi)
{
    for (int64_t g = 0; g < K / bank; ++g) {
        for (int i = 0; i < bank; ++i) {
            const int64_t k = g * bank + i;
            const float vi = fabsf(orc_bf16_to_f32(row[k]));
            int rank = 0; /* channels of the bank ranked above channel k */
            for (int j = 0; j < bank; ++j) {
                const float vj = fabsf(orc_bf16_to_f32(row[g * bank + j]));
                if (vj > vi || (vj == vi && j < i)) ++rank;
            }
            hi[k] = (char)(rank < h);
        }
    }
}

/* Element-level SQ-format of weight rows (bf16 [rows, ld]).
 * Outputs: lo [rows, K] int8 codes (-8 at high positions), s_lo [rows],
 * hi_mask [rows, K] (1 at high positions), hi_codes [rows, K] E4M3 (0 at low
 * positions), s_hi [rows].  K % bank == 0, 1 <= h < bank. */
int orc_sqf_weights(const uint16_t *src, int64_t rows, int64_t K, int64_t ld, int bank, int h,
                    int8_t *lo, float *s_lo, uint8_t *hi_mask, uint8_t *hi_codes, float *s_hi)
{
    if (bank < 2 || h < 1 || h >= bank || K % bank != 0 || ld < K) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *row = src + r * ld;
        char *hi = (char *)(hi_mask + r * K);
        orc_bank_select(row, K, bank, h, hi);
        float a = 0.0f, ah = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            const float v = fabsf(orc_bf16_to_f32(row[k]));
            if (hi[k]) { if (v > ah) ah = v; }
            else if (v > a) a = v;
        }
        const float s = (a == 0.0f) ? 0.0f : a / 7.0f;
        const float sh = (ah == 0.0f) ? 0.0f : ah / 448.0f;
        s_lo[r] = s;
        s_hi[r] = sh;
        for (int64_t k = 0; k < K; ++k) {
            const float x = orc_bf16_to_f32(row[k]);
            if (hi[k]) {
                lo[r * K + k] = -8;
                hi_codes[r * K + k] = (ah == 0.0f) ? 0 : orc_e4m3_encode(x / sh);
            } else {
                int q = 0;
                if (a != 0.0f) {
                    q = (int)nearbyintf(x / s);
                    if (q > ORC_QMAX) q = ORC_QMAX;
                    if (q < -ORC_QMAX) q = -ORC_QMAX;
                }
                lo[r * K + k] = (int8_t)q;
                hi_codes[r * K + k] = 0;
            }
        }
    }
    return 0;
}

/* Products of the element-level format for Mr token rows against N weight
 * rows.  qx4 / sx4: INT4 codes and scales of the tokens over all K channels;
 * qx8 / sx8: their E4M3 codes and scales.
 *   acc_lo [Mr, N]  exact integer sum over the low positions (int64)
 *   acc_hi [Mr, N]  sum of decoded E4M3 products over the high positions (fp64)
 *   y      [Mr, N]  acc_lo sx4 s_lo + acc_hi sx8 s_hi (fp64) */
int orc_sqf_linear_rows(const int8_t *qx4, const float *sx4, const uint8_t *qx8, const float *sx8, int64_t Mr,
                        const int8_t *lo, const float *s_lo, const uint8_t *hi_mask, const uint8_t *hi_codes,
                        const float *s_hi, int64_t N, int64_t K, int64_t *acc_lo, double *acc_hi, double *y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < Mr; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t al = 0;
            double ahs = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                if (hi_mask[n * K + k])
                    ahs += orc_e4m3_decode(qx8[m * K + k]) * orc_e4m3_decode(hi_codes[n * K + k]);
                else
                    al += (int64_t)qx4[m * K + k] * (int64_t)lo[n * K + k];
            }
            acc_lo[m * N + n] = al;
            acc_hi[m * N + n] = ahs;
            y[m * N + n] = (double)al * (double)sx4[m] * (double)s_lo[n] + ahs * (double)sx8[m] * (double)s_hi[n];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ static outlier selection
 * SQ-format write-up of arXiv:2512.05409, section 5 (static strategy for
 * activations) and section 9 (importance scores): the mean activation of each
 * channel is collected on calibration data, and the importance of a channel
 * is its activation times its contribution through the weights.  OSC
 * (arXiv:2604.12782) selects the outlier channels offline, group-wise.
 * Reading taken:
 *   score[k] = mean_m |X[m,k]| * ||W[:,k]||_2                   (fp64)
 *   group g (channels g*G .. g*G+G-1) scores sum_j score[g*G+j]  (G = 1: per channel)
 *   O = the channels of the nO/G groups with the largest group score, ties to
 *       the lower group index, in ascending channel order.
 * Each column sum runs over the rows in order, 0 to rows-1, in fp64 (|x| and
 * x*x of a bf16 value are exact in fp64, so the only rounding is that of the
 * additions).  This is the plain statement of the two sums.  Any order of
 * adding n nonnegative terms in fp64 lands within (n-1)*2^-53 of the exact
 * sum, relative, so another evaluation order differs from this one by at
 * most twice that.
 */
static double orc_col_sum(const uint16_t *A, int64_t rows, int64_t ld, int64_t k, int square)
{
    double total = 0.0;
    for (int64_t r = 0; r < rows; ++r) {
        const double v = (double)orc_bf16_to_f32(A[r * ld + k]);
        total += square ? v * v : fabs(v);
    }
    return total;
}

static const double *orc_sort_keys;
static int orc_group_cmp(const void *pa, const void *pb)
{
    const int64_t a = *(const int64_t *)pa, b = *(const int64_t *)pb;
    if (orc_sort_keys[a] > orc_sort_keys[b]) return -1;
    if (orc_sort_keys[a] < orc_sort_keys[b]) return 1;
    return (a < b) ? -1 : (a > b) ? 1 : 0;
}

/* X: calibration activations bf16 [Mc, ldx]; W: weights bf16 [N, ldw].
 * Outputs: O [nO] int32 (ascending), score [K] fp64 per channel.
 * Returns 0, or -1 on invalid sizes. */
int orc_select_outliers(const uint16_t *X, int64_t Mc, int64_t K, int64_t ldx,
                        const uint16_t *W, int64_t N, int64_t ldw,
                        int64_t nO, int64_t group, int32_t *O, double *score)
{
    if (Mc <= 0 || N <= 0 || K <= 0 || ldx < K || ldw < K || group < 1 || K % group != 0 || nO < 0 || nO > K ||
        nO % group != 0)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k) {
        const double mean_abs = orc_col_sum(X, Mc, ldx, k, 0) / (double)Mc;
        score[k] = mean_abs * sqrt(orc_col_sum(W, N, ldw, k, 1));
    }
    const int64_t ng = K / group, pick = nO / group;
    double *gs = (double *)malloc((size_t)ng * sizeof(double));
    int64_t *idx = (int64_t *)malloc((size_t)ng * sizeof(int64_t));
    char *chosen = (char *)calloc((size_t)ng, 1);
    if (!gs || !idx || !chosen) { free(gs); free(idx); free(chosen); return -1; }
    for (int64_t g = 0; g < ng; ++g) {
        double t = 0.0;
        for (int64_t j = 0; j < group; ++j) t += score[g * group + j];
        gs[g] = t;
        idx[g] = g;
    }
    orc_sort_keys = gs;
    qsort(idx, (size_t)ng, sizeof(int64_t), orc_group_cmp);
    for (int64_t i = 0; i < pick; ++i) chosen[idx[i]] = 1;
    int64_t j = 0;
    for (int64_t g = 0; g < ng; ++g)
        if (chosen[g])
            for (int64_t c = 0; c < group; ++c) O[j++] = (int32_t)(g * group + c);
    free(gs);
    free(idx);
    free(chosen);
    return 0;
}

#ifdef _OPENMP
#include <omp.h>
#endif
/* Number of host threads the parallel loops above use. */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
