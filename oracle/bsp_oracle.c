/*
 * bsp_oracle.c -- plain, slow CPU oracle for the block-scaled linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or constant generator with
 * the CUDA library.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (x86-64 SSE arithmetic: every float operation below is one IEEE-754 binary32
 * operation rounded to nearest-even; -ffp-contract=off forbids fused
 * multiply-adds, so each statement rounds exactly once.)
 *
 * Sources (page title, then the symbol or section on that page):
 *   [FV-QAT]  hao-ai-lab-FastVideo fastvideo/layers/quantization/nvfp4_qat_config.py
 *             -- NVFP4QATQuantizeMethod.apply, convert_model_to_fp4
 *   [FV-CFG]  hao-ai-lab-FastVideo fastvideo/layers/quantization/nvfp4_config.py
 *             -- module docstring ("e2m1 mantissa, fp32 alpha, layout_128x4 scale
 *             layout, group size 16"), _nvfp4_quantize, _mm_fp4, the register_fake
 *             shape functions, convert_model_to_nvfp4
 *   [SGL]     sgl-project sglang python/sglang/srt/layers/quantization/nvfp4_online.py
 *             -- ModelOptNvFp4OnlineFusedMoEMethod._quantize_weight_nvfp4
 *   [MXFP8]   vllm-omni vllm_omni/quantization/mxfp8_config.py
 *             -- DiffusionMXFP8Config docstring (group 32, float8_e8m0fnu, OCP MX)
 *
 * The pages name the formats (e2m1, e4m3, e8m0) and the data flow but print
 * none of the quantizer arithmetic (it sits inside a vendor library).  The
 * steps written here are the readings listed in the design notes, one
 * statement per step:
 *   NVFP4 group of 16 (x_i exact fp32 values of bf16 inputs, gs fp32):
 *     amax = max |x_i|
 *     s    = fl32(fl32(amax / 6) * gs)
 *     sfb  = e4m3_rne_satfinite(s),  sf = value(sfb)
 *     inv  = sf == 0 ? 0 : fl32(gs / sf)
 *     code_i = e2m1_rne_satfinite(fl32(x_i * inv))      (sign kept, -0 -> 0x8)
 *   MXFP8 group of 32:
 *     E = floor(log2(amax)) (-inf for amax == 0),  e = clamp(E - 8, -127, 127)
 *     sfb = e + 127,  q_i = e4m3_rne_satfinite(x_i * 2^-e)
 *   Scale bytes are placed with the 128x4 tile map (see bspo_sf_offset).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Scalar formats (value of every encoding, from the format definitions).    */
/* ------------------------------------------------------------------------ */

/* bf16: sign, 8-bit exponent (bias 127), 7-bit mantissa.  Exact in double. */
double bspo_bf16_value(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int e = (bits >> 7) & 0xFF;
    int m = bits & 0x7F;
    double v;
    if (e == 0xFF)
        v = (m == 0) ? INFINITY : NAN;
    else if (e == 0)
        v = ldexp((double)m, -126 - 7);
    else
        v = ldexp(1.0 + m / 128.0, e - 127);
    return sign ? -v : v;
}

/* fp16 (IEEE binary16): sign, 5-bit exponent (bias 15), 10-bit mantissa.
 * Exact in double. */
double bspo_f16_value(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int e = (bits >> 10) & 0x1F;
    int m = bits & 0x3FF;
    double v;
    if (e == 0x1F)
        v = (m == 0) ? INFINITY : NAN;
    else if (e == 0)
        v = ldexp((double)m, -14 - 10);
    else
        v = ldexp(1.0 + m / 1024.0, e - 15);
    return sign ? -v : v;
}

/* Input element formats of the quantizers: 0 = bf16, 1 = fp16. */
static double elem_value(uint16_t bits, int fmt)
{
    return fmt ? bspo_f16_value(bits) : bspo_bf16_value(bits);
}

/* e2m1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.  No inf/NaN. */
double bspo_e2m1_value(int code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -v : v;
}

/* e4m3 (fn): sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.
 * S.1111.111 is NaN; there is no infinity.  Largest finite value 448. */
double bspo_e4m3_value(int byte)
{
    int sign = (byte >> 7) & 1;
    int e = (byte >> 3) & 0xF;
    int m = byte & 7;
    double v;
    if (e == 0xF && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -6 - 3);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* e8m0: 8-bit unsigned exponent, value 2^(b - 127); 0xFF is NaN. */
double bspo_e8m0_value(int byte)
{
    if (byte == 0xFF)
        return NAN;
    return ldexp(1.0, byte - 127);
}

/* ------------------------------------------------------------------------ */
/* Round-to-nearest-even with saturation, by nearest-value search.           */
/* ------------------------------------------------------------------------ */

/* Returns the non-negative code in [0, ncodes) whose value is nearest to the
 * magnitude a; on a tie, the code with a clear lowest bit (the even mantissa).
 * The codes' values increase with the code, so this is RNE on the grid.  The
 * two candidates that decide a tie lie next to a, so their distances to a are
 * exact differences of short binary fractions. */
static int nearest_code(double a, double (*value)(int), int ncodes)
{
    int best = 0;
    double best_d = fabs(value(0) - a);
    for (int c = 1; c < ncodes; ++c) {
        double d = fabs(value(c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return best;
}

/* e2m1, RNE, saturating: |v| >= 6 gives magnitude code 7 (6.0).  The sign of
 * v (including -0) is kept.  NaN has no e2m1 encoding: returns -1. */
int bspo_e2m1_encode(double v)
{
    if (isnan(v))
        return -1;
    double a = fabs(v);
    int mag = (a >= 6.0) ? 7 : nearest_code(a, bspo_e2m1_value, 8);
    return (signbit(v) ? 8 : 0) | mag;
}

/* e4m3, RNE, saturating to +-448 (0x7E / 0xFE).  NaN -> 0x7F. */
int bspo_e4m3_encode(double v)
{
    if (isnan(v))
        return 0x7F;
    double a = fabs(v);
    int mag = (a >= 448.0) ? 0x7E : nearest_code(a, bspo_e4m3_value, 0x7F);
    return (signbit(v) ? 0x80 : 0) | mag;
}

/* bf16 nearest-even rounding of a double (no saturation: overflow gives inf,
 * as IEEE rounding does).  Used to round the fp64 reference GEMM output. */
uint16_t bspo_bf16_round(double y)
{
    if (isnan(y))
        return 0x7FC0;
    uint16_t sign = signbit(y) ? 0x8000 : 0;
    double a = fabs(y);
    float f = (float)a;
    uint32_t fb;
    memcpy(&fb, &f, 4);
    int32_t b = (int32_t)(fb >> 16); /* truncation of fl32(a) to bf16 */
    if (b >= 0x7F80)
        return sign | 0x7F80;
    int32_t best = -1;
    double best_d = 0.0;
    for (int32_t c = b - 1; c <= b + 1; ++c) {
        if (c < 0 || c > 0x7F80)
            continue;
        double cv = (c == 0x7F80) ? ldexp(1.0, 128) : bspo_bf16_value((uint16_t)c);
        double d = fabs(cv - a);
        if (best < 0 || d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return sign | (uint16_t)best;
}

/* ------------------------------------------------------------------------ */
/* 128x4 scale-factor tile map ([FV-QAT] / [FV-CFG]: layout_128x4).          */
/* ------------------------------------------------------------------------ */

/* Rows are padded to a multiple of 128 and scale columns to a multiple of 4.
 * The padded [rows, cols] scale matrix is cut into 128x4 tiles, stored one
 * after the other along the columns of a 128-row band, bands one after the
 * other.  Inside a 512-byte tile, row r (0..127) and column c (0..3) sit at
 * byte 16*(r % 32) + 4*(r / 32) + c. */
int64_t bspo_sf_offset(int64_t r, int64_t c, int64_t cols_padded)
{
    int64_t band = r / 128, tile_col = c / 4;
    int64_t rr = r % 128, cc = c % 4;
    return (band * (cols_padded / 4) + tile_col) * 512 + (rr % 32) * 16 + (rr / 32) * 4 + cc;
}

static int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

int64_t bspo_sf_bytes(int64_t rows, int64_t cols)
{
    return round_up(rows, 128) * round_up(cols, 4);
}

/* layout_8x4 ([FV] nvfp4_config.py: SfLayout.layout_8x4, rows padded to 8;
 * the pages do not give the byte order inside a tile -- the reading here is a
 * row-major 8x4 tile of 32 bytes, tiles ordered by row tile, then column
 * tile, like the 128x4 tiles). */
int64_t bspo_sf_offset_8x4(int64_t r, int64_t c, int64_t cols_padded)
{
    return ((r / 8) * (cols_padded / 4) + c / 4) * 32 + (r % 8) * 4 + c % 4;
}

int64_t bspo_sf_bytes_8x4(int64_t rows, int64_t cols)
{
    return round_up(rows, 8) * round_up(cols, 4);
}

/* Layouts: 0 = 128x4, 1 = 8x4. */
static int64_t sf_offset_layout(int64_t r, int64_t c, int64_t cols_padded, int layout)
{
    return layout ? bspo_sf_offset_8x4(r, c, cols_padded) : bspo_sf_offset(r, c, cols_padded);
}

static int64_t sf_bytes_layout(int64_t rows, int64_t cols, int layout)
{
    return layout ? bspo_sf_bytes_8x4(rows, cols) : bspo_sf_bytes(rows, cols);
}

/* ------------------------------------------------------------------------ */
/* Global scales ([FV-QAT] convert_model_to_fp4; [SGL] weight_scale_2).      */
/* ------------------------------------------------------------------------ */

/* amax of |x| as the pages compute it: abs().nan_to_num().amax() on the bf16
 * tensor -- NaN counts as 0 and +-inf as the largest finite bf16 value. */
float bspo_amax_fmt(const uint16_t *x, int64_t n, int fmt)
{
    double top = fmt ? bspo_f16_value(0x7BFF) : bspo_bf16_value(0x7F7F); /* largest finite */
    double amax = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double a = fabs(elem_value(x[i], fmt));
        if (isnan(a))
            a = 0.0;
        else if (isinf(a))
            a = top;
        if (a > amax)
            amax = a;
    }
    return (float)amax; /* exact: a bf16 or fp16 value */
}

float bspo_amax_bf16(const uint16_t *x, int64_t n)
{
    return bspo_amax_fmt(x, n, 0);
}

/* Encode global scale fp8_fp4_max/amax in fp32, fp8_fp4_max = e4m3_max * 6;
 * an all-zero tensor gets 1.0 (the guarded form of [SGL], where
 * weight_scale_2 is 1 when amax is 0).  [SGL] _quantize_weight_nvfp4 takes
 * e4m3_max = 448 (the largest e4m3), or 256 with its 4over6 setting. */
float bspo_nvfp4_global_scale_max(float amax, float fp8_fp4_max)
{
    if (amax > 0.0f)
        return fp8_fp4_max / amax;
    return 1.0f;
}

/* 448*6/amax: [FV-QAT] convert_model_to_fp4. */
float bspo_nvfp4_global_scale(float amax)
{
    return bspo_nvfp4_global_scale_max(amax, 448.0f * 6.0f);
}

/* Per-row (per-token) scales: gs[m] from the row amax; inv[m] = fl32(1/gs[m]),
 * the decode factor the GEMM applies to row m. */
void bspo_row_global_scales_fmt(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x, int fmt,
                                float *gs, float *inv_gs)
{
    for (int64_t m = 0; m < M; ++m) {
        float g = bspo_nvfp4_global_scale(bspo_amax_fmt(x + m * ld_x, K, fmt));
        if (gs)
            gs[m] = g;
        if (inv_gs)
            inv_gs[m] = 1.0f / g;
    }
}

void bspo_row_global_scales(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x,
                            float *gs, float *inv_gs)
{
    bspo_row_global_scales_fmt(x, M, K, ld_x, 0, gs, inv_gs);
}

/* ------------------------------------------------------------------------ */
/* NVFP4 quantizer.                                                          */
/* ------------------------------------------------------------------------ */

/* One group of 16 values; writes the e4m3 scale byte and 16 e2m1 codes. */
void bspo_nvfp4_quantize_group(const float *x, float gs, uint8_t *sfb_out, uint8_t *codes)
{
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > amax)
            amax = a;
    }
    float t = amax / 6.0f;
    float s = t * gs;
    int sfb = bspo_e4m3_encode((double)s);
    float sf = (float)bspo_e4m3_value(sfb);
    float inv = (sf == 0.0f) ? 0.0f : gs / sf;
    for (int i = 0; i < 16; ++i) {
        float v = x[i] * inv;
        /* A NaN product (a NaN element, or 0 * inf once the encode scale has
         * overflowed to +inf) has no e2m1 value; the saturating conversion
         * the quantizers use gives it the largest positive magnitude, code 7. */
        codes[i] = isnan(v) ? 7 : (uint8_t)bspo_e2m1_encode((double)v);
    }
    *sfb_out = (uint8_t)sfb;
}

/* x: bf16 (fmt 0) or fp16 (fmt 1) [M, K] with row stride ld_x (elements).
 * gs: one value, or one per row when per_row != 0.  codes: [M, K/2] bytes,
 * element 2j in the low nibble of byte j and element 2j+1 in the high nibble.
 * sf: bspo_sf_bytes(M, K/16) bytes in the 128x4 tile map; padding rows and
 * columns are 0.  Returns 0, or -1 when K is not a multiple of 16. */
int bspo_nvfp4_quantize_layout(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x, int fmt, int layout,
                               const float *gs, int per_row, uint8_t *codes, uint8_t *sf)
{
    if (K % 16 != 0 || M < 0)
        return -1;
    int64_t cols = K / 16, cols_p = round_up(cols, 4);
    memset(sf, 0, (size_t)sf_bytes_layout(M, cols, layout));
    float xs[16];
    uint8_t q[16];
    for (int64_t m = 0; m < M; ++m) {
        float g = per_row ? gs[m] : gs[0];
        for (int64_t c = 0; c < cols; ++c) {
            for (int i = 0; i < 16; ++i)
                xs[i] = (float)elem_value(x[m * ld_x + c * 16 + i], fmt); /* exact */
            uint8_t sfb;
            bspo_nvfp4_quantize_group(xs, g, &sfb, q);
            sf[sf_offset_layout(m, c, cols_p, layout)] = sfb;
            for (int j = 0; j < 8; ++j)
                codes[m * (K / 2) + c * 8 + j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
    return 0;
}

int bspo_nvfp4_quantize_fmt(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x, int fmt,
                            const float *gs, int per_row, uint8_t *codes, uint8_t *sf)
{
    return bspo_nvfp4_quantize_layout(x, M, K, ld_x, fmt, 0, gs, per_row, codes, sf);
}

int bspo_nvfp4_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x,
                        const float *gs, int per_row, uint8_t *codes, uint8_t *sf)
{
    return bspo_nvfp4_quantize_fmt(x, M, K, ld_x, 0, gs, per_row, codes, sf);
}

/* ------------------------------------------------------------------------ */
/* MXFP8 quantizer ([MXFP8]: 32 elements per float8_e8m0fnu scale, e4m3).     */
/* ------------------------------------------------------------------------ */

void bspo_mxfp8_quantize_group(const double *x, uint8_t *sfb_out, uint8_t *q)
{
    double amax = 0.0;
    for (int i = 0; i < 32; ++i)
        if (fabs(x[i]) > amax)
            amax = fabs(x[i]);
    int e;
    if (amax == 0.0) {
        e = -127; /* floor(log2 0) = -inf, clamped */
    } else {
        int fe;
        frexp(amax, &fe); /* amax = f * 2^fe, f in [0.5, 1) */
        int E = fe - 1;   /* floor(log2 amax) */
        e = E - 8;        /* 8 = exponent of the largest e4m3 value (448 = 1.75 * 2^8) */
        if (e < -127)
            e = -127;
        if (e > 127)
            e = 127;
    }
    for (int i = 0; i < 32; ++i)
        q[i] = (uint8_t)bspo_e4m3_encode(ldexp(x[i], -e));
    *sfb_out = (uint8_t)(e + 127);
}

/* x: bf16 [M, K] (row stride ld_x); q: e4m3 [M, K]; sf: bspo_sf_bytes(M, K/32)
 * bytes in the 128x4 tile map, padding 0.  Returns -1 if K % 32 != 0. */
int bspo_mxfp8_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x,
                        uint8_t *q, uint8_t *sf)
{
    if (K % 32 != 0 || M < 0)
        return -1;
    int64_t cols = K / 32, cols_p = round_up(cols, 4);
    memset(sf, 0, (size_t)bspo_sf_bytes(M, cols));
    double xs[32];
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t c = 0; c < cols; ++c) {
            for (int i = 0; i < 32; ++i)
                xs[i] = bspo_bf16_value(x[m * ld_x + c * 32 + i]);
            uint8_t sfb;
            bspo_mxfp8_quantize_group(xs, &sfb, q + m * K + c * 32);
            sf[bspo_sf_offset(m, c, cols_p)] = sfb;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Decoders (the GEMM operands as real numbers).                             */
/* ------------------------------------------------------------------------ */

/* Decode rows[i] of an NVFP4 operand ([rows_total, K/2] codes + tile-mapped
 * scales) to out[i*K + k] = e2m1(code) * e4m3(scale).  Exact in double. */
void bspo_nvfp4_dequantize_rows_layout(const uint8_t *codes, const uint8_t *sf, int64_t K, int layout,
                                       const int64_t *rows, int64_t nrows, double *out)
{
    int64_t cols_p = round_up(K / 16, 4);
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows[i];
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            int code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            double s = bspo_e4m3_value(sf[sf_offset_layout(r, k / 16, cols_p, layout)]);
            out[i * K + k] = bspo_e2m1_value(code) * s;
        }
    }
}

void bspo_nvfp4_dequantize_rows(const uint8_t *codes, const uint8_t *sf, int64_t K,
                                const int64_t *rows, int64_t nrows, double *out)
{
    bspo_nvfp4_dequantize_rows_layout(codes, sf, K, 0, rows, nrows, out);
}

void bspo_mxfp8_dequantize_rows(const uint8_t *q, const uint8_t *sf, int64_t K,
                                const int64_t *rows, int64_t nrows, double *out)
{
    int64_t cols_p = round_up(K / 32, 4);
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows[i];
        for (int64_t k = 0; k < K; ++k) {
            double s = bspo_e8m0_value(sf[bspo_sf_offset(r, k / 32, cols_p)]);
            out[i * K + k] = bspo_e4m3_value(q[r * K + k]) * s;
        }
    }
}

/* Element-wise helpers for array work from Python. */
void bspo_bf16_round_array(const double *y, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = bspo_bf16_round(y[i]);
}

void bspo_e4m3_encode_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = (uint8_t)bspo_e4m3_encode((double)v[i]);
}

void bspo_e2m1_encode_array(const float *v, int64_t n, int8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = (int8_t)bspo_e2m1_encode((double)v[i]);
}
