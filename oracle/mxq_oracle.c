/*
 * mxq_oracle.c -- plain, slow, obviously-correct CPU reference (TEST INFRASTRUCTURE).
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg load this
 * library.  It shares no code with the CUDA library and must never be reached from
 * the product path.  See mxq_oracle.h for the sources and the definitions adopted.
 *
 * Style: each function is the definition written out, in double precision where the
 * method does not fix fp32.  Scaling by powers of two is done with ldexp and is
 * exact; the only roundings are rint() (IEEE round-half-even in the default mode)
 * where a definition rounds, and the fp32 divide / multiply the per-group scale rule
 * prescribes.  Build without -ffast-math and with -ffp-contract=off.
 */
#include "mxq_oracle.h"

#include <math.h>
#include <string.h>

/* ---- bf16 ------------------------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32: widening is exact, subnormals kept. */
double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_floor_log2(double a) {
    int e;
    (void)frexp(a, &e); /* a = f * 2^e with f in [0.5, 1) */
    return e - 1;
}

/* Round a double to the nearest bf16, ties to even, keeping subnormals (quantum
 * 2^-133 below 2^-126) and overflowing to infinity.  NaN becomes 0x7FC0. */
uint16_t oracle_double_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int p = oracle_floor_log2(a);
    int quantum_exp = (p < -126 ? -126 : p) - 7; /* 7 stored fraction bits */
    double r = ldexp(rint(ldexp(a, -quantum_exp)), quantum_exp);
    if (r >= 0x1p128) return (uint16_t)(sign | 0x7F80);
    float f = (float)r; /* exact: r has at most 8 significant bits and is in range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* ---- E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits) --------------- */

double oracle_e4m3_decode(uint8_t code) {
    int s = code >> 7, E = (code >> 3) & 15, m = code & 7;
    if (E == 15 && m == 7) return NAN;
    double mag = (E == 0) ? ldexp((double)m, -9)          /* subnormal: m * 2^-9 */
                          : ldexp((double)(8 + m), E - 10); /* (1 + m/8) * 2^(E-7) */
    return s ? -mag : mag;
}

/* Nearest finite E4M3 value, ties to the even code, magnitudes of 448 and above
 * saturate to 448.  The sign is kept, so -0 and negative values that round to zero
 * give 0x80.  NaN gives 0x7F with the input's sign bit. */
uint8_t oracle_e4m3_encode(double v) {
    uint8_t sign = signbit(v) ? 0x80 : 0;
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    double a = fabs(v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < 0x1p-6) {
        /* subnormal range, spacing 2^-9; a result of 8 is the smallest normal 0x08 */
        double m = rint(ldexp(a, 9));
        return (uint8_t)(sign | (uint8_t)m);
    }
    int p = oracle_floor_log2(a);        /* -6 .. 8 */
    double r = rint(ldexp(a, 3 - p));   /* 8 .. 16: implicit bit plus 3 fraction bits */
    int E = p + 7, m = (int)r - 8;
    if (m == 8) { /* rounded up into the next binade */
        E += 1;
        m = 0;
    }
    return (uint8_t)(sign | (uint8_t)((E << 3) | m));
}

void oracle_e4m3_encode_f64_array(const double* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e4m3_encode_f32_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode((double)v[i]);
}

void oracle_double_to_bf16_array(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_double_to_bf16(v[i]);
}

/* ---- E8M0 --------------------------------------------------------------------- */

double oracle_e8m0_decode(uint8_t b) {
    if (b == 0xFF) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* Scale byte of a block: e = floor(log2(amax)) - 8, clamped to [-127, 127]; an
 * all-zero block takes the bottom of the range (log2 0 = -inf); a block whose amax
 * is not finite takes the NaN scale 0xFF. */
uint8_t oracle_mx_scale_byte(double amax) {
    if (isnan(amax) || isinf(amax)) return 0xFF;
    int e;
    if (amax == 0.0) {
        e = -127;
    } else {
        e = oracle_floor_log2(amax) - 8;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
    }
    return (uint8_t)(e + 127);
}

/* ---- MX quantize ---------------------------------------------------------------- */

/* Quantize one 32-element block given as 32 bf16 values read with `stride`
 * (elements) between them; writes 32 codes with `qstride` between them and
 * returns the scale byte. */
static uint8_t quantize_block(const uint16_t* x, int64_t stride, uint8_t* q, int64_t qstride) {
    double amax = 0.0;
    int nonfinite = 0;
    for (int i = 0; i < 32; ++i) {
        double v = oracle_bf16_to_double(x[i * stride]);
        if (isnan(v) || isinf(v)) nonfinite = 1;
        else if (fabs(v) > amax) amax = fabs(v);
    }
    uint8_t b = nonfinite ? 0xFF : oracle_mx_scale_byte(amax);
    for (int i = 0; i < 32; ++i) {
        double v = oracle_bf16_to_double(x[i * stride]);
        uint8_t code;
        if (b == 0xFF) {
            code = (uint8_t)((signbit(v) ? 0x80 : 0) | 0x7F);
        } else {
            int e = (int)b - 127;
            code = oracle_e4m3_encode(ldexp(v, -e)); /* x * 2^-e, exact in double */
        }
        q[i * qstride] = code;
    }
    return b;
}

void oracle_mx_quantize(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols, int axes,
                        uint8_t* q_row, uint8_t* s_row, uint8_t* q_col, uint8_t* s_col) {
    for (int64_t e = 0; e < batch; ++e) {
        const uint16_t* xm = x + e * rows * cols;
        if (axes & 1) { /* 1x32 blocks along each row */
            for (int64_t r = 0; r < rows; ++r)
                for (int64_t j = 0; j < cols / 32; ++j)
                    s_row[(e * rows + r) * (cols / 32) + j] =
                        quantize_block(xm + r * cols + 32 * j, 1,
                                       q_row + (e * rows + r) * cols + 32 * j, 1);
        }
        if (axes & 2) { /* 32x1 blocks down each column; output is the transpose */
            for (int64_t c = 0; c < cols; ++c)
                for (int64_t i = 0; i < rows / 32; ++i)
                    s_col[(e * cols + c) * (rows / 32) + i] =
                        quantize_block(xm + (32 * i) * cols + c, cols,
                                       q_col + (e * cols + c) * rows + 32 * i, 1);
        }
    }
}

/* ---- MX dequantize -------------------------------------------------------------- */

static uint16_t dequantize_one(uint8_t code, uint8_t b) {
    double v = oracle_e4m3_decode(code) * oracle_e8m0_decode(b); /* exact product */
    return oracle_double_to_bf16(v);
}

void oracle_mx_dequantize(const uint8_t* q, const uint8_t* s, int64_t batch, int64_t rows,
                          int64_t cols, int axis, uint16_t* y) {
    for (int64_t e = 0; e < batch; ++e)
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c) {
                uint8_t code, b;
                if (axis == 1) {
                    code = q[(e * rows + r) * cols + c];
                    b = s[(e * rows + r) * (cols / 32) + c / 32];
                } else {
                    code = q[(e * cols + c) * rows + r];
                    b = s[(e * cols + c) * (rows / 32) + r / 32];
                }
                y[(e * rows + r) * cols + c] = dequantize_one(code, b);
            }
}

/* ---- per-group rowwise FP8 scaling ------------------------------------------------ */

/* Group g covers rows [start_g, end_g): start_0 = 0, end_g = offs[g] clamped to
 * [end_{g-1}, M], start_g = end_{g-1}. */
void oracle_group_bounds(const int32_t* offs, int32_t G, int64_t M, int64_t* start, int64_t* end) {
    int64_t prev = 0;
    for (int32_t g = 0; g < G; ++g) {
        int64_t e = offs[g];
        if (e < prev) e = prev;
        if (e > M) e = M;
        start[g] = prev;
        end[g] = e;
        prev = e;
    }
}

void oracle_per_group_quant(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                            int32_t G, int layout, uint8_t* q, float* scales) {
    const float eps = 1e-12f; /* the fp32 value nearest to 1e-12 */
    int64_t prev = 0;
    for (int32_t g = 0; g < G; ++g) {
        int64_t start = prev, end = offs[g];
        if (end < prev) end = prev;
        if (end > M) end = M;
        prev = end;
        for (int64_t k = 0; k < K; ++k) {
            /* amax over the group's rows of this feature (exact: bf16 values) */
            double amax = 0.0;
            int nonfinite = 0;
            for (int64_t m = start; m < end; ++m) {
                double v = oracle_bf16_to_double(x[m * K + k]);
                if (isnan(v) || isinf(v)) nonfinite = 1;
                else if (fabs(v) > amax) amax = fabs(v);
            }
            float a = (float)amax; /* exact */
            float s = nonfinite ? NAN : 448.0f / fmaxf(a, eps); /* IEEE fp32 divide */
            scales[(int64_t)g * K + k] = s;
            for (int64_t m = start; m < end; ++m) {
                float xf = (float)oracle_bf16_to_double(x[m * K + k]);
                float p = xf * s; /* one fp32 RNE multiply */
                uint8_t code = oracle_e4m3_encode((double)p);
                if (layout == 0) q[m * K + k] = code;
                else q[k * M + m] = code;
            }
        }
    }
}

/* ---- layouts for the scaled grouped GEMM ------------------------------------------ */

/* Plain transpose of each (rows, cols) byte matrix of the batch. */
void oracle_transpose_u8(const uint8_t* src, int64_t batch, int64_t rows, int64_t cols, uint8_t* dst) {
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c)
                dst[(b * cols + c) * rows + r] = src[(b * rows + r) * cols + c];
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int64_t oracle_mx_scales_blocked_bytes(int64_t batch, int64_t rows, int64_t n_k, int32_t G) {
    const int64_t col_tiles = ceil_div(n_k, 4);
    if (G <= 0) return batch * ceil_div(rows, 128) * col_tiles * 512;
    /* sum over groups of 128 * ceil(n_g / 128) <= rows + 127 G, a multiple of 128 */
    return ((rows + 127 * (int64_t)G) / 128) * col_tiles * 512;
}

/* Byte offset of (padded row p, scale column k) in the blocked layout whose rows have
 * col_tiles tiles of 4 scale columns. */
static int64_t blocked_offset(int64_t p, int64_t k, int64_t col_tiles) {
    const int64_t tile = (p / 128) * col_tiles + k / 4;
    const int64_t r = p % 128;
    return tile * 512 + (r % 32) * 16 + (r / 32) * 4 + (k % 4);
}

void oracle_mx_scales_to_blocked(const uint8_t* s, int64_t batch, int64_t rows, int64_t n_k,
                                 const int32_t* offs, int32_t G, uint8_t* out) {
    const int64_t col_tiles = ceil_div(n_k, 4);
    if (G <= 0) {
        const int64_t per_matrix = ceil_div(rows, 128) * 128; /* padded rows */
        for (int64_t b = 0; b < batch; ++b)
            for (int64_t p = 0; p < per_matrix; ++p)
                for (int64_t k = 0; k < 4 * col_tiles; ++k) {
                    const uint8_t v = (p < rows && k < n_k) ? s[(b * rows + p) * n_k + k] : 0;
                    out[blocked_offset(b * per_matrix + p, k, col_tiles)] = v;
                }
        return;
    }
    int64_t prev = 0, padded = 0;
    for (int32_t g = 0; g < G; ++g) {
        int64_t end = offs[g];
        if (end < prev) end = prev;
        if (end > rows) end = rows;
        const int64_t n = end - prev, n_pad = ceil_div(n, 128) * 128;
        for (int64_t i = 0; i < n_pad; ++i)
            for (int64_t k = 0; k < 4 * col_tiles; ++k) {
                const uint8_t v = (i < n && k < n_k) ? s[(prev + i) * n_k + k] : 0;
                out[blocked_offset(padded + i, k, col_tiles)] = v;
            }
        padded += n_pad;
        prev = end;
    }
}

/* ---- MXFP8 grouped GEMM ---------------------------------------------------------------- */

void oracle_mx_grouped_gemm(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb, const uint8_t* sb,
                            const int32_t* offs, int32_t G, int64_t M, int64_t N, int64_t K, double* out,
                            double* abs_sum) {
    const int64_t nk = K / 32;
    int64_t prev = 0;
    for (int32_t g = 0; g < G; ++g) {
        int64_t end = offs[g];
        if (end < prev) end = prev;
        if (end > M) end = M;
        for (int64_t m = prev; m < end; ++m)
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0, mag = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    const double a = oracle_e4m3_decode(qa[m * K + k]) * oracle_e8m0_decode(sa[m * nk + k / 32]);
                    const double b = oracle_e4m3_decode(qb[((int64_t)g * N + n) * K + k]) *
                                     oracle_e8m0_decode(sb[((int64_t)g * N + n) * nk + k / 32]);
                    acc += a * b;
                    mag += fabs(a * b);
                }
                out[m * N + n] = acc;
                if (abs_sum) abs_sum[m * N + n] = mag;
            }
        prev = end;
    }
}
