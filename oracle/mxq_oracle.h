/*
 * mxq_oracle.h -- plain CPU reference for the MXFP8 / per-group FP8 quantization path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or call
 * this code; only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no source, header, table or helper with the CUDA library.
 *
 * Sources of the operations (page title, section):
 *   - "[mxfp8 MoE training] Support mxfp8 all to all in expert parallel" (torchtitan
 *     PR 1765), Summary: the all-to-all wrapper quantizes its input to mxfp8 (e4m3
 *     data + e8m0 scales), exchanges both, and dequantizes back to the original
 *     precision.  The page names the formats but never spells out their arithmetic.
 *   - "[moe training] fix uncoalesced global accesses in per group rowwise scaling
 *     kernel" (pytorch/ao PR 2761), Summary and Performance tables: the per-group
 *     rowwise FP8 scaling kernel on a (16640, 5120) bf16 input split into 16..128
 *     groups, with row-major or column-major E4M3 output.
 *
 * The arithmetic below is the plain OCP-MX reading: E4M3 elements (bias 7, max 448,
 * no infinities, S.1111.111 is NaN), E8M0 scales 2^(b-127), one scale per 32
 * elements derived as floor(log2(block amax)) - 8 clamped to E8M0's range, and
 * saturating round-to-nearest-even element encoding.  The per-group scale is
 * 448 / max(amax, 1e-12) in fp32.  Every reading of a point the pages leave open is
 * listed in the design notes of the repository.
 *
 * Everything here is single-threaded plain C.  Floating-point work that the method
 * does not fix to fp32 is done in double precision, where every step used below is
 * exact, so the only roundings are the ones the definitions call for.
 */
#ifndef MXQ_ORACLE_H
#define MXQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- scalar formats ---------------------------------------------------------- */
double  oracle_bf16_to_double(uint16_t bits);
uint16_t oracle_double_to_bf16(double v);          /* RNE, subnormals kept, overflow -> inf */
double  oracle_e4m3_decode(uint8_t code);           /* NaN for S.1111.111 */
uint8_t oracle_e4m3_encode(double v);               /* saturating RNE; NaN in -> 0x7F|sign */
double  oracle_e8m0_decode(uint8_t b);              /* 2^(b-127); NaN for 0xFF */
int     oracle_floor_log2(double a);                /* exact floor(log2 a), a > 0 finite */
uint8_t oracle_mx_scale_byte(double amax);          /* E8M0 byte for a block amax */

/* Array forms of the scalar routines (plain loops), for exhaustive sweeps. */
void oracle_e4m3_encode_f64_array(const double* v, int64_t n, uint8_t* out);
void oracle_e4m3_encode_f32_array(const float* v, int64_t n, uint8_t* out);
void oracle_double_to_bf16_array(const double* v, int64_t n, uint16_t* out);

/* ---- MX quantize / dequantize ------------------------------------------------ */
/* axes: bit 0 = 1x32 row blocks, bit 1 = 32x1 column blocks.
 * x: (batch, rows, cols) bf16 bits, row-major.  rows, cols multiples of 32.
 * q_row (batch, rows, cols), s_row (batch, rows, cols/32);
 * q_col (batch, cols, rows) = per-matrix transpose, s_col (batch, cols, rows/32). */
void oracle_mx_quantize(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols, int axes,
                        uint8_t* q_row, uint8_t* s_row, uint8_t* q_col, uint8_t* s_col);

/* axis 1: q/s in the row layout above; axis 2: q/s in the column layout above.
 * y: (batch, rows, cols) bf16 bits, row-major, for both. */
void oracle_mx_dequantize(const uint8_t* q, const uint8_t* s, int64_t batch, int64_t rows,
                          int64_t cols, int axis, uint16_t* y);

/* ---- per-group rowwise FP8 scaling ------------------------------------------- */
/* x: (M, K) bf16 bits row-major; offs: G int32 exclusive end offsets (host memory).
 * layout 0: q (M, K) row-major; layout 1: q (K, M) (column-major view of (M, K)).
 * scales: (G, K) fp32.  Rows past the last group's end are left untouched. */
void oracle_per_group_quant(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                            int32_t G, int layout, uint8_t* q, float* scales);

/* The group bounds the clamp rule gives: start[g], end[g] for g in [0, G). */
void oracle_group_bounds(const int32_t* offs, int32_t G, int64_t M, int64_t* start, int64_t* end);

/* ---- layouts the scaled grouped GEMM consumes --------------------------------- */
/* Byte transpose: dst[b][c][r] = src[b][r][c] for (batch, rows, cols) src.  The
 * column-major per-group codes (K, M) become the row-major (M, K) ones with
 * rows = K, cols = M. */
void oracle_transpose_u8(const uint8_t* src, int64_t batch, int64_t rows, int64_t cols, uint8_t* dst);

/* Capacity, in bytes, of the blocked scale layout below. */
int64_t oracle_mx_scales_blocked_bytes(int64_t batch, int64_t rows, int64_t n_k, int32_t G);

/* E8M0 block scales (batch, rows, n_k) -> the blocked layout of the tensor-core
 * block-scaled MMA: tiles of 128 rows x 4 scale columns (512 bytes); tile (t, j) of
 * a matrix (or of a group's padded rows) at byte (t * ceil(n_k/4) + j) * 512; inside
 * a tile, row r and scale column k at byte (r % 32) * 16 + (r / 32) * 4 + k.
 * G == 0: each matrix's rows padded to a multiple of 128, matrices one after another.
 * G > 0 (batch 1): the rows of group g (the clamp rule of oracle_group_bounds) start
 * at padded row P_g = sum over h < g of 128 * ceil(n_h / 128).  Padding bytes are 0;
 * bytes past the last used tile keep their value. */
void oracle_mx_scales_to_blocked(const uint8_t* s, int64_t batch, int64_t rows, int64_t n_k,
                                 const int32_t* offs, int32_t G, uint8_t* out);

/* ---- MXFP8 grouped GEMM (the consumer of the quantized expert tokens) ---------- */
/* out[m][n] = sum over k of E4M3(qa[m][k]) * 2^(sa[m][k/32] - 127)
 *                          * E4M3(qb[g][n][k]) * 2^(sb[g][n][k/32] - 127)
 * for every row m of group g (the clamp rule of oracle_group_bounds over M rows),
 * exactly in double precision (products of E4M3 values and powers of two are exact;
 * the sum is accumulated in double, whose error the tests bound).  qa (M, K) and sa
 * (M, K/32) are the row layout of oracle_mx_quantize; qb (G, N, K) and sb (G, N, K/32)
 * the row layout of the G expert matrices.  K % 32 == 0.  out (M, N) doubles; rows in
 * no group are left untouched.  abs_sum (M, N), if not NULL, receives
 * sum over k of |a_k * b_k| for the error bound. */
void oracle_mx_grouped_gemm(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb, const uint8_t* sb,
                            const int32_t* offs, int32_t G, int64_t M, int64_t N, int64_t K, double* out,
                            double* abs_sum);

#ifdef __cplusplus
}
#endif
#endif
