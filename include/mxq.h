/*
 * mxq.h -- C ABI of the B200 (sm_100a) MXFP8 / per-group FP8 quantization library
 * (libmxq.so).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every data pointer is a DEVICE pointer owned by the caller.  The library
 *    never allocates, frees or synchronizes; it only enqueues kernels.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Work runs asynchronously on that stream, in stream order.
 *  - Return value: an mxq_status.  Argument errors are found on the host before
 *    anything is launched, and then nothing is launched and no byte is written.
 *    MXQ_ERR_CUDA means a launch was rejected by the CUDA runtime; errors raised
 *    while a kernel runs surface, as usual, on the next synchronizing CUDA call.
 *  - Sizes are int64_t element counts.  A size of zero is a valid empty problem:
 *    the call returns MXQ_OK and launches nothing, and the data pointers of the empty
 *    tensors may be NULL (the per-group call with M == 0 still writes its scales
 *    when K > 0 and G > 0, so it still needs offs and scales).
 *  - bf16 tensors are IEEE binary32's upper halves (torch.bfloat16), little endian.
 *    E4M3 codes are OCP FP8 E4M3 ("e4m3fn": bias 7, max 448, no infinity,
 *    S.1111.111 = NaN).  E8M0 scales are biased exponents: value 2^(b-127),
 *    0xFF = NaN.
 *  - Alignment: bf16 and E4M3 tensors must start on a 16-byte boundary, fp32 scales
 *    on 4 bytes, offsets on 4 bytes; E8M0 scale arrays have no requirement.
 *
 * Where the operations come from (page title, section)
 * ----------------------------------------------------
 *  "[mxfp8 MoE training] Support mxfp8 all to all in expert parallel" (torchtitan
 *  PR 1765), Summary: the expert-parallel all-to-all is made cheaper by quantizing
 *  its payload to mxfp8 (e4m3 data plus e8m0 scales), exchanging both, and
 *  dequantizing on arrival.  mx_quantize and mx_dequantize are those two local steps.
 *
 *  "[moe training] fix uncoalesced global accesses in per group rowwise scaling
 *  kernel" (pytorch/ao PR 2761), Summary and Performance: the per-group rowwise FP8
 *  scaling kernel that feeds the scaled grouped GEMM, writing its E4M3 output in
 *  row-major (the GEMM's left operand) or column-major layout.
 *  fp8_per_group_rowwise_quant is that kernel.
 *
 *  The pages name the formats but not their arithmetic.  The library implements the
 *  plain OCP-MX reading, which the CPU oracle in the test suite also follows:
 *    MX block of 32:  b = clamp(floor(log2(amax)) - 8, -127, 127) + 127
 *                     (all-zero block: b = 0), q_i = satRNE_E4M3(x_i * 2^(127-b));
 *                     a block holding Inf or NaN gets b = 0xFF and q_i = 0x7F|sign.
 *    MX dequant:      y = bf16_RNE(E4M3(q) * 2^(b-127)); NaN code or NaN scale
 *                     gives the bf16 NaN 0x7FC0.
 *    per-group:       s[g,k] = fp32(448 / max(amax[g,k], fp32(1e-12))) (IEEE divide),
 *                     q[m,k] = satRNE_E4M3(fp32(x[m,k] * s[g(m),k])).
 *  Results are bit-exact with that reading (tolerance 0).
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXQ_OK = 0,
    MXQ_ERR_NULL = 1,            /* a required pointer is NULL */
    MXQ_ERR_SHAPE = 2,           /* negative size, size not a multiple the layout needs,
                                    or a size product that overflows int64 */
    MXQ_ERR_ALIGN = 3,           /* a pointer violates the alignment rule above */
    MXQ_ERR_ARG = 4,             /* an enum argument out of range */
    MXQ_ERR_CUDA = 5,            /* the CUDA runtime rejected a launch or an attribute call */
    MXQ_ERR_NOT_IMPLEMENTED = 6  /* reserved */
} mxq_status;

/* Default limit of the kernels' bounded waits (see mxq_set_wait_limit_ns). */
#define MXQ_WAIT_LIMIT_DEFAULT_NS 2000000000ull

/* Which block axes mx_quantize produces (bit mask) / which layout mx_dequantize reads. */
enum { MXQ_AXIS_ROW = 1,   /* 1x32 blocks along each row */
       MXQ_AXIS_COL = 2 }; /* 32x1 blocks down each column */

/* Output layouts of fp8_per_group_rowwise_quant. */
enum { MXQ_LAYOUT_ROW_MAJOR = 0, MXQ_LAYOUT_COL_MAJOR = 1 };

/*
 * mx_quantize -- MXFP8 quantize of a bf16 tensor along rows, columns, or both.
 * Source: the torchtitan page above, Summary ("quantizes the inputs to mxfp8").
 *
 *  x_bf16  (batch, rows, cols) bf16, row-major, 16-byte aligned.
 *  axes    MXQ_AXIS_ROW, MXQ_AXIS_COL or both; with both, x is read once.
 *  cols must be a multiple of 32, and so must rows when column blocks are requested
 *  (MXQ_ERR_SHAPE otherwise); 1x32 blocks alone take any number of rows (the token
 *  counts of an all-to-all split are arbitrary).
 *  Row blocks (MXQ_AXIS_ROW):
 *    q_row (batch, rows, cols) E4M3, 16-byte aligned;  s_row (batch, rows, cols/32) E8M0.
 *  Column blocks (MXQ_AXIS_COL), written transposed per matrix, so each block is
 *  contiguous -- the same bytes as row blocks of x^T:
 *    q_col (batch, cols, rows) E4M3, 16-byte aligned;  s_col (batch, cols, rows/32) E8M0.
 *  Pointers of an axis that is not requested are ignored and may be NULL.
 */
int mx_quantize(const void* x_bf16, int64_t batch, int64_t rows, int64_t cols, int axes,
                uint8_t* q_row, uint8_t* s_row, uint8_t* q_col, uint8_t* s_col,
                void* stream);

/*
 * mx_dequantize -- MXFP8 dequantize back to bf16.
 * Source: the torchtitan page above, Summary ("dequantize outputs back to original
 * precision").
 *
 *  axis MXQ_AXIS_ROW: q (batch, rows, cols) and s (batch, rows, cols/32), the row
 *       layout of mx_quantize.  axis MXQ_AXIS_COL: q (batch, cols, rows) and
 *       s (batch, cols, rows/32), its column layout.
 *  y_bf16 is always (batch, rows, cols) row-major bf16, 16-byte aligned.
 *  cols must be a multiple of 32; rows too for MXQ_AXIS_COL.
 */
int mx_dequantize(const uint8_t* q, const uint8_t* s, int64_t batch, int64_t rows,
                  int64_t cols, int axis, void* y_bf16, void* stream);

/*
 * fp8_per_group_rowwise_quant -- per-group rowwise FP8 scaling of expert tokens.
 * Source: the torchao page above, Summary and Performance.
 *
 *  x_bf16  (M, K) bf16 row-major, 16-byte aligned; K must be a multiple of 8.
 *  offs    G int32 exclusive END offsets, in DEVICE memory.  Group g is rows
 *          [start_g, end_g) with start_0 = 0, end_g = min(max(offs[g], end_{g-1}), M),
 *          start_g = end_{g-1}; so malformed offsets (decreasing, negative or past M)
 *          are clamped, never an error and never an out-of-bounds access.  Reading
 *          them needs no host synchronization.
 *  out_layout  MXQ_LAYOUT_ROW_MAJOR: q is (M, K) row-major;
 *              MXQ_LAYOUT_COL_MAJOR: q is (K, M) row-major, i.e. (M, K) column-major.
 *  q       E4M3 output, 16-byte aligned.  Bytes of rows that belong to no group
 *          (rows at or past end_{G-1}) are left untouched.
 *  scales  (G, K) fp32, written for every group, empty groups included
 *          (an empty group or all-zero feature gets 448 / fp32(1e-12)).
 *  G must be at most 65535.
 *  No scratch memory is needed: every CTA, or every thread-block cluster of up to 8
 *  CTAs, owns whole (group, column-slab) tiles, and no CTA waits on one outside its
 *  cluster.  A CTA waits a bounded time (2 s by default, see mxq_set_wait_limit_ns) for
 *  the copy of its tile into shared memory, and as long for its cluster's partial
 *  maxima.  If any CTA of a cluster gives up, the whole cluster skips that (group,
 *  column-slab) tile: none of its codes and none of its scales are written (a caller
 *  that pre-fills the outputs sees the fill there), and the event is counted (see
 *  mxq_wait_timeouts).  No output is ever derived from incomplete maxima.
 */
int fp8_per_group_rowwise_quant(const void* x_bf16, int64_t M, int64_t K, const int32_t* offs,
                                int32_t G, int out_layout, uint8_t* q, float* scales,
                                void* stream);

/*
 * fp8_per_group_rowwise_quant_batched -- per-group rowwise FP8 scaling of a 3-D tensor
 * of E matrices, each matrix its own group (no offsets).
 * Source: torchtitan "[float8] add float8 rowwise MoE prototype", Limitations (shared
 * experts need the grouped GEMM's left operand as a 3-D tensor); the arithmetic is that
 * of fp8_per_group_rowwise_quant with group e = rows [e M, (e + 1) M).
 *  x_bf16  (E, M, K) bf16, row-major, 16-byte aligned; K a multiple of 8.
 *  MXQ_LAYOUT_ROW_MAJOR: q (E, M, K).  MXQ_LAYOUT_COL_MAJOR: q (E, K, M), each matrix
 *  column-major (the K-major operand of a product that contracts over M).
 *  scales  (E, K) fp32, 448 / max(amax, fp32(1e-12)) per (matrix, feature).
 *  E <= 65535, E * M < 2^31.  Returns as fp8_per_group_rowwise_quant.
 */
int fp8_per_group_rowwise_quant_batched(const void* x_bf16, int64_t E, int64_t M, int64_t K, int out_layout,
                                        uint8_t* q, float* scales, void* stream);

/*
 * fp8_per_group_rowwise_plan -- what fp8_per_group_rowwise_quant launches for a problem
 * of these sizes (the group-offset scheduler's host side; its choice depends only on M,
 * K, G, the layout and the SM count, never on the offsets' values).  Host only:
 * launches nothing and touches no device memory.
 *  n_sm       SM count to plan for; 0 means the current device's (148 when no device
 *             can be queried).
 *  *kernel    0 nothing to launch (K == 0 or G == 0); 1 the shared-memory tile kernel
 *             (a (group, slab) tile per CTA, or per thread-block cluster of *cluster
 *             CTAs); 2 the pair kernel (column-major, two neighbouring groups per CTA);
 *             3 the two-pass streaming kernel (groups too large for the tiles).
 *  *slab_cols columns per tile (16, 32 or 64; 32 for the streaming kernel).
 *  *cluster   CTAs per tile (1, 2, 4 or 8).
 *  *tile_rows rows of its group a CTA keeps in shared memory (0 for the streaming
 *             kernel); a group's rows beyond that go through global memory.
 *  *threads   threads per CTA.
 *  Returns MXQ_OK, MXQ_ERR_NULL (an output pointer is NULL), MXQ_ERR_ARG (layout) or
 *  MXQ_ERR_SHAPE (the size rules of fp8_per_group_rowwise_quant).
 */
int fp8_per_group_rowwise_plan(int64_t M, int64_t K, int32_t G, int out_layout, int n_sm,
                               int* kernel, int* slab_cols, int* cluster, int* tile_rows,
                               int* threads);

/*
 * mxq_transpose_u8 -- byte transpose of each matrix of a batch:
 * dst[b][c][r] = src[b][r][c], src (batch, rows, cols), dst (batch, cols, rows).
 * Source: the torchao page above, Summary: for many groups the per-group kernel's
 * output is written column-major and then transformed to the row-major layout the
 * scaled grouped GEMM's left operand needs.  With src the column-major codes of
 * fp8_per_group_rowwise_quant, (K, M), rows = K and cols = M give the row-major
 * (M, K) codes.  Any sizes and alignments (the fast path wants rows and cols
 * multiples of 16 and both pointers 16-byte aligned).  src and dst must not overlap.
 * Returns MXQ_OK, MXQ_ERR_SHAPE, MXQ_ERR_NULL or MXQ_ERR_CUDA.
 */
int mxq_transpose_u8(const uint8_t* src, int64_t batch, int64_t rows, int64_t cols, uint8_t* dst, void* stream);

/*
 * mx_scales_to_blocked -- E8M0 block scales in the tiled order the tensor cores'
 * block-scaled MMA reads them in (the MXFP8 grouped GEMMs of the torchtitan page,
 * Performance, consume MX scales this way).
 *  s    (batch, rows, n_k) E8M0, row-major: the s_row output of mx_quantize (n_k =
 *       cols / 32), or its s_col output with rows = cols.
 *  Output: tiles of 128 rows x 4 scale columns (512 bytes); row r and scale column k
 *  of a tile at byte (r % 32) * 16 + (r / 32) * 4 + k; tile (t, j) of a matrix at
 *  byte (t * ceil(n_k / 4) + j) * 512 of that matrix's part.
 *  G == 0 (offs ignored, may be NULL): each matrix's rows padded to a multiple of
 *       128, matrices one after another.
 *  G > 0 (batch must be 1): offs are the G int32 end offsets of
 *       fp8_per_group_rowwise_quant (device memory, same clamp rule); group g's rows
 *       start at padded row P_g = sum over h < g of 128 * ceil(n_h / 128), so every
 *       group begins a fresh tile, as a grouped GEMM's 128-row M tiles need.
 *  Padding rows and scale columns are written as 0.  `out` must hold
 *  mx_scales_blocked_bytes(batch, rows, n_k, G) bytes, 16-byte aligned; bytes past
 *  the used tiles (G > 0) are left untouched.
 * Returns MXQ_OK, MXQ_ERR_SHAPE, MXQ_ERR_NULL, MXQ_ERR_ALIGN or MXQ_ERR_CUDA.
 */
int mx_scales_to_blocked(const uint8_t* s, int64_t batch, int64_t rows, int64_t n_k, const int32_t* offs,
                         int32_t G, uint8_t* out, void* stream);

/* Bytes mx_scales_to_blocked writes at most for these sizes (a bound when G > 0);
 * -1 for invalid sizes. */
int64_t mx_scales_blocked_bytes(int64_t batch, int64_t rows, int64_t n_k, int32_t G);

/*
 * mx_grouped_gemm -- MXFP8 grouped GEMM on the tensor cores' block-scaled MMA: the
 * consumer of the quantized expert tokens.  Source: the torchtitan mxfp8 all-to-all
 * page, Performance (the "+ MXFP8 Grouped GEMMs" rows), and the torchao per-group
 * page, Summary (the quantized tokens are the scaled grouped GEMM's left operand).
 *  For every row m of group g (offs: G int32 end offsets in device memory, the clamp
 *  rule of fp8_per_group_rowwise_quant over M rows):
 *    out[m][n] = bf16_RNE( sum_k A[m][k] 2^(sa[m][k/32]-127) * B[g][n][k] 2^(sb[g][n][k/32]-127) ),
 *  the products exact and the sum accumulated in fp32 by the tensor cores (not in a
 *  fixed order: results agree with the exact sum within fp32 accumulation error).
 *  qa   (M, K) E4M3, the 1x32 row layout of mx_quantize (16-byte aligned).
 *  sfa  its E8M0 scales (M, K/32) rearranged by mx_scales_to_blocked with the same
 *       offs and G (every group padded to 128-row tiles).
 *  qb   (G, N, K) E4M3: expert g's (N, K) matrix quantized with 1x32 blocks along K.
 *  sfb  its scales (G, N, K/32) rearranged by mx_scales_to_blocked with G = 0.
 *  out  (M, N) bf16 row-major; rows in no group are left untouched.
 *  K must be a multiple of 128 and N of 256; all pointers 16-byte aligned (offs 4).
 *  No scratch memory.  Every wait inside the kernel is bounded (2 s); a CTA that gives
 *  up stores nothing more (outputs it has not written are left untouched) and is
 *  counted by mxq_wait_timeouts.
 * Returns MXQ_OK, MXQ_ERR_SHAPE, MXQ_ERR_NULL, MXQ_ERR_ALIGN or MXQ_ERR_CUDA.
 */
int mx_grouped_gemm(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb, const uint8_t* sfb,
                    const int32_t* offs, int32_t G, int64_t M, int64_t N, int64_t K, void* out_bf16, void* stream);

/*
 * mx_e4m3_encode_f32 -- the fp32 -> E4M3 conversion every kernel above uses
 * (round to nearest even, magnitudes above 448 saturate to 448, NaN -> 0x7F|sign),
 * exposed so it can be checked exhaustively.  x: n fp32 values, 16-byte aligned;
 * q: n codes, 16-byte aligned.
 */
int mx_e4m3_encode_f32(const float* x, int64_t n, uint8_t* q, void* stream);

/* Human-readable name of a status code (static storage). */
const char* mxq_status_string(int status);

/* Text of the last CUDA runtime error seen by a call on this host thread, or "". */
const char* mxq_last_cuda_error(void);

/*
 * mxq_wait_timeouts -- diagnostics: *count receives the number of kernel CTAs on the
 * current device, since the library was loaded, that gave up a bounded wait (a copy
 * into shared memory, or a cluster sibling's partial maxima, that did not arrive in
 * time).  Their (group, column-slab) tiles were skipped: codes and scales there were
 * not written.  It is 0 in a healthy run.
 * Synchronous (waits for the device).  Returns MXQ_OK, MXQ_ERR_NULL or MXQ_ERR_CUDA.
 */
int mxq_wait_timeouts(unsigned int* count);

/*
 * mxq_wait_abandoned -- diagnostics: of the CTAs counted by mxq_wait_timeouts, those
 * whose copies in flight into their shared memory had still not landed 20 s after they
 * gave up.  Such a CTA exited anyway, so a late copy may have written into shared memory
 * that a later CTA owns: every output of every launch since is then undefined.  0 in a
 * healthy run.  Synchronous.  Returns MXQ_OK, MXQ_ERR_NULL or MXQ_ERR_CUDA.
 */
int mxq_wait_abandoned(unsigned int* count);

/*
 * mxq_set_wait_limit_ns -- diagnostics: the limit, in nanoseconds, of the bounded waits
 * of every later fp8_per_group_rowwise_quant launch from this process (default
 * MXQ_WAIT_LIMIT_DEFAULT_NS).  0 makes every such wait give up at once, so the give-up
 * path (skipped tiles, counted in mxq_wait_timeouts) can be exercised on purpose; the
 * wait for copies still in flight after giving up keeps its own long limit.  Takes
 * effect at launch; not thread-safe with respect to concurrent launches that expect
 * another limit.  Always returns MXQ_OK.
 */
int mxq_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* MXQ_H */
