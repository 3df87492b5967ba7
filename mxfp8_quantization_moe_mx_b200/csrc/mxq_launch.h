// mxq_launch.h -- host-side launchers of the libmxq kernels (internal to the library).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mxq {

// Number of SMs of the current device (cached per device).
int sm_count();

// 2-D tensor map over a row-major bf16 (outer, inner) array: boxes of box_outer rows x
// box_inner elements, zero fill out of bounds, no swizzle.  False if the driver refuses.
bool encode_bf16_tile_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                          uint32_t box_outer);

// 2-D tensor map over a row-major byte (outer, inner) array, boxes of box_outer rows x
// box_inner bytes (box_inner <= 128), 128-byte swizzle (the tensor cores' K-major
// operand layout), zero fill out of bounds.
bool encode_u8_tile_map_sw128(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                              uint32_t box_outer);
// Row-major uint8 (outer, inner) tensor map, no swizzle, zero fill out of bounds.
bool encode_u8_map_plain(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                         uint32_t box_outer);

cudaError_t launch_quant_rows(const uint16_t* x, uint8_t* q, uint8_t* s, int64_t n_blocks,
                              cudaStream_t stream);
cudaError_t launch_quant_tile(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols,
                              bool do_row, bool do_col, uint8_t* q_row, uint8_t* s_row,
                              uint8_t* q_col, uint8_t* s_col, cudaStream_t stream);
cudaError_t launch_encode_f32(const float* x, uint8_t* q, int64_t n, cudaStream_t stream);

cudaError_t launch_dequant_rows(const uint8_t* q, const uint8_t* s, uint16_t* y, int64_t n,
                                cudaStream_t stream);
cudaError_t launch_dequant_tile(const uint8_t* q, const uint8_t* s, int64_t batch, int64_t rows,
                                int64_t cols, uint16_t* y, cudaStream_t stream);

// What launch_per_group runs for a problem (host logic only; also behind the C ABI's
// fp8_per_group_rowwise_plan): the kernel, slab width w, cluster size cl, rows a CTA
// keeps in shared memory (r_cap) and threads per CTA, for a device of n_sm SMs.
enum { PG_PLAN_NONE = 0, PG_PLAN_TILE = 1, PG_PLAN_PAIR = 2, PG_PLAN_STREAM = 3 };
struct PerGroupPlan {
    int kind, w, cl, r_cap, threads;
};
PerGroupPlan plan_per_group(int64_t M, int64_t K, int32_t G, bool col_major, int n_sm, bool batched = false);

// rows_per_group > 0: a batched tensor of G matrices of that many rows, each matrix one
// group (offs unused); column-major codes then go to one (K, rows_per_group) matrix per
// group.
cudaError_t launch_per_group(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, bool col_major, uint8_t* q, float* scales,
                             cudaStream_t stream, int rows_per_group = 0);

// Byte transpose of each (rows, cols) matrix of the batch.
cudaError_t launch_transpose_u8(const uint8_t* src, int64_t batch, int64_t rows, int64_t cols, uint8_t* dst,
                                cudaStream_t stream);

// E8M0 scales -> the 128 x 4 tiled layout of the block-scaled MMA (G > 0: per group).
int64_t scales_blocked_bytes(int64_t batch, int64_t rows, int64_t n_k, int32_t G);
cudaError_t launch_scales_to_blocked(const uint8_t* s, int64_t batch, int64_t rows, int64_t n_k,
                                     const int32_t* offs, int32_t G, uint8_t* out, cudaStream_t stream);

// MXFP8 grouped GEMM (tcgen05 block-scaled MMA); scales in the blocked layout.
cudaError_t launch_mx_grouped_gemm(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb, const uint8_t* sfb,
                                   const int32_t* offs, int32_t G, int64_t M, int64_t N, int64_t K, uint16_t* out,
                                   cudaStream_t stream);
unsigned int read_gemm_timeouts();

// Number of per-group CTAs that gave up a bounded wait, and of those whose copies in
// flight did not land within the drain limit either (synchronous reads).
unsigned int read_wait_timeouts();
unsigned int read_wait_abandoned();

// Limit of the bounded waits of later per-group launches (0: give up at once).
void set_wait_limit_ns(uint64_t ns);

}  // namespace mxq
