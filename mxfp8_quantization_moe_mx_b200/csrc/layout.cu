// layout.cu -- layout kernels between the quantizers and the scaled grouped GEMM (sm_100a).
//
// Source: torchao "[moe training] fix uncoalesced global accesses in per group rowwise
// scaling kernel", Summary: for many groups the per-group kernel writes its E4M3 output
// column-major and the output is transformed to the row-major layout the scaled grouped
// GEMM's left operand needs afterwards.  And the MXFP8 grouped GEMMs of the torchtitan
// mxfp8 all-to-all page (Performance) take E8M0 block scales in the tiled order the
// tensor cores' block-scaled MMA reads them in.
//
//  * transpose_u8: (batch, rows, cols) bytes -> (batch, cols, rows).  A CTA stages a
//    256 x 128-byte tile in shared memory with 16-byte loads (a warp reads four whole
//    128-byte rows; 16-byte chunks XOR-swizzled by row group); each thread then reads a
//    32-row x 4-column block (conflict-free thanks to the swizzle), transposes it in
//    registers with byte permutes (eight per 4 x 4 block) and writes four 32-byte
//    runs, one per output row; a warp's four row groups make each of its 32 output
//    rows one whole 128-byte line.  Needs rows and cols multiples of 16 and 16-byte-aligned
//    pointers; other shapes take a plain 32 x 32 byte-tile kernel.
//  * scales_to_blocked: E8M0 scales (rows, n_k) -> tiles of 128 rows x 4 scale
//    columns, row r and column k of a tile at byte (r % 32) * 16 + (r / 32) * 4 + k,
//    tiles ordered by row tile then column tile; each group's rows (by the offsets'
//    clamp rule) padded to whole tiles.  One CTA per padded 128-row tile: it finds its
//    group from the device offsets (a running maximum and a sum of padded sizes, one
//    warp, no host sync), then each thread writes one 16-byte tile line (the four
//    row quarters' four scales of one line).

#include <cstdint>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

// ---- byte transpose ------------------------------------------------------------------

constexpr int TR_ROWS = 256, TR_COLS = 128;  // source tile (rows x bytes)

// Transpose of a 4 x 4 byte block: w[i] holds row i (byte j = column j); returns the
// four columns (byte i = row i).
__device__ __forceinline__ void transpose4x4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t& c0,
                                             uint32_t& c1, uint32_t& c2, uint32_t& c3) {
    const uint32_t a_lo = __byte_perm(w0, w1, 0x5140), a_hi = __byte_perm(w0, w1, 0x7362);
    const uint32_t b_lo = __byte_perm(w2, w3, 0x5140), b_hi = __byte_perm(w2, w3, 0x7362);
    c0 = __byte_perm(a_lo, b_lo, 0x5410);
    c1 = __byte_perm(a_lo, b_lo, 0x7632);
    c2 = __byte_perm(a_hi, b_hi, 0x5410);
    c3 = __byte_perm(a_hi, b_hi, 0x7632);
}

// 16-byte chunk position of chunk `ch` of tile row r: rows in different 32-row groups
// are XOR-swizzled apart so the transposed reads below hit distinct banks.
__device__ __forceinline__ int tr_chunk(int r, int ch) { return ch ^ (((r >> 5) & 3) << 1); }

__global__ void __launch_bounds__(256) transpose_u8_kernel(const uint8_t* __restrict__ src, int64_t rows,
                                                          int64_t cols, uint8_t* __restrict__ dst) {
    __shared__ __align__(16) uint8_t tile[TR_ROWS * TR_COLS];
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int64_t b = blockIdx.z;
    const int64_t R0 = (int64_t)blockIdx.y * TR_ROWS, C0 = (int64_t)blockIdx.x * TR_COLS;
    const uint8_t* s = src + b * rows * cols;
    uint8_t* d = dst + b * rows * cols;
    // load: thread t takes 16-byte chunk t % 8 of rows t / 8 + 32 i (a warp: 4 whole rows)
    {
        const int ch = t & 7;
        const int64_t c = C0 + 16 * ch;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = (t >> 3) + 32 * i;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (R0 + r < rows && c < cols) v = ld_nc_v4(s + (R0 + r) * cols + c);
            *reinterpret_cast<uint4*>(tile + r * TR_COLS + 16 * tr_chunk(r, ch)) = v;
        }
    }
    __syncthreads();
    // transpose: thread (cg, rg) -> source columns 4cg..4cg+3 x rows 32rg..32rg+31 ->
    // output rows C0 + 4cg + j, bytes R0 + 32rg .. +31.  Lane (rgl = lane % 4, cgl =
    // lane / 4): a warp covers 8 column groups x 4 row groups, so each of its 32 output
    // rows receives 128 contiguous bytes (a whole line) from four lanes.
    const int rg = 4 * (warp & 1) + (lane & 3), cg = 8 * (warp >> 1) + (lane >> 2);
    uint32_t col[4][8];
#pragma unroll
    for (int i4 = 0; i4 < 8; ++i4) {
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = 32 * rg + 4 * i4 + u;
            w[u] = *reinterpret_cast<const uint32_t*>(tile + r * TR_COLS + 16 * tr_chunk(r, cg >> 2) + 4 * (cg & 3));
        }
        transpose4x4(w[0], w[1], w[2], w[3], col[0][i4], col[1][i4], col[2][i4], col[3][i4]);
    }
    const int64_t r_out = R0 + 32 * rg;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int64_t c = C0 + 4 * cg + j;
        if (c >= cols) continue;
        uint8_t* o = d + c * rows + r_out;
        if (r_out < rows) *reinterpret_cast<uint4*>(o) = make_uint4(col[j][0], col[j][1], col[j][2], col[j][3]);
        if (r_out + 16 < rows)
            *reinterpret_cast<uint4*>(o + 16) = make_uint4(col[j][4], col[j][5], col[j][6], col[j][7]);
    }
}

// Any shape and alignment: 32 x 32 byte tiles, one byte per thread and step.
__global__ void __launch_bounds__(256) transpose_u8_any_kernel(const uint8_t* __restrict__ src, int64_t rows,
                                                              int64_t cols, uint8_t* __restrict__ dst) {
    __shared__ uint8_t tile[32][33];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    const int64_t b = blockIdx.z;
    const int64_t R0 = (int64_t)blockIdx.y * 32, C0 = (int64_t)blockIdx.x * 32;
    const uint8_t* s = src + b * rows * cols;
    uint8_t* d = dst + b * rows * cols;
    for (int i = ty; i < 32; i += 8)
        if (R0 + i < rows && C0 + tx < cols) tile[i][tx] = s[(R0 + i) * cols + C0 + tx];
    __syncthreads();
    for (int i = ty; i < 32; i += 8)
        if (C0 + i < cols && R0 + tx < rows) d[(C0 + i) * rows + R0 + tx] = tile[tx][i];
}

cudaError_t launch_transpose_u8(const uint8_t* src, int64_t batch, int64_t rows, int64_t cols, uint8_t* dst,
                                cudaStream_t stream) {
    constexpr int64_t LIM = 65535;
    const bool fast = rows % 16 == 0 && cols % 16 == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
                      (reinterpret_cast<uintptr_t>(dst) & 15) == 0;
    const int64_t tr = fast ? TR_ROWS : 32, tc = fast ? TR_COLS : 32;
    const int64_t gx = (cols + tc - 1) / tc, gy = (rows + tr - 1) / tr;
    if (gx > 0x7FFFFFFFLL || gy > LIM) return cudaErrorInvalidConfiguration;
    for (int64_t b0 = 0; b0 < batch; b0 += LIM) {
        const dim3 grid((unsigned)gx, (unsigned)gy, (unsigned)std::min(batch - b0, LIM));
        const uint8_t* s = src + b0 * rows * cols;
        uint8_t* d = dst + b0 * rows * cols;
        if (fast)
            transpose_u8_kernel<<<grid, 256, 0, stream>>>(s, rows, cols, d);
        else
            transpose_u8_any_kernel<<<grid, 256, 0, stream>>>(s, rows, cols, d);
    }
    return cudaGetLastError();
}

// ---- E8M0 scales -> blocked tensor-core layout ----------------------------------------------

// One CTA per padded 128-row tile (blockIdx.x); blockIdx.y = matrix (G == 0 only).
// Thread t writes tile line l = t % 32 of column tiles j = t / 32, t / 32 + 8, ...: the
// 16 bytes (a = 0..3 row quarters) x (c = 0..3 scale columns) of rows 32a + l.
__global__ void __launch_bounds__(256) scales_to_blocked_kernel(const uint8_t* __restrict__ s, int64_t rows,
                                                               int64_t n_k, const int32_t* __restrict__ offs,
                                                               int32_t G, uint8_t* __restrict__ out) {
    __shared__ int64_t info[3];  // source first row of the tile, valid rows in it, destination tile index
    const int t = threadIdx.x, lane = t & 31;
    const int64_t col_tiles = (n_k + 3) / 4;
    const int64_t tile = blockIdx.x;
    if (G <= 0) {
        const int64_t per_matrix = (rows + 127) / 128;
        if (t == 0) {
            info[0] = (int64_t)blockIdx.y * rows + tile * 128;
            info[1] = min((int64_t)128, rows - tile * 128);
            info[2] = (int64_t)blockIdx.y * per_matrix + tile;
        }
    } else if (t < 32) {
        // padded tiles of the groups, in order: the group whose tiles hold `tile`
        int run = 0;           // running maximum of the offsets (the clamp rule)
        int64_t padded = 0;    // padded tiles of the groups before the current chunk
        bool found = false;
        for (int h0 = 0; h0 < G && !found; h0 += 32) {
            const int h = h0 + lane;
            int e = h < G ? offs[h] : 0;
            e = max(e, 0);
            // inclusive running maximum over the chunk, carried from the previous chunks
#pragma unroll
            for (int sh = 1; sh < 32; sh <<= 1) {
                const int o = __shfl_up_sync(FULL_MASK, e, sh);
                if (lane >= sh) e = max(e, o);
            }
            e = max(e, run);
            const int up = __shfl_up_sync(FULL_MASK, e, 1);
            const int prev_e = lane == 0 ? run : up;
            const int64_t end = min((int64_t)e, rows), start = min((int64_t)prev_e, rows);
            const int64_t n_tiles = h < G ? (end - start + 127) / 128 : 0;
            // exclusive prefix sum of the tile counts
            int64_t inc = n_tiles;
#pragma unroll
            for (int sh = 1; sh < 32; sh <<= 1) {
                const int64_t o = __shfl_up_sync(FULL_MASK, inc, sh);
                if (lane >= sh) inc += o;
            }
            const int64_t first = padded + inc - n_tiles;
            const bool mine = h < G && tile >= first && tile < first + n_tiles;
            const unsigned who = __ballot_sync(FULL_MASK, mine);
            if (mine) {
                info[0] = start + (tile - first) * 128;
                info[1] = min((int64_t)128, end - info[0]);
                info[2] = tile;
            }
            found = who != 0;
            padded += __shfl_sync(FULL_MASK, inc, 31);
            run = __shfl_sync(FULL_MASK, e, 31);
        }
        if (!found && lane == 0) info[1] = -1;  // past the last used tile: nothing to write
    }
    __syncthreads();
    const int64_t r0 = info[0], valid = info[1], dt = info[2];
    if (valid < 0) return;
    const bool vec = (n_k & 3) == 0 && (reinterpret_cast<uintptr_t>(s) & 3) == 0;
    for (int64_t j = t >> 5; j < col_tiles; j += 8) {
        uint32_t w[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int r = 32 * a + lane;
            uint32_t v = 0;
            if (r < valid) {
                const uint8_t* src = s + (r0 + r) * n_k + 4 * j;
                if (vec) {
                    v = __ldg(reinterpret_cast<const uint32_t*>(src));
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if (4 * j + c < n_k) v |= (uint32_t)src[c] << (8 * c);
                }
            }
            w[a] = v;
        }
        *reinterpret_cast<uint4*>(out + (dt * col_tiles + j) * 512 + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

int64_t scales_blocked_bytes(int64_t batch, int64_t rows, int64_t n_k, int32_t G) {
    const int64_t col_tiles = (n_k + 3) / 4;
    if (G <= 0) return batch * ((rows + 127) / 128) * col_tiles * 512;
    return ((rows + 127 * (int64_t)G) / 128) * col_tiles * 512;
}

cudaError_t launch_scales_to_blocked(const uint8_t* s, int64_t batch, int64_t rows, int64_t n_k,
                                     const int32_t* offs, int32_t G, uint8_t* out, cudaStream_t stream) {
    constexpr int64_t LIM = 65535;
    if (G <= 0) {
        const int64_t tiles = (rows + 127) / 128;
        if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
        for (int64_t b0 = 0; b0 < batch; b0 += LIM) {
            const dim3 grid((unsigned)tiles, (unsigned)std::min(batch - b0, LIM));
            const int64_t per_matrix_out = tiles * ((n_k + 3) / 4) * 512;
            scales_to_blocked_kernel<<<grid, 256, 0, stream>>>(s + b0 * rows * n_k, rows, n_k, nullptr, 0,
                                                               out + b0 * per_matrix_out);
        }
    } else {
        const int64_t tiles = (rows + 127 * (int64_t)G) / 128;  // bound on the used tiles
        if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
        if (tiles > 0) scales_to_blocked_kernel<<<(unsigned)tiles, 256, 0, stream>>>(s, rows, n_k, offs, G, out);
    }
    return cudaGetLastError();
}

}  // namespace mxq
