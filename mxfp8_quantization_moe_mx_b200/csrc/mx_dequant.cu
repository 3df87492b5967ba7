// mx_dequant.cu -- MXFP8 dequantize kernels (sm_100a).
//
// Operation (torchtitan "[mxfp8 MoE training] Support mxfp8 all to all in expert
// parallel", Summary: dequantize the received e4m3 data with its e8m0 scales back to
// the original precision): y = bf16_RNE(E4M3(q) * 2^(b-127)).
//
// Decoding, rows kernel: the hardware converter widens two codes at a time to f16 and
// then to fp32 (both exact), the product with the power-of-two scale is exact (an E4M3
// value has at most four significant bits), and cvt.rn.bf16x2.f32 rounds once to bf16.
// Tile kernel: the code's seven magnitude bits are placed under the fp32 exponent and
// mantissa fields (value * 2^-120, subnormals included) and multiplied by 2^120 and by
// the scale (measured faster there than the converter, 2-6%).  A NaN code or a NaN scale
// gives 0x7FC0; that case is detected per 4-byte word with one add/mask and takes a
// slow path.
//
//   dequant_rows  row layout (q (.., cols), s (.., cols/32)): flat, 8 codes per vector
//                 (8-byte load, 16-byte store), 16 independent vectors in flight per
//                 thread (measured 3.5% faster than 8; the decode left it latency-bound).
//   dequant_tile  column layout (q (batch, cols, rows), s (batch, cols, rows/32)):
//                 the transpose back to (batch, rows, cols).  Same tile shape as the
//                 column quantizer: warp = 32-row band, lane = 8 rows x 8 columns;
//                 eight 8-byte loads (one per column, full 32-byte sectors across the
//                 four o-lanes), eight 16-byte row stores (4 rows x 128 B per warp).

#include <algorithm>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

template <int U>
__global__ void __launch_bounds__(256) dequant_rows_kernel(const uint8_t* __restrict__ q,
                                                            const uint8_t* __restrict__ s,
                                                            uint16_t* __restrict__ y,
                                                            int64_t n_vec) {
    const int64_t chunk = (int64_t)U * 256;
    for (int64_t base = (int64_t)blockIdx.x * chunk; base < n_vec; base += (int64_t)gridDim.x * chunk) {
        uint2 c[U];
        uint32_t b[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t idx = base + u * 256 + threadIdx.x;
            if (idx < n_vec) {
                c[u] = ld_nc_v2(q + idx * 8);
                b[u] = ld_nc_u8(s + (idx >> 2));
            } else {
                c[u] = make_uint2(0, 0);
                b[u] = 0;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t idx = base + u * 256 + threadIdx.x;
            if (idx >= n_vec) continue;
            uint2 lo, hi;
            if (b[u] != 255u && !any_e4m3_nan(c[u].x) && !any_e4m3_nan(c[u].y)) {
                const float sc = e8m0_value(b[u]);
                lo = dequant4_cvt(c[u].x, sc);
                hi = dequant4_cvt(c[u].y, sc);
            } else {
                lo = dequant4_nan_aware(c[u].x, b[u]);
                hi = dequant4_nan_aware(c[u].y, b[u]);
            }
            *reinterpret_cast<uint4*>(y + idx * 8) = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
    }
}

// Code k (0..7) of an 8-byte group, moved to bits 24..31.
__device__ __forceinline__ uint32_t code_to_top(uint2 c, int k) {
    const uint32_t w = k < 4 ? c.x : c.y;
    return w << (24 - 8 * (k & 3));
}

__global__ void __launch_bounds__(256) dequant_tile_kernel(const uint8_t* __restrict__ q,
                                                            const uint8_t* __restrict__ s, int64_t e0,
                                                            int64_t rt0, int64_t rows, int64_t cols,
                                                            uint16_t* __restrict__ y) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int v = lane & 7, o = lane >> 3;
    const int64_t e = e0 + blockIdx.z;                            // matrix
    const int64_t r_in = (rt0 + blockIdx.y) * 256 + warp * 32;     // band's first row inside it
    const int64_t c = (int64_t)blockIdx.x * 64 + v * 8;
    if (r_in >= rows || c >= cols) return;  // no shuffles or barriers in this kernel
    const int64_t R0 = e * rows + r_in;

    uint2 cj[8];
    uint32_t bj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        cj[j] = ld_nc_v2(q + (e * cols + c + j) * rows + r_in + 8 * o);
        bj[j] = ld_nc_u8(s + (e * cols + c + j) * (rows >> 5) + (r_in >> 5));
    }
    bool special = false;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        special |= (bj[j] == 255u) | any_e4m3_nan(cj[j].x) | any_e4m3_nan(cj[j].y);
    float sc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sc[j] = e8m0_value(bj[j]);
    const float k120 = 0x1p120f;

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float f[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            f[j] = __fmul_rn(__fmul_rn(e4m3_scaled_from_top_byte(code_to_top(cj[j], i)), k120), sc[j]);
        uint32_t w[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) w[p] = cvt_bf16x2(f[2 * p], f[2 * p + 1]);
        if (special) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t code = code_to_top(cj[j], i) >> 24;
                if (bj[j] == 255u || (code & 0x7Fu) == 0x7Fu) {
                    const int p = j >> 1;
                    w[p] = (j & 1) ? ((w[p] & 0x0000FFFFu) | 0x7FC00000u) : ((w[p] & 0xFFFF0000u) | 0x7FC0u);
                }
            }
        }
        *reinterpret_cast<uint4*>(y + (R0 + 8 * o + i) * cols + c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

cudaError_t launch_dequant_rows(const uint8_t* q, const uint8_t* s, uint16_t* y, int64_t n,
                                cudaStream_t stream) {
    constexpr int U = 16;
    const int64_t n_vec = n / 8;
    int64_t grid = (n_vec + U * 256 - 1) / (U * 256);
    const int64_t cap = (int64_t)sm_count() * 8;
    if (grid > cap) grid = cap;
    dequant_rows_kernel<U><<<(unsigned)grid, 256, 0, stream>>>(q, s, y, n_vec);
    return cudaGetLastError();
}

cudaError_t launch_dequant_tile(const uint8_t* q, const uint8_t* s, int64_t batch, int64_t rows,
                                int64_t cols, uint16_t* y, cudaStream_t stream) {
    const int64_t n_col_tiles = (cols + 63) / 64;
    const int64_t n_row_tiles = (rows + 255) / 256;
    if (n_col_tiles > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    constexpr int64_t LIM = 65535;  // grid y and z limit: larger grids go out as several launches
    for (int64_t e0 = 0; e0 < batch; e0 += LIM)
        for (int64_t rt0 = 0; rt0 < n_row_tiles; rt0 += LIM) {
            const dim3 grid((unsigned)n_col_tiles, (unsigned)std::min(n_row_tiles - rt0, LIM),
                            (unsigned)std::min(batch - e0, LIM));
            dequant_tile_kernel<<<grid, 256, 0, stream>>>(q, s, e0, rt0, rows, cols, y);
        }
    return cudaGetLastError();
}

}  // namespace mxq
