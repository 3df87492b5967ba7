// mx_quant.cu -- MXFP8 quantize kernels (sm_100a).
//
// Operation (torchtitan "[mxfp8 MoE training] Support mxfp8 all to all in expert
// parallel", Summary: quantize the all-to-all payload to mxfp8 = e4m3 data + e8m0
// scales): every 32-element block gets b = max(E(amax) - 8, 0) (E = biased bf16
// exponent of the block's max magnitude, i.e. floor(log2 amax) - 8 + 127) and every
// element becomes satRNE_E4M3(x * 2^(127-b)).  The multiply by a power of two is
// exact in fp32, so the only rounding is the hardware convert's.
//
// Two kernels:
//   quant_rows  1x32 blocks.  In memory the blocks of a row-major (.., cols) tensor
//               with cols % 32 == 0 are simply consecutive 64-byte runs, and their
//               scale bytes are consecutive too, so the kernel treats the tensor as
//               one flat array of blocks: four lanes per block, 16-byte loads,
//               512 contiguous bytes per warp load, 256 per warp store.  Each warp
//               prefetches its next loop step into L2.
//   quant_tile  32x1 blocks (and, in dual mode, 1x32 blocks from the same read).
//               A CTA owns 256 rows x 64 columns; warp w owns one 32-row block band;
//               lane (o = lane/8, v = lane%8) holds rows 8o..8o+7 x columns 8v..8v+7
//               (eight 16-byte loads straight into registers, each warp load = 4 rows
//               x 128 B; several resident CTAs per SM hide the latency).
//               Column maxima are reduced in registers and over the four o-lanes
//               with two shuffles; the eight codes of one column and eight rows
//               are packed into one 8-byte store, so the transposed codes go out in
//               full 32-byte sectors; the column scales are staged in shared memory
//               and leave as one 8-byte run per column and tile.  Grid (column tile,
//               row tile, matrix); each CTA prefetches into L2 the tile of the CTA half
//               a wave later; a warp whose band is all finite skips the per-block NaN
//               checks.

#include <algorithm>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

// ---------------------------------------------------------------------------------------
// 1x32 blocks, flat.  Each warp iteration covers 8*U consecutive blocks; lane l loads
// part (l%4) of block (u*8 + l/4) for u in [0, U).
// ---------------------------------------------------------------------------------------
template <int U>
__global__ void __launch_bounds__(256) quant_rows_kernel(const uint16_t* __restrict__ x,
                                                          uint8_t* __restrict__ q,
                                                          uint8_t* __restrict__ s,
                                                          int64_t n_blocks) {
    static_assert(U >= 1 && U <= 4, "one scale byte per lane: at most 32 blocks per warp step");
    const int lane = threadIdx.x & 31;
    const int part = lane & 3, sub = lane >> 2;
    const int64_t warps_per_cta = blockDim.x >> 5;
    const int64_t gwarp = (int64_t)blockIdx.x * warps_per_cta + (threadIdx.x >> 5);
    const int64_t n_warps = (int64_t)gridDim.x * warps_per_cta;

    for (int64_t base = gwarp * (8 * U); base < n_blocks; base += n_warps * (8 * U)) {
        {   // L2 prefetch of this warp's next step: 8U blocks of 64 bytes, a line per lane
            const int64_t nb = base + n_warps * (8 * U) + 2 * lane;
            if (lane < 4 * U && nb < n_blocks) prefetch_l2(x + nb * 32);
        }
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t blk = base + u * 8 + sub;
            v[u] = blk < n_blocks ? ld_nc_v4(x + blk * 32 + part * 8) : make_uint4(0, 0, 0, 0);
        }
        uint32_t sb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            uint32_t m = mag2(amax2(amax2(v[u].x, v[u].y), amax2(v[u].z, v[u].w)));
            m = max(m & 0xFFFFu, m >> 16);
            m = max(m, __shfl_xor_sync(FULL_MASK, m, 1));
            m = max(m, __shfl_xor_sync(FULL_MASK, m, 2));
            const uint32_t b = e8m0_of_amax(m);
            sb[u] = b;
            uint2 out;
            if (b != 255u) {
                const float mul = mx_mult(b);
                out.x = quant4(v[u].x, v[u].y, mul);
                out.y = quant4(v[u].z, v[u].w, mul);
            } else {
                out.x = nan4(v[u].x, v[u].y);
                out.y = nan4(v[u].z, v[u].w);
            }
            const int64_t blk = base + u * 8 + sub;
            if (blk < n_blocks) *reinterpret_cast<uint2*>(q + blk * 32 + part * 8) = out;
        }
        // Scale bytes: lane L writes block base + L, which lane 4*(L%8) computed at step L/8.
        uint32_t mine = 0;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t t = __shfl_sync(FULL_MASK, sb[u], (lane & 7) * 4);
            if ((lane >> 3) == u) mine = t;
        }
        if (lane < 8 * U && base + lane < n_blocks) s[base + lane] = (uint8_t)mine;
    }
}

// ---------------------------------------------------------------------------------------
// 32x1 blocks (and, with DO_ROW, 1x32 blocks) of one 32-row band x 64 columns, held by a
// warp in registers: lane (o = lane/8, v = lane%8) holds rows 8o .. 8o+7 of the band x
// columns c .. c+7 (d[i] = row 8o+i).  `cm` are the lane's column maxima over the whole
// band (magnitudes, bf16 bits, two columns per word).  With SPECIAL == false every
// element of the warp's band is finite, so no block can get the NaN scale and the
// per-block checks are left out; SPECIAL == true is the general path.
//  * Column blocks: the eight codes of one column and eight rows go out as one 8-byte
//    store at qc + j * rows.  The scale bytes go to col_stage[col][band] when col_stage
//    is given (the caller writes each column's eight band scales as one 8-byte run),
//    else straight to s_col (sc, column stride rows/32).
//  * Row blocks: maxima of two rows at once (one bf16x2 word, two shuffles over the
//    four lanes of a block); each lane stores 8 codes of a row.  With row_pair the two
//    block scales of a row are stored as one 2-byte word by lane v = 0.
// ---------------------------------------------------------------------------------------
template <bool DO_ROW, bool SPECIAL>
__device__ __forceinline__ void quant_band(const uint4 (&d)[8], const uint32_t (&cm)[4], bool cv, int o, int v,
                                           uint8_t* __restrict__ qc, int64_t rows, uint8_t* col_stage,
                                           uint8_t* __restrict__ sc, int band, uint8_t* __restrict__ qr,
                                           uint8_t* __restrict__ sr, int64_t cols, bool row_pair) {
    if (cv) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int w = j >> 1;
            const uint32_t am = (j & 1) ? (cm[w] >> 16) : (cm[w] & 0xFFFFu);
            const uint32_t b = SPECIAL ? e8m0_of_amax(am) : e8m0_of_finite_amax(am);
            uint32_t wd[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) wd[i] = w == 0 ? d[i].x : w == 1 ? d[i].y : w == 2 ? d[i].z : d[i].w;
            uint2 out;
            if (!SPECIAL || b != 255u) {
                const float mul = mx_mult(b);
                float p[8];
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float a0 = (j & 1) ? bf16_hi(wd[i]) : bf16_lo(wd[i]);
                    const float a1 = (j & 1) ? bf16_hi(wd[i + 1]) : bf16_lo(wd[i + 1]);
                    if (DO_ROW)
                        fmul2(a0, a1, mul, mul, p[i], p[i + 1]);
                    else  // one axis: the scalar form measured faster
                        fmul2s(a0, a1, mul, mul, p[i], p[i + 1]);
                }
                out.x = cvt4_e4m3(p[0], p[1], p[2], p[3]);
                out.y = cvt4_e4m3(p[4], p[5], p[6], p[7]);
            } else {
                uint32_t sg[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) sg[i] = ((j & 1) ? (wd[i] >> 24) : (wd[i] >> 8)) & 0x80u;
                out.x = (sg[0] | (sg[1] << 8) | (sg[2] << 16) | (sg[3] << 24)) | 0x7F7F7F7Fu;
                out.y = (sg[4] | (sg[5] << 8) | (sg[6] << 16) | (sg[7] << 24)) | 0x7F7F7F7Fu;
            }
            *reinterpret_cast<uint2*>(qc + j * rows) = out;
        }
        // column scale bytes: lane o handles columns 2o and 2o+1 of its vector
        const uint32_t m = o == 0 ? cm[0] : o == 1 ? cm[1] : o == 2 ? cm[2] : cm[3];
        const uint32_t m0 = m & 0xFFFFu, m1 = m >> 16;
        const uint8_t b0 = (uint8_t)(SPECIAL ? e8m0_of_amax(m0) : e8m0_of_finite_amax(m0));
        const uint8_t b1 = (uint8_t)(SPECIAL ? e8m0_of_amax(m1) : e8m0_of_finite_amax(m1));
        if (col_stage) {
            col_stage[(8 * v + 2 * o) * 8 + band] = b0;
            col_stage[(8 * v + 2 * o + 1) * 8 + band] = b1;
        } else {
            sc[0] = b0;
            sc[rows >> 5] = b1;
        }
    }

    if (DO_ROW) {
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            // (even-column max, odd-column max) of rows i and i+1, then one word holding
            // both rows' maxima; the shuffles take in the other three lanes of the block
            const uint32_t ra = amax2(amax2(d[i].x, d[i].y), amax2(d[i].z, d[i].w));
            const uint32_t rb = amax2(amax2(d[i + 1].x, d[i + 1].y), amax2(d[i + 1].z, d[i + 1].w));
            uint32_t pm = amax2(__byte_perm(ra, rb, 0x5410), __byte_perm(ra, rb, 0x7632));
            pm = amax2(pm, __shfl_xor_sync(FULL_MASK, pm, 1));
            pm = mag2(amax2(pm, __shfl_xor_sync(FULL_MASK, pm, 2)));
            uint32_t bb[2];
            bb[0] = SPECIAL ? e8m0_of_amax(pm & 0xFFFFu) : e8m0_of_finite_amax(pm & 0xFFFFu);
            bb[1] = SPECIAL ? e8m0_of_amax(pm >> 16) : e8m0_of_finite_amax(pm >> 16);
            const uint32_t nb = __shfl_xor_sync(FULL_MASK, bb[0] | (bb[1] << 16), 4);  // the rows' other blocks
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4& r = d[i + h];
                const uint32_t b = bb[h];
                uint2 out;
                if (!SPECIAL || b != 255u) {
                    const float mul = mx_mult(b);
                    out.x = quant4(r.x, r.y, mul);
                    out.y = quant4(r.z, r.w, mul);
                } else {
                    out.x = nan4(r.x, r.y);
                    out.y = nan4(r.z, r.w);
                }
                if (cv) {
                    *reinterpret_cast<uint2*>(qr + (i + h) * cols) = out;
                    uint8_t* srow = sr + (i + h) * (cols >> 5);
                    if (row_pair) {
                        if (v == 0) *reinterpret_cast<uint16_t*>(srow) = (uint16_t)(b | (((nb >> (16 * h)) & 0xFFu) << 8));
                    } else if ((v & 3) == 0) {
                        *srow = (uint8_t)b;
                    }
                }
            }
        }
    }
}

// One 256 x 64 tile of one matrix per CTA (warp w = band w), loaded straight into
// registers: eight 16-byte loads per lane, a warp load = 4 rows x 128 B, several CTAs
// per SM hiding the latency.  Grid (column tiles, row tiles, matrices) from the row tile
// rt0 and matrix e0 on (the host splits grids beyond the y/z limits into several
// launches), so no CTA divides its index.  With
// rows % 256 == 0 the column scales of a tile are staged in shared memory: each column's
// eight band scales leave as one 8-byte store instead of eight byte stores.  Dual mode
// keeps up to 85 registers (three CTAs per SM) so that nothing spills; the column axis
// alone fits 64 (four CTAs per SM).
template <bool DO_ROW>
__global__ void __launch_bounds__(256, DO_ROW ? 3 : 4) quant_tile_kernel(
    const uint16_t* __restrict__ x, int64_t e0, int64_t rt0, int64_t rows, int64_t cols,
    uint8_t* __restrict__ q_row, uint8_t* __restrict__ s_row, uint8_t* __restrict__ q_col,
    uint8_t* __restrict__ s_col, bool row_pair, bool stage, uint32_t pf_dx, uint32_t pf_dy) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int v = lane & 7, o = lane >> 3;
    const int64_t ct = blockIdx.x;
    const int64_t c = ct * 64 + v * 8;  // first column of this lane's vector
    const bool cv = c < cols;           // cols % 32 == 0: whole vector in or out
    __shared__ __align__(8) uint8_t col_sc[64 * 8];
    const int64_t e = e0 + blockIdx.z;     // matrix
    const int64_t rt = rt0 + blockIdx.y;   // row tile inside it
    const int64_t r_in = rt * 256 + warp * 32;  // band's first row inside matrix e
    if (pf_dx | pf_dy) {
        // L2 prefetch of the tile pf_dy * gridDim.x + pf_dx CTAs further on in launch
        // order (part of a wave: a CTA that will start soon), one 128-byte row per thread;
        // the target's block index by carries, without a division in the common case
        uint32_t tx = blockIdx.x + pf_dx, ty = blockIdx.y + pf_dy, tz = blockIdx.z;
        if (tx >= gridDim.x) {
            tx -= gridDim.x;
            ++ty;
        }
        if (ty >= gridDim.y) {
            tz += ty / gridDim.y;
            ty %= gridDim.y;
        }
        const int64_t prow = (rt0 + ty) * 256 + threadIdx.x, pc = (int64_t)tx * 64;
        if (tz < gridDim.z && prow < rows && pc < cols) prefetch_l2(x + ((e0 + tz) * rows + prow) * cols + pc);
    }
    if (r_in < rows) {                          // the same for the whole warp
        const int64_t R0 = e * rows + r_in;
        uint4 d[8];
        const uint16_t* src = x + (R0 + 8 * o) * cols + c;
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = cv ? ld_nc_v4(src + i * cols) : make_uint4(0, 0, 0, 0);
        // column maxima over the band: the lane's 8 rows, then the four o-lanes
        uint32_t cm[4];
        cm[0] = amax2(d[0].x, d[1].x); cm[1] = amax2(d[0].y, d[1].y);
        cm[2] = amax2(d[0].z, d[1].z); cm[3] = amax2(d[0].w, d[1].w);
#pragma unroll
        for (int i = 2; i < 8; ++i) {
            cm[0] = amax2(cm[0], d[i].x);
            cm[1] = amax2(cm[1], d[i].y);
            cm[2] = amax2(cm[2], d[i].z);
            cm[3] = amax2(cm[3], d[i].w);
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            cm[w] = amax2(cm[w], __shfl_xor_sync(FULL_MASK, cm[w], 8));
            cm[w] = mag2(amax2(cm[w], __shfl_xor_sync(FULL_MASK, cm[w], 16)));
        }
        // a half at or above 0x7F80 is an Inf or NaN in that column: adding 0x80
        // to each (magnitude) half sets its top bit exactly then, with no carry
        // between the halves
        const uint32_t k80 = 0x00800080u;
        const bool finite =
            (((cm[0] + k80) | (cm[1] + k80) | (cm[2] + k80) | (cm[3] + k80)) & 0x80008000u) == 0u;
        const bool all_finite = __all_sync(FULL_MASK, finite);
        uint8_t* qc = q_col + (e * cols + c) * rows + r_in + 8 * o;
        uint8_t* sc = s_col + (e * cols + c + 2 * o) * (rows >> 5) + (r_in >> 5);
        uint8_t* qr = DO_ROW ? q_row + (R0 + 8 * o) * cols + c : nullptr;
        uint8_t* sr = DO_ROW ? s_row + (R0 + 8 * o) * (cols >> 5) + (c >> 5) : nullptr;
        uint8_t* stg = stage ? col_sc : nullptr;
        if (all_finite)
            quant_band<DO_ROW, false>(d, cm, cv, o, v, qc, rows, stg, sc, warp, qr, sr, cols, row_pair);
        else
            quant_band<DO_ROW, true>(d, cm, cv, o, v, qc, rows, stg, sc, warp, qr, sr, cols, row_pair);
    }
    if (stage) {
        __syncthreads();
        const int tid = threadIdx.x;
        const int64_t col = ct * 64 + tid;
        if (tid < 64 && col < cols)
            *reinterpret_cast<uint2*>(s_col + (e * cols + col) * (rows >> 5) + rt * 8) =
                *reinterpret_cast<const uint2*>(col_sc + tid * 8);
    }
}

// ---------------------------------------------------------------------------------------
// fp32 -> E4M3 with the same convert, four values per thread.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) encode_f32_kernel(const float* __restrict__ x,
                                                          uint8_t* __restrict__ q, int64_t n) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i * 4 < n; i += stride) {
        if (i * 4 + 4 <= n) {
            const uint4 w = ld_nc_v4(x + i * 4);
            const uint32_t r = cvt_e4m3x2(__uint_as_float(w.x), __uint_as_float(w.y)) |
                               (cvt_e4m3x2(__uint_as_float(w.z), __uint_as_float(w.w)) << 16);
            *reinterpret_cast<uint32_t*>(q + i * 4) = r;
        } else {
            for (int64_t k = i * 4; k < n; ++k) q[k] = (uint8_t)(cvt_e4m3x2(x[k], 0.0f) & 0xFFu);
        }
    }
}

// ---- launchers ---------------------------------------------------------------------------

constexpr double QT_PF_WAVES = 0.5;  // prefetch distance of the tile kernel, in waves of CTAs (swept: 0.5..2)

cudaError_t launch_quant_rows(const uint16_t* x, uint8_t* q, uint8_t* s, int64_t n_blocks,
                              cudaStream_t stream) {
    constexpr int U = 4;
    const int64_t per_cta = 8 * U * 8;  // 8 warps x 32 blocks
    int64_t grid = (n_blocks + per_cta - 1) / per_cta;
    const int64_t cap = (int64_t)sm_count() * 8;  // grid-stride beyond 8 CTAs per SM
    if (grid > cap) grid = cap;
    quant_rows_kernel<U><<<(unsigned)grid, 256, 0, stream>>>(x, q, s, n_blocks);
    return cudaGetLastError();
}

cudaError_t launch_quant_tile(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols,
                              bool do_row, bool do_col, uint8_t* q_row, uint8_t* s_row,
                              uint8_t* q_col, uint8_t* s_col, cudaStream_t stream) {
    if (!do_col) return cudaErrorInvalidValue;  // 1x32 blocks alone take launch_quant_rows
    const int64_t n_col_tiles = (cols + 63) / 64;
    const int64_t n_row_tiles = (rows + 255) / 256;
    if (n_col_tiles > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    // a row's two block scales of a tile as one 2-byte store: an even number of blocks
    // per row and a 2-byte-aligned s_row
    const bool row_pair = (cols % 64) == 0 && (reinterpret_cast<uintptr_t>(s_row) & 1) == 0;
    // the column scales of a tile staged in shared memory: eight whole bands per tile and
    // 8-byte-aligned runs
    const bool stage = (rows % 256) == 0 && (reinterpret_cast<uintptr_t>(s_col) & 7) == 0;
    // each CTA prefetches into L2 the tile of the CTA QT_PF_WAVES waves (of all resident
    // CTAs) later: pf_ahead = pf_dy * grid.x + pf_dx
    const uint32_t pf_ahead = (uint32_t)(QT_PF_WAVES * sm_count() * (do_row ? 3 : 4));
    constexpr int64_t LIM = 65535;  // grid y and z limit
    for (int64_t e0 = 0; e0 < batch; e0 += LIM)
        for (int64_t rt0 = 0; rt0 < n_row_tiles; rt0 += LIM) {
            const dim3 grid((unsigned)n_col_tiles, (unsigned)std::min(n_row_tiles - rt0, LIM),
                            (unsigned)std::min(batch - e0, LIM));
            const uint32_t pf_dx = pf_ahead % grid.x, pf_dy = pf_ahead / grid.x;
            if (do_row)
                quant_tile_kernel<true><<<grid, 256, 0, stream>>>(x, e0, rt0, rows, cols, q_row, s_row, q_col, s_col,
                                                                  row_pair, stage, pf_dx, pf_dy);
            else
                quant_tile_kernel<false><<<grid, 256, 0, stream>>>(x, e0, rt0, rows, cols, q_row, s_row, q_col, s_col,
                                                                   row_pair, stage, pf_dx, pf_dy);
        }
    return cudaGetLastError();
}

cudaError_t launch_encode_f32(const float* x, uint8_t* q, int64_t n, cudaStream_t stream) {
    const int64_t n4 = (n + 3) / 4;
    int64_t grid = (n4 + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (grid > cap) grid = cap;
    encode_f32_kernel<<<(unsigned)grid, 256, 0, stream>>>(x, q, n);
    return cudaGetLastError();
}

}  // namespace mxq
