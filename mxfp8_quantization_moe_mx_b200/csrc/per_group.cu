// per_group.cu -- per-group rowwise FP8 scaling kernels (sm_100a).
//
// Operation (torchao "[moe training] fix uncoalesced global accesses in per group
// rowwise scaling kernel", Summary and Performance): a bf16 (M, K) tensor of expert
// tokens, split into G contiguous row groups by int32 end offsets; for every
// (group g, feature k): amax over the group's rows, fp32 scale s = 448 / max(amax,
// fp32(1e-12)) (IEEE divide), and E4M3 codes q = satRNE_E4M3(fp32(x * s)), written
// row-major (M, K) -- the left operand of the scaled grouped GEMM -- or column-major.
//
// The page's Triton kernel lost its time in uncoalesced row-major stores.  Here both
// layouts store full 32-byte sectors.  The hard part is the dependency: a group's
// whole column must be reduced before any of its bytes is written.  Every CTA owns
// whole (group, column-slab) tiles, so no CTA ever waits for another, and no tile is
// read from DRAM twice:
//
//  * Small groups (the host's choice from the average group size): one CTA per
//    (group, 64-column slab), one thread per row of the group -- thread (o = tid/8,
//    v = tid%8) holds octet o (rows 8o..8o+7) x columns 8v..8v+7 in registers, loaded
//    with eight 16-byte loads issued at once (a warp load = 4 rows x 128 B).  Maxima,
//    scales and codes come from those registers.  Rows of an unusually large group
//    beyond the CTA size are streamed twice.
//  * Large groups: one CTA per (group, 32-column slab) tile, 128..512 threads.  Pass 1
//    streams the tile (thread (o = tid/4, v = tid%4): octet o of each round x columns
//    8v..8v+7, eight 16-byte loads in flight per thread) for the column maxima; pass 2
//    streams it again for the conversion.  Pass-1 loads carry an L2 evict_last policy
//    and pass-2 loads and code stores evict_first, so a tile stays in L2 until its
//    second read and is released by it; the host picks the CTA size (4, 2 or 1 CTAs
//    per SM) from the resident-tile budget.  DRAM then sees each byte of x about once.
//    Tiles are launched slab-fastest, so the tiles running side by side cover whole
//    rows of one group.
//  * Reductions use packed bf16 magnitude maxima, warp shuffles and shared memory.
//    Row-major output: each lane writes 8 codes of one row.  Column-major output: each
//    lane packs the 8 rows of one column into one 8-byte store; octets cut by a group
//    boundary fall back to byte stores.
//  * Group bounds come straight from the device offsets without a host sync: the
//    clamp rule end_g = min(max(offs[g], end_{g-1}), M) equals min(M, max(0,
//    offs[0..g])), a running maximum each CTA reduces itself.  Empty groups still
//    write their scales.

#include <algorithm>
#include <cmath>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int PG_SMALL_COLS = 64;
constexpr int PG_SMALL_MAX_THREADS = 512;
constexpr int PG_BIG_COLS = 32;
constexpr int PG_BIG_THREADS = 512;
// Bytes of (estimated) large-group tiles allowed to be resident at once; chosen by a
// sweep over 40, 80, 160 and 320 MB on the (16640 | 65536, 5120) shapes.
constexpr double PG_RESIDENT_BUDGET = 160e6;

// Rows [start, end) of a group.
struct GroupRows {
    int64_t start, end;
};

// Group bounds from the device offsets: a block-wide maximum of offs[0..g-1].
__device__ __forceinline__ GroupRows group_rows(const int32_t* __restrict__ offs, int g, int64_t M,
                                                int* red_scratch) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, n_warps = blockDim.x >> 5;
    int pm = 0;
    for (int i = tid; i < g; i += blockDim.x) pm = max(pm, offs[i]);
#pragma unroll
    for (int sh = 16; sh; sh >>= 1) pm = max(pm, __shfl_xor_sync(FULL_MASK, pm, sh));
    if (lane == 0) red_scratch[warp] = pm;
    __syncthreads();
    pm = 0;
    for (int w = 0; w < n_warps; ++w) pm = max(pm, red_scratch[w]);
    GroupRows gr;
    gr.start = min((int64_t)pm, M);
    gr.end = min((int64_t)max(pm, offs[g]), M);
    return gr;
}

// Rows r0 + i (i in [lo, hi)) of an octet that belong to the group.
__device__ __forceinline__ void clip_octet(int64_t r0, const GroupRows& gr, int* lo, int* hi) {
    *lo = (int)max((int64_t)0, min((int64_t)8, gr.start - r0));
    *hi = (int)max((int64_t)0, min((int64_t)8, gr.end - r0));
}

// HINT: loads carry the L2 policy `pol`.
template <bool HINT = false>
__device__ __forceinline__ void load_octet(uint4 (&d)[8], const uint16_t* __restrict__ x, int64_t r0,
                                           int lo, int hi, int64_t K, int64_t c, uint64_t pol = 0) {
    const uint16_t* src = x + r0 * K + c;
#pragma unroll
    for (int i = 0; i < 8; ++i, src += K)
        d[i] = (i >= lo && i < hi) ? (HINT ? ld_nc_v4_hint(src, pol) : ld_nc_v4(src)) : make_uint4(0, 0, 0, 0);
}

__device__ __forceinline__ void amax_octet(const uint4 (&d)[8], uint32_t (&cm)[4]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        cm[0] = amax2(cm[0], d[i].x);
        cm[1] = amax2(cm[1], d[i].y);
        cm[2] = amax2(cm[2], d[i].z);
        cm[3] = amax2(cm[3], d[i].w);
    }
}

__device__ __forceinline__ uint32_t word_of(const uint4& a, int w) {
    return w == 0 ? a.x : w == 1 ? a.y : w == 2 ? a.z : a.w;
}

// Scale of a column from the bit pattern of its amax: 448 / max(amax, fp32(1e-12)),
// IEEE divide; a column holding Inf/NaN gets a NaN scale.
__device__ __forceinline__ float group_scale(uint32_t amax_bits) {
    return amax_bits >= 0x7F80u ? __uint_as_float(0x7FC00000u)
                                : __fdiv_rn(448.0f, fmaxf(__uint_as_float(amax_bits << 16), 1e-12f));
}

// Convert the rows [lo, hi) of one octet x this lane's 8 columns (scales f) and store;
// with HINT the 8-byte stores carry the L2 policy `pol`.
template <bool COL_MAJOR, bool HINT = false>
__device__ __forceinline__ void store_octet(const uint4 (&d)[8], const float (&f)[8],
                                            uint8_t* __restrict__ q, int64_t r0, int lo, int hi,
                                            int64_t M, int64_t K, int64_t c, bool vec_col_store,
                                            uint64_t pol = 0) {
    if (!COL_MAJOR) {
        uint8_t* dst = q + r0 * K + c;
        const bool full = lo == 0 && hi == 8;
#pragma unroll
        for (int i = 0; i < 8; ++i, dst += K) {
            if (!full && (i < lo || i >= hi)) continue;
            float p[8];
            fmul2(bf16_lo(d[i].x), bf16_hi(d[i].x), f[0], f[1], p[0], p[1]);
            fmul2(bf16_lo(d[i].y), bf16_hi(d[i].y), f[2], f[3], p[2], p[3]);
            fmul2(bf16_lo(d[i].z), bf16_hi(d[i].z), f[4], f[5], p[4], p[5]);
            fmul2(bf16_lo(d[i].w), bf16_hi(d[i].w), f[6], f[7], p[6], p[7]);
            uint2 out;
            out.x = cvt4_e4m3(p[0], p[1], p[2], p[3]);
            out.y = cvt4_e4m3(p[4], p[5], p[6], p[7]);
            if (HINT)
                st_v2_hint(dst, out, pol);
            else
                *reinterpret_cast<uint2*>(dst) = out;
        }
    } else {
        const bool full = vec_col_store && lo == 0 && hi == 8;
        uint8_t* dst = q + c * M + r0;
#pragma unroll
        for (int j = 0; j < 8; ++j, dst += M) {
            float p[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const uint32_t w0 = word_of(d[i], j >> 1), w1 = word_of(d[i + 1], j >> 1);
                fmul2((j & 1) ? bf16_hi(w0) : bf16_lo(w0), (j & 1) ? bf16_hi(w1) : bf16_lo(w1), f[j], f[j],
                      p[i], p[i + 1]);
            }
            uint2 out;
            out.x = cvt4_e4m3(p[0], p[1], p[2], p[3]);
            out.y = cvt4_e4m3(p[4], p[5], p[6], p[7]);
            if (full) {
                if (HINT)
                    st_v2_hint(dst, out, pol);
                else
                    *reinterpret_cast<uint2*>(dst) = out;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i >= lo && i < hi) dst[i] = (uint8_t)(((i < 4 ? out.x : out.y) >> (8 * (i & 3))) & 0xFFu);
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Small groups: grid (n_slabs64, G), blockDim = the group size rounded up (<= 512).
// ---------------------------------------------------------------------------------------
template <bool COL_MAJOR>
__global__ void __launch_bounds__(PG_SMALL_MAX_THREADS) per_group_small_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, const int32_t* __restrict__ offs,
    uint8_t* __restrict__ q, float* __restrict__ scales, bool vec_col_store) {
    __shared__ uint32_t red[PG_SMALL_MAX_THREADS / 32][32];
    __shared__ float sc[PG_SMALL_COLS];
    __shared__ int scratch[PG_SMALL_MAX_THREADS / 32];

    const int T = blockDim.x, n_warps = T >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid & 7, o = tid >> 3, oct_per_cta = T >> 3;
    const int g = blockIdx.y;
    const int64_t k0 = (int64_t)blockIdx.x * PG_SMALL_COLS;
    const int64_t c = k0 + 8 * v;
    const bool cv = c < K;
    const GroupRows gr = group_rows(offs, g, M, scratch);
    const int64_t ob = gr.start >> 3;
    const int64_t oe = gr.end > gr.start ? (gr.end + 7) >> 3 : ob;

    // the resident octet: all eight row loads in flight at once
    const int64_t oct = ob + o;
    const bool have = cv && oct < oe;
    int lo = 0, hi = 0;
    if (have) clip_octet(oct * 8, gr, &lo, &hi);
    uint4 d[8];
    load_octet(d, x, oct * 8, lo, hi, K, c);  // lo == hi == 0 loads nothing
    uint32_t cm[4] = {0, 0, 0, 0};
    amax_octet(d, cm);
    if (cv) {  // rows beyond the CTA, one at a time (the resident octet stays live in d)
        for (int64_t ox = ob + oct_per_cta + o; ox < oe; ox += oct_per_cta) {
            int l2, h2;
            clip_octet(ox * 8, gr, &l2, &h2);
            const uint16_t* src = x + ox * 8 * K + c;
            for (int i = l2; i < h2; ++i) {
                const uint4 e = ld_nc_v4(src + i * K);
                cm[0] = amax2(cm[0], e.x);
                cm[1] = amax2(cm[1], e.y);
                cm[2] = amax2(cm[2], e.z);
                cm[3] = amax2(cm[3], e.w);
            }
        }
    }
    // reduce: lanes of a column (xor 8, 16), then warps
#pragma unroll
    for (int sh = 8; sh <= 16; sh <<= 1)
#pragma unroll
        for (int w = 0; w < 4; ++w) cm[w] = amax2(cm[w], __shfl_xor_sync(FULL_MASK, cm[w], sh));
    if (lane < 8)
#pragma unroll
        for (int w = 0; w < 4; ++w) red[warp][lane * 4 + w] = cm[w];
    __syncthreads();
    if (tid < 32) {
        uint32_t m = 0;
        for (int w = 0; w < n_warps; ++w) m = amax2(m, red[w][tid]);
        m = mag2(m);
        // word tid = columns 8*(tid/4) + 2*(tid%4) + {0, 1} of the slab
        const int col0 = 8 * (tid >> 2) + 2 * (tid & 3);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float s = group_scale(h ? (m >> 16) : (m & 0xFFFFu));
            sc[col0 + h] = s;
            if (k0 + col0 + h < K) scales[(int64_t)g * K + k0 + col0 + h] = s;
        }
    }
    __syncthreads();
    if (cv) {
        float f[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = sc[8 * v + j];
        if (have) store_octet<COL_MAJOR>(d, f, q, oct * 8, lo, hi, M, K, c, vec_col_store);
        for (int64_t ox = ob + oct_per_cta + o; ox < oe; ox += oct_per_cta) {
            int l2, h2;
            clip_octet(ox * 8, gr, &l2, &h2);
            load_octet(d, x, ox * 8, l2, h2, K, c);
            store_octet<COL_MAJOR>(d, f, q, ox * 8, l2, h2, M, K, c, vec_col_store);
        }
    }
}

// ---------------------------------------------------------------------------------------
// Large groups: grid (n_slabs32, G), 512 threads, two streaming passes over the tile.
// ---------------------------------------------------------------------------------------
template <bool COL_MAJOR>
__global__ void __launch_bounds__(PG_BIG_THREADS, 1) per_group_big_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, const int32_t* __restrict__ offs,
    uint8_t* __restrict__ q, float* __restrict__ scales, bool vec_col_store) {
    __shared__ uint32_t red[PG_BIG_THREADS / 32][16];
    __shared__ float sc[PG_BIG_COLS];
    __shared__ int scratch[PG_BIG_THREADS / 32];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, n_warps = blockDim.x >> 5;
    const int v = tid & 3, o = tid >> 2;
    const int OCTS = blockDim.x >> 2;  // octets per round
    const int g = blockIdx.y;
    const int64_t k0 = (int64_t)blockIdx.x * PG_BIG_COLS;
    const int64_t c = k0 + 8 * v;
    const bool cv = c < K;
    const GroupRows gr = group_rows(offs, g, M, scratch);
    const int64_t ob = gr.start >> 3;
    const int64_t oe = gr.end > gr.start ? (gr.end + 7) >> 3 : ob;

    const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();

    // ---- pass 1: column maxima (the tile's lines are kept in L2 for pass 2)
    uint32_t cm[4] = {0, 0, 0, 0};
    uint4 d[8];
    if (cv) {
        for (int64_t oc = ob + o; oc < oe; oc += OCTS) {
            int lo, hi;
            clip_octet(oc * 8, gr, &lo, &hi);
            load_octet<true>(d, x, oc * 8, lo, hi, K, c, keep);
            amax_octet(d, cm);
        }
    }
    // lanes of a column: same v, o within the warp = lane / 4 (xor 4, 8, 16)
#pragma unroll
    for (int sh = 4; sh <= 16; sh <<= 1)
#pragma unroll
        for (int w = 0; w < 4; ++w) cm[w] = amax2(cm[w], __shfl_xor_sync(FULL_MASK, cm[w], sh));
    if (lane < 4)
#pragma unroll
        for (int w = 0; w < 4; ++w) red[warp][lane * 4 + w] = cm[w];
    __syncthreads();
    if (tid < 16) {
        uint32_t m = 0;
        for (int w = 0; w < n_warps; ++w) m = amax2(m, red[w][tid]);
        m = mag2(m);
        // word tid = columns 8*(tid/4) + 2*(tid%4) + {0, 1} of the slab
        const int col0 = 8 * (tid >> 2) + 2 * (tid & 3);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float s = group_scale(h ? (m >> 16) : (m & 0xFFFFu));
            sc[col0 + h] = s;
            if (k0 + col0 + h < K) scales[(int64_t)g * K + k0 + col0 + h] = s;
        }
    }
    __syncthreads();

    // ---- pass 2: the tile again (from L2, releasing its lines) -> E4M3
    if (cv) {
        float f[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = sc[8 * v + j];
        for (int64_t oc = ob + o; oc < oe; oc += OCTS) {
            int lo, hi;
            clip_octet(oc * 8, gr, &lo, &hi);
            load_octet<true>(d, x, oc * 8, lo, hi, K, c, drop);
            store_octet<COL_MAJOR, true>(d, f, q, oc * 8, lo, hi, M, K, c, vec_col_store, drop);
        }
    }
}

// ---- host side ---------------------------------------------------------------------------

// The small-group kernel while the average group (with 30% headroom for multinomial
// spread) fits one CTA of at most 512 threads; the streaming kernel beyond that, with
// 512, 256 or 128 threads per CTA (one, two or four CTAs per SM at up to 128
// registers): the most CTAs per SM whose resident tiles -- each one's second pass
// must still find it in L2 -- fit the budget, tiles estimated from the average group
// plus 15%.
cudaError_t launch_per_group(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, bool col_major, uint8_t* q, float* scales,
                             cudaStream_t stream) {
    if (K == 0 || G == 0) return cudaSuccess;
    const bool vec_col_store = (M % 8) == 0;
    const double want = std::max(1.0, (double)((M + G - 1) / G) * 1.3);
    if (want <= (double)PG_SMALL_MAX_THREADS) {
        const int threads = std::max(32, (int)std::ceil(want / 32.0) * 32);
        const dim3 grid((unsigned)((K + PG_SMALL_COLS - 1) / PG_SMALL_COLS), (unsigned)G);
        if (col_major)
            per_group_small_kernel<true><<<grid, threads, 0, stream>>>(x, M, K, offs, q, scales, vec_col_store);
        else
            per_group_small_kernel<false><<<grid, threads, 0, stream>>>(x, M, K, offs, q, scales, vec_col_store);
    } else {
        const double tile_bytes = want / 1.3 * 1.15 * PG_BIG_COLS * 2;
        const double per_sm = PG_RESIDENT_BUDGET / ((double)sm_count() * tile_bytes);
        const int threads = per_sm >= 4.0 ? 128 : per_sm >= 2.0 ? 256 : PG_BIG_THREADS;
        const dim3 grid((unsigned)((K + PG_BIG_COLS - 1) / PG_BIG_COLS), (unsigned)G);
        if (col_major)
            per_group_big_kernel<true><<<grid, threads, 0, stream>>>(x, M, K, offs, q, scales, vec_col_store);
        else
            per_group_big_kernel<false><<<grid, threads, 0, stream>>>(x, M, K, offs, q, scales, vec_col_store);
    }
    return cudaGetLastError();
}

}  // namespace mxq
