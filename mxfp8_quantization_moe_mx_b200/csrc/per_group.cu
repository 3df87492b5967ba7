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
// whole column must be reduced before any of its bytes is written.
//
//  * Tile kernel (groups up to a few thousand rows): a (group, W-column slab) tile,
//    W = 64, 32 or 16, is brought into shared memory by 4 KB TMA boxes completing on
//    an mbarrier, so DRAM reads each byte of x once and the bytes in flight cost no
//    registers.  The column maxima, the scales and the codes all come from shared
//    memory.  A tile too large for one SM is split by rows among a thread-block
//    cluster of 2..8 CTAs.  Each CTA pushes its partial column maxima into every
//    other CTA's shared memory with st.async, completing on that CTA's mbarrier:
//    no cluster-wide fence, one relaxed cluster barrier pair.  Row-major: a lane
//    converts 8 columns of a row and stores 8 bytes.  Column-major: a lane converts
//    an octet of rows x 8 columns into eight 8-byte column words.  With W < 64 it
//    reads the octet's rows in rotated order, which keeps the shared-memory reads
//    conflict-free, then rotates each word back.  Octets are aligned
//    to 32 rows, so a warp's column stores fill whole sectors.  Warp 1 of each CTA
//    prefetches into L2 (evict_last) the tile of the CTA half a wave of resident CTAs
//    later, so that CTA's TMA copies mostly hit L2 (not for 16-column column-major
//    tiles, where it measured slower).
//  * Pair kernel (column-major output, groups of up to about 170 rows): one CTA and one
//    tile per pair of neighbouring groups; the octet holding their boundary is
//    assembled from both groups' codes, so it is stored as whole column words.
//  * Streaming kernel (larger groups): one CTA per (group, 32-column slab) tile,
//    128..512 threads.  Pass 1 streams the tile for the column maxima (thread
//    (o = tid/4, v = tid%4): octet o of each round x columns 8v..8v+7, eight 16-byte
//    loads in flight); pass 2 streams it again for the conversion.  Pass-1 loads
//    carry an L2 evict_last policy, pass-2 loads and code stores evict_first, so a
//    tile stays in L2 until its second read; the host sizes the CTAs from a
//    resident-tile budget.
//  * Reductions use packed bf16 magnitude maxima (max.NaN.xorsign.abs), warp
//    shuffles and shared memory.
//  * Group bounds come straight from the device offsets without a host sync: the
//    clamp rule end_g = min(max(offs[g], end_{g-1}), M) equals min(M, max(0,
//    offs[0..g])), a running maximum each CTA reduces itself.  Empty groups still
//    write their scales.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>

#include "mxq.h"

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int PG_BIG_COLS = 32;
// Rows of a group beyond its shared-memory tile are streamed from global memory; one lane
// per row prefetches the row this many loop steps ahead into L2.
constexpr int PG_OVF_PF_STEPS = 8;
constexpr int PG_BIG_THREADS = 512;
// Bytes of (estimated) large-group tiles allowed to be resident at once; chosen by a
// sweep over 40, 80, 160 and 320 MB on the (16640 | 65536, 5120) shapes.
constexpr double PG_RESIDENT_BUDGET = 160e6;

// Rows [start, end) of a group.
struct GroupRows {
    int64_t start, end;
};

// End offset of group i: from the device offsets, or (rows_per_group > 0) i + 1 whole
// matrices of a batched (3-D) tensor, each matrix one group.
__device__ __forceinline__ int end_offset(const int32_t* __restrict__ offs, int i, int rows_per_group) {
    return rows_per_group > 0 ? (i + 1) * rows_per_group : offs[i];
}

// Group bounds from the device offsets: a block-wide maximum of offs[0..g-1].
__device__ __forceinline__ GroupRows group_rows(const int32_t* __restrict__ offs, int g, int64_t M,
                                                int* red_scratch, int rows_per_group) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, n_warps = blockDim.x >> 5;
    int pm = 0;
    for (int i = tid; i < g; i += blockDim.x) pm = max(pm, end_offset(offs, i, rows_per_group));
#pragma unroll
    for (int sh = 16; sh; sh >>= 1) pm = max(pm, __shfl_xor_sync(FULL_MASK, pm, sh));
    if (lane == 0) red_scratch[warp] = pm;
    __syncthreads();
    pm = 0;
    for (int w = 0; w < n_warps; ++w) pm = max(pm, red_scratch[w]);
    GroupRows gr;
    gr.start = min((int64_t)pm, M);
    gr.end = min((int64_t)max(pm, end_offset(offs, g, rows_per_group)), M);
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

// Codes of column j of an octet: rows 0..7 as bytes 0..7.
__device__ __forceinline__ uint2 octet_column_codes(const uint4 (&d)[8], const float (&f)[8], int j) {
    float p[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const uint32_t w0 = word_of(d[i], j >> 1), w1 = word_of(d[i + 1], j >> 1);
        fmul2((j & 1) ? bf16_hi(w0) : bf16_lo(w0), (j & 1) ? bf16_hi(w1) : bf16_lo(w1), f[j], f[j], p[i],
              p[i + 1]);
    }
    uint2 out;
    out.x = cvt4_e4m3(p[0], p[1], p[2], p[3]);
    out.y = cvt4_e4m3(p[4], p[5], p[6], p[7]);
    return out;
}

// Codes of column j of an octet under the scale fj.
__device__ __forceinline__ uint2 octet_column_codes_s(const uint4 (&d)[8], float fj, int j) {
    float p[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const uint32_t w0 = word_of(d[i], j >> 1), w1 = word_of(d[i + 1], j >> 1);
        fmul2((j & 1) ? bf16_hi(w0) : bf16_lo(w0), (j & 1) ? bf16_hi(w1) : bf16_lo(w1), fj, fj, p[i], p[i + 1]);
    }
    uint2 out;
    out.x = cvt4_e4m3(p[0], p[1], p[2], p[3]);
    out.y = cvt4_e4m3(p[4], p[5], p[6], p[7]);
    return out;
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
            const uint2 out = octet_column_codes(d, f, j);
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
// Small and medium groups: one CTA per (group, W-column slab) tile, the tile brought into
// shared memory by TMA and reduced and converted from there.  grid (n_slabs_W, G).
// ---------------------------------------------------------------------------------------
constexpr int PG_TILE_BOX_BYTES = 4096;          // one TMA box: 4 KB of the tile
constexpr int PG_TILE_TARGET_BYTES = 48 * 1024;  // default bound on a CTA's tile (see the shape orders)
constexpr double PG_TILE_SIGMAS = 1.5;           // tile rows: n + PG_TILE_SIGMAS * sqrt(n) + 16
constexpr int PG_TILE_THREADS = 128;
// CTAs per SM the register budget of a tile kernel allows (launch bounds): 8 for
// row-major (64 registers); column-major 6 (80 registers) for 16-column slabs and 5
// (up to 102) for 32- and 64-column ones, whose 35..48 KB tiles allow five or six per SM
// anyway -- measured: the wider slabs gain 3-5% from the registers (65536 rows x 16
// groups, 16640 x 32 groups), 16-column slabs lose 9% from the lost CTA (8192-row groups).
__host__ __device__ constexpr int pg_min_blocks(bool col_major, int w) { return col_major ? (w == 16 ? 6 : 5) : 8; }
constexpr uint64_t PG_DRAIN_LIMIT_NS = 20000000000ull;  // after giving up: wait for copies in flight
constexpr double PG_PF_WAVES = 0.5;              // L2 prefetch distance, in waves of resident CTAs

__device__ unsigned int g_wait_timeouts = 0;     // CTAs that gave up a bounded wait
__device__ unsigned int g_wait_abandoned = 0;    // ... and whose copies in flight did not land either

// Limit of the bounded waits of the launches that follow (host side; the kernels take it
// as an argument).  0 makes every such wait give up at once.
std::atomic<uint64_t> g_wait_limit_ns{MXQ_WAIT_LIMIT_DEFAULT_NS};

// After a CTA gave up waiting on `bar`: wait (with a long limit) for the copies still in
// flight into its shared memory, so that none lands after the CTA has exited; a CTA whose
// copies do not land even then is counted separately.  Called by every thread.
__device__ __forceinline__ void drain_after_give_up(uint64_t* bar) {
    const bool drained = mbar_wait_bounded(bar, 0, PG_DRAIN_LIMIT_NS);
    if (__syncthreads_or(!drained) && threadIdx.x == 0) atomicAdd(&g_wait_abandoned, 1u);
}

__device__ __forceinline__ uint8_t* align128(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 127) & ~(uintptr_t)127);
}

// Tile geometry for a W-column slab: rows per TMA box, and the row granularity that
// keeps a box's shared-memory destination 128-byte aligned.
__host__ __device__ constexpr int pg_box_rows(int w) { return PG_TILE_BOX_BYTES / (2 * w); }
__host__ __device__ constexpr int pg_align_rows(int w) { return w >= 64 ? 1 : 128 / (2 * w); }
__host__ __device__ constexpr int pg_tile_rows_alloc(int r_cap, int w) {
    return (r_cap > pg_box_rows(w) ? r_cap : pg_box_rows(w)) + pg_align_rows(w);
}
__host__ __device__ constexpr int pg_tile_smem(int r_cap, int w) { return 128 + pg_tile_rows_alloc(r_cap, w) * w * 2; }

// Store bytes [lo, hi) of the little-endian word w to dst[lo..hi) in naturally
// aligned pieces of 8, 4, 2 or 1 bytes.  (TAG only gives each calling kernel its own
// out-of-line instance, so the callers keep separate register allocations.)
template <int TAG>
__device__ __noinline__ void store_byte_range(uint8_t* dst, uint64_t w, int lo, int hi, uint64_t pol) {
    int a = lo;
    while (a < hi) {
        const uintptr_t addr = reinterpret_cast<uintptr_t>(dst + a);
        const int n = hi - a;
        if (n >= 8 && (addr & 7) == 0) {
            st_v2_hint(dst + a, make_uint2((uint32_t)(w >> (8 * a)), (uint32_t)(w >> (8 * a + 32))), pol);
            a += 8;
        } else if (n >= 4 && (addr & 3) == 0) {
            *reinterpret_cast<uint32_t*>(dst + a) = (uint32_t)(w >> (8 * a));
            a += 4;
        } else if (n >= 2 && (addr & 1) == 0) {
            *reinterpret_cast<uint16_t*>(dst + a) = (uint16_t)(w >> (8 * a));
            a += 2;
        } else {
            dst[a] = (uint8_t)(w >> (8 * a));
            a += 1;
        }
    }
}

// Store bytes [lo, hi) of the word w at dst (8-byte aligned when aligned8): one 8-byte
// store for a whole word, at most three naturally aligned pieces for a head (hi == 8)
// or tail (lo == 0) word, byte pieces otherwise.
__device__ __forceinline__ void store_word_range(uint8_t* dst, uint64_t w, int lo, int hi, bool aligned8,
                                                 uint64_t pol) {
    if (aligned8 && lo == 0 && hi == 8) {
        st_v2_hint(dst, make_uint2((uint32_t)w, (uint32_t)(w >> 32)), pol);
    } else if (aligned8 && (lo == 0 || hi == 8)) {
        if (hi == 8) {
            if (lo & 1) dst[lo] = (uint8_t)(w >> (8 * lo));
            const int a2 = (lo + 1) & ~1;
            if (a2 & 2) *reinterpret_cast<uint16_t*>(dst + a2) = (uint16_t)(w >> (8 * a2));
            const int a4 = (lo + 3) & ~3;
            if (a4 == 4) *reinterpret_cast<uint32_t*>(dst + 4) = (uint32_t)(w >> 32);
        } else {
            if (hi & 4) *reinterpret_cast<uint32_t*>(dst) = (uint32_t)w;
            if (hi & 2) *reinterpret_cast<uint16_t*>(dst + (hi & 4)) = (uint16_t)(w >> (8 * (hi & 4)));
            if (hi & 1) dst[hi & 6] = (uint8_t)(w >> (8 * (hi & 6)));
        }
    } else {
        store_byte_range<1>(dst, w, lo, hi, pol);
    }
}


// Column-major conversion of rows [r_lo, r_hi) straight from global memory, one row
// per lane step (rows first + lane, step `step`; 8 byte stores per row).  Only rows of
// a group larger than its tile come here.  (TAG: one out-of-line instance per calling
// kernel.)
template <int TAG>
__device__ __noinline__ void convert_rows_col_major(const uint16_t* __restrict__ x, int64_t r_lo, int64_t r_hi,
                                                    int first, int step, const float* f, uint8_t* __restrict__ q,
                                                    int64_t M, int64_t K, int64_t c) {
    for (int64_t r = r_lo + first; r < r_hi; r += step) {
        const uint4 e = ld_nc_v4(x + r * K + c);
        const uint32_t wd[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float val = (j & 1) ? bf16_hi(wd[j >> 1]) : bf16_lo(wd[j >> 1]);
            q[(c + j) * M + r] = (uint8_t)(cvt_e4m3x2(__fmul_rn(val, f[j]), 0.0f) & 0xFFu);
        }
    }
}

// Column maxima (four bf16x2 words) of rows r0, r0 + step, ... < r_hi (rows of a group
// beyond its tile) folded into cm: four loads in flight per lane, kept in L2 (evict_last) for the conversion's second
// read.  (Out of line, so the tile kernel keeps its own register allocation.)
__device__ __noinline__ uint4 overflow_maxima(const uint16_t* __restrict__ x, int64_t r0, int64_t r_hi, int step,
                                              int64_t K, int64_t c, uint4 cm, bool lead) {
    const uint64_t keep = l2_policy_evict_last();
    const int64_t ahead = PG_OVF_PF_STEPS * 4 * (int64_t)step;
    uint32_t m0 = cm.x, m1 = cm.y, m2 = cm.z, m3 = cm.w;
    for (int64_t r = r0; r < r_hi; r += 4 * (int64_t)step) {
        if (lead) {  // one lane per row: its line, some loop steps ahead, into L2
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (r + u * step + ahead < r_hi) prefetch_l2(x + (r + u * step + ahead) * K + c);
        }
        uint4 e[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            e[u] = r + u * step < r_hi ? ld_nc_v4_hint(x + (r + u * step) * K + c, keep) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            m0 = amax2(m0, e[u].x);
            m1 = amax2(m1, e[u].y);
            m2 = amax2(m2, e[u].z);
            m3 = amax2(m3, e[u].w);
        }
    }
    return make_uint4(m0, m1, m2, m3);
}

// Column-major conversion of rows [r_lo, r_hi) of a group beyond its tile, from global
// memory (second read: evict_first).  With M % 8 == 0 the rows from the first multiple of
// 8 to the last go as octets, one per lane step (8 rows loaded, eight 8-byte column
// words stored: whole sectors across four lanes); the rows before and after, and all
// rows when M % 8 != 0, one row per lane step with byte stores.  Lanes: first + i * step.
__device__ __noinline__ void convert_overflow_col_major(const uint16_t* __restrict__ x, int64_t r_lo, int64_t r_hi,
                                                        int first, int step, bool lead, const float* fp,
                                                        uint8_t* __restrict__ q, int64_t M, int64_t K, int64_t c) {
    float f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = fp[j];
    const uint64_t drop = l2_policy_evict_first();
    const int64_t a = (M & 7) ? r_hi : min(r_hi, (r_lo + 7) & ~(int64_t)7);  // aligned body [a, b)
    const int64_t b = (M & 7) ? r_hi : max(a, r_hi & ~(int64_t)7);
    const int64_t ahead = 2 * 8 * (int64_t)step;  // two loop steps
    for (int64_t r = a + 8 * (int64_t)first; r + 8 <= b; r += 8 * (int64_t)step) {
        if (lead && r + ahead + 8 <= b) {  // one lane per row group: the octet two steps ahead
#pragma unroll
            for (int t = 0; t < 8; ++t) prefetch_l2(x + (r + ahead + t) * K + c);
        }
        uint4 d[8];
        load_octet<true>(d, x, r, 0, 8, K, c, drop);
#pragma unroll
        for (int j = 0; j < 8; ++j) st_v2_hint(q + (c + j) * M + r, octet_column_codes(d, f, j), drop);
    }
    for (int64_t r = r_lo + first; r < r_hi; r += step) {
        if (r >= a && r < b) {  // inside the body: skip to its end
            r += ((b - r + step - 1) / step) * step - step;
            continue;
        }
        const uint4 e = ld_nc_v4(x + r * K + c);
        const uint32_t wd[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float val = (j & 1) ? bf16_hi(wd[j >> 1]) : bf16_lo(wd[j >> 1]);
            q[(c + j) * M + r] = (uint8_t)(cvt_e4m3x2(__fmul_rn(val, f[j]), 0.0f) & 0xFFu);
        }
    }
}

// Conversion and store of a tile's rows (the part of per_group_tile_kernel after the
// scales are known).
template <bool COL_MAJOR, int W>
__device__ __forceinline__ void convert_tile(const uint8_t* tile, const uint16_t* __restrict__ x, int64_t start,
                                             int64_t end, int64_t rows, int res, int r_cap, const float* sc,
                                             uint8_t* __restrict__ q, int64_t M, int64_t K, int64_t c, int v,
                                             int rl) {
    constexpr int L = W / 8;
    constexpr int ROW_B = 2 * W;
    constexpr int N_RL = PG_TILE_THREADS / L;
    float f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = sc[8 * v + j];
    const uint64_t drop = l2_policy_evict_first();

    if (!COL_MAJOR) {
        // ---- row-major: each lane converts 8 columns of a row and stores 8 bytes
        const uint8_t* sp = tile + 16 * v;
        uint8_t* dst = q + (start + rl) * K + c;
        const int64_t dstep = (int64_t)N_RL * K;
        for (int r = rl; r < res; r += N_RL, dst += dstep) {
            const uint4 e = lds_v4(sp + r * ROW_B);
            float p[8];
            fmul2(bf16_lo(e.x), bf16_hi(e.x), f[0], f[1], p[0], p[1]);
            fmul2(bf16_lo(e.y), bf16_hi(e.y), f[2], f[3], p[2], p[3]);
            fmul2(bf16_lo(e.z), bf16_hi(e.z), f[4], f[5], p[4], p[5]);
            fmul2(bf16_lo(e.w), bf16_hi(e.w), f[6], f[7], p[6], p[7]);
            st_v2_hint(dst, make_uint2(cvt4_e4m3(p[0], p[1], p[2], p[3]), cvt4_e4m3(p[4], p[5], p[6], p[7])), drop);
        }
        // rows beyond the resident ones: read again from global memory
        for (int64_t rg = start + r_cap + rl; rg < end; rg += N_RL) {
            uint4 d[8];
            load_octet(d, x, rg, 0, 1, K, c);
            store_octet<false>(d, f, q, rg, 0, 1, M, K, c, false);
        }
    } else {
        // ---- column-major: lane = (octet k of rows base + 8k .. +7, 8 columns), octets
        // aligned to 32 rows so a warp's 8-byte column stores fill whole sectors.  At step
        // t a lane reads row (t + rot) % 8 of its octet, rot = k % 8, so the rows a warp
        // reads at once fall in distinct bank groups; two byte permutes put each column
        // word back in row order.  A cut octet (a group's first or last) reads a row inside
        // the group in place of each row outside it: those bytes are never stored.
        const int64_t base = start & ~(int64_t)31;
        const int rel0 = (int)(start - base);
        const int rel_end = rel0 + res;
        const uint32_t tile_s = smem_addr(tile) + 16 * v;
        for (int k = rl; 8 * k < rel_end; k += N_RL) {
            const int lo = max(0, rel0 - 8 * k), hi = min(8, rel_end - 8 * k);
            if (lo >= hi) continue;  // before the first row (the 32-row alignment)
            const int rot = W == 64 ? 0 : k & 7;  // 128-byte rows: any 4 rows are conflict-free
            const uint32_t perm = __funnelshift_l(0x76543210u, 0x76543210u, 4 * rot);  // nibble i: (i - rot) % 8
            const uint32_t perm_lo = perm & 0xFFFFu, perm_hi = perm >> 16;
            const bool whole = lo == 0 && hi == 8;
            const uint32_t oct = tile_s + (uint32_t)((8 * k - rel0) * ROW_B);  // row 0 (mod 2^32)
            if (W < 64 && whole && (M & 7) == 0) {
                // whole octet: rotated rows without clamping, 8-byte column stores
                uint8_t* dst = q + c * M + base + 8 * k;
                uint4 e[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) e[t] = lds_v4_at(oct + (uint32_t)(((t + rot) & 7) * ROW_B));
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint2 w = octet_column_codes(e, f, j);  // byte t = row (t + rot) % 8
                    st_v2_hint(dst + j * M, make_uint2(__byte_perm(w.x, w.y, perm_lo), __byte_perm(w.x, w.y, perm_hi)),
                               drop);
                }
                continue;
            }
            uint4 e[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (W == 64)  // (this form keeps the 64-column kernels free of spills)
                    e[t] = (t >= lo && t < hi) ? lds_v4(tile + (8 * k + t - rel0) * ROW_B + 16 * v)
                                               : make_uint4(0, 0, 0, 0);
                else
                    e[t] = lds_v4_at(oct + (uint32_t)(min(max((t + rot) & 7, lo), hi - 1) * ROW_B));
            }
            uint8_t* dst = q + c * M + base + 8 * k;
            if (whole && (M & 7) == 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j, dst += M) {
                    const uint2 w = octet_column_codes(e, f, j);  // byte t = row (t + rot) % 8
                    st_v2_hint(dst,
                               W == 64 ? w
                                       : make_uint2(__byte_perm(w.x, w.y, perm_lo), __byte_perm(w.x, w.y, perm_hi)),
                               drop);
                }
            } else if ((M & 7) == 0 && (lo == 0 || hi == 8)) {
                // the octet holding the group's first (hi == 8) or last (lo == 0) row:
                // its bytes of each 8-byte-aligned column word in at most three
                // naturally aligned pieces
#pragma unroll
                for (int j = 0; j < 8; ++j, dst += M) {
                    const uint2 w2 = octet_column_codes(e, f, j);
                    const uint64_t w = W == 64 ? (((uint64_t)w2.y << 32) | w2.x)
                                               : (((uint64_t)__byte_perm(w2.x, w2.y, perm_hi) << 32) |
                                                  __byte_perm(w2.x, w2.y, perm_lo));
                    if (hi == 8) {
                        if (lo & 1) dst[lo] = (uint8_t)(w >> (8 * lo));
                        const int a2 = (lo + 1) & ~1;
                        if (a2 & 2) *reinterpret_cast<uint16_t*>(dst + a2) = (uint16_t)(w >> (8 * a2));
                        const int a4 = (lo + 3) & ~3;
                        if (a4 == 4) *reinterpret_cast<uint32_t*>(dst + 4) = (uint32_t)(w >> 32);
                    } else {
                        if (hi & 4) *reinterpret_cast<uint32_t*>(dst) = (uint32_t)w;
                        if (hi & 2) *reinterpret_cast<uint16_t*>(dst + (hi & 4)) = (uint16_t)(w >> (8 * (hi & 4)));
                        if (hi & 1) dst[hi & 6] = (uint8_t)(w >> (8 * (hi & 6)));
                    }
                }
            } else {
                for (int j = 0; j < 8; ++j, dst += M) {
                    const uint2 w2 = octet_column_codes(e, f, j);
                    const uint64_t w = W == 64 ? (((uint64_t)w2.y << 32) | w2.x)
                                               : (((uint64_t)__byte_perm(w2.x, w2.y, perm_hi) << 32) |
                                                  __byte_perm(w2.x, w2.y, perm_lo));
                    store_byte_range<0>(dst, w, lo, hi, drop);
                }
            }
        }
        if (rows > r_cap) {  // rows beyond the resident ones, from global memory
            if (W == 64)  // (the row-at-a-time form keeps this instance free of spills)
                convert_rows_col_major<0>(x, start + r_cap, end, rl, N_RL, f, q, M, K, c);
            else
                convert_overflow_col_major(x, start + r_cap, end, rl, N_RL, v == 0, f, q, M, K, c);
        }
    }
}

template <bool COL_MAJOR, int W, int CL>
__global__ void __launch_bounds__(PG_TILE_THREADS, pg_min_blocks(COL_MAJOR, W))
    per_group_tile_kernel(const __grid_constant__ CUtensorMap xmap, const uint16_t* __restrict__ x, int64_t M,
                          int64_t K, const int32_t* __restrict__ offs, uint8_t* __restrict__ q,
                          float* __restrict__ scales, int r_cap, uint32_t pf_ahead, uint64_t wait_ns,
                          int rows_per_group) {
    constexpr int L = W / 8;                  // lanes per row, 8 columns each
    constexpr int BOX_R = pg_box_rows(W);     // rows per TMA box
    constexpr int ALIGN_R = pg_align_rows(W);
    constexpr int ROW_B = 2 * W;              // bytes per tile row
    constexpr int N_WARPS = PG_TILE_THREADS / 32;
    constexpr int N_RL = PG_TILE_THREADS / L; // row lanes
    __shared__ uint64_t bar;
    __shared__ uint64_t xbar;                 // cluster exchange: all partial maxima landed
    __shared__ uint32_t red[N_WARPS][W / 2];
    __shared__ uint32_t parts[CL][W / 2];     // column maxima of every CTA of the cluster
    __shared__ uint32_t skips[CL];            // which CTAs of the cluster gave up on their tile
    __shared__ float sc[W];
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* tile = align128(dyn_smem);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid % L, rl = tid / L;
    const int g = blockIdx.y;
    const int rank = CL > 1 ? (int)cluster_ctarank() : 0;
    const int64_t k0 = (int64_t)(blockIdx.x / CL) * W;
    const int64_t c = k0 + 8 * v;
    const bool cv = c < K;
    if (tid == 0) {
        mbar_init(&bar, 1);
        if (CL > 1) {
            mbar_init(&xbar, 1);
            mbar_arrive_expect_tx(&xbar, (uint32_t)(CL * (W / 2 + 1) * 4));
        }
    }

    // group bounds: every warp reduces the running maximum of offs[0..g-1] itself
    int pm = 0;
    for (int i = lane; i < g; i += 32) pm = max(pm, end_offset(offs, i, rows_per_group));
#pragma unroll
    for (int sh = 16; sh; sh >>= 1) pm = max(pm, __shfl_xor_sync(FULL_MASK, pm, sh));
    const int64_t g_start = min((int64_t)pm, M);
    const int64_t g_end = min((int64_t)max(pm, end_offset(offs, g, rows_per_group)), M);
    // this CTA's rows [start, end): the group split among the CL CTAs of the cluster at
    // multiples of 32 rows (so no two CTAs write into one sector of a column)
    int64_t start = g_start, end = g_end;
    if (CL > 1) {
        const int64_t chunk = (g_end - g_start + CL - 1) / CL;
        if (rank > 0) start = min(g_end, max(g_start, (g_start + rank * chunk) & ~(int64_t)31));
        if (rank < CL - 1) end = min(g_end, max(g_start, (g_start + (rank + 1) * chunk) & ~(int64_t)31));
    }
    const int64_t rows = end - start;
    int res = (int)min(rows, (int64_t)r_cap);  // rows resident in shared memory
    __syncthreads();                           // barriers initialised
    if (CL > 1) cluster_arrive_relaxed();      // ... and, once every CTA arrived, cluster-wide

    if (tid == 0 && res > 0) {
        // boxes at 0, BOX_R, ...; the last one ends at res (its start rounded up to
        // ALIGN_R rows so the destination stays 128-byte aligned), so at most
        // ALIGN_R - 1 rows past the group are fetched
        const uint64_t pol = l2_policy_evict_first();
        const int n_box = (res + BOX_R - 1) / BOX_R;
        mbar_arrive_expect_tx(&bar, (uint32_t)(n_box * PG_TILE_BOX_BYTES));
        for (int b = 0; b < n_box; ++b) {
            const int y = (b == n_box - 1 && b > 0) ? (res - BOX_R + ALIGN_R - 1) / ALIGN_R * ALIGN_R : b * BOX_R;
            tma_load_2d(tile + y * ROW_B, &xmap, (int)k0, (int)(start + y), &bar, pol);
        }
    }
    if (pf_ahead && warp == 1) {
        // L2 prefetch of the tile of the CTA pf_ahead further on in launch order (part of
        // a wave: a CTA that starts soon), found the way that CTA finds its own rows
        const uint32_t gx = gridDim.x, tgt = blockIdx.x + gx * blockIdx.y + pf_ahead;
        if (tgt < gx * gridDim.y) {
            const int g2 = (int)(tgt / gx), bx2 = (int)(tgt % gx), rank2 = bx2 % CL;
            int pm2 = 0;
            for (int i = lane; i < g2; i += 32) pm2 = max(pm2, end_offset(offs, i, rows_per_group));
#pragma unroll
            for (int sh = 16; sh; sh >>= 1) pm2 = max(pm2, __shfl_xor_sync(FULL_MASK, pm2, sh));
            if (lane == 0) {
                const int64_t gs = min((int64_t)pm2, M);
                const int64_t ge = min((int64_t)max(pm2, end_offset(offs, g2, rows_per_group)), M);
                int64_t s2 = gs, e2 = ge;
                if (CL > 1) {
                    const int64_t chunk = (ge - gs + CL - 1) / CL;
                    if (rank2 > 0) s2 = min(ge, max(gs, (gs + rank2 * chunk) & ~(int64_t)31));
                    if (rank2 < CL - 1) e2 = min(ge, max(gs, (gs + (rank2 + 1) * chunk) & ~(int64_t)31));
                }
                const int res2 = (int)min(e2 - s2, (int64_t)r_cap);
                const uint64_t keep = l2_policy_evict_last();
                for (int y = 0; y < res2; y += BOX_R) tma_prefetch_2d(&xmap, (bx2 / CL) * W, (int)(s2 + y), keep);
            }
        }
    }
    // A CTA that gives up a wait skips its tile; in a cluster every CTA then skips it
    // (neither codes nor scales of this (group, slab) are written), so no output is
    // derived from incomplete maxima.
    bool skip = false, gave_up = false;
    if (res > 0) {
        const bool landed = mbar_wait_bounded(&bar, 0, wait_ns);
        if (__syncthreads_or(!landed)) {  // the whole CTA gives up together
            drain_after_give_up(&bar);
            gave_up = skip = true;
            res = 0;
        }
    }

    // ---- column maxima: resident rows from shared memory (a warp reads consecutive
    // rows, conflict-free), the rest from global memory
    uint32_t cm[4] = {0, 0, 0, 0};
    if (cv && !skip) {
        const uint8_t* sp = tile + 16 * v;
        int r = rl;
        for (; r + 3 * N_RL < res; r += 4 * N_RL) {
            uint4 e[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) e[u] = lds_v4(sp + (r + u * N_RL) * ROW_B);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                cm[0] = amax2(cm[0], e[u].x);
                cm[1] = amax2(cm[1], e[u].y);
                cm[2] = amax2(cm[2], e[u].z);
                cm[3] = amax2(cm[3], e[u].w);
            }
        }
        for (; r < res; r += N_RL) {
            const uint4 e = lds_v4(sp + r * ROW_B);
            cm[0] = amax2(cm[0], e.x);
            cm[1] = amax2(cm[1], e.y);
            cm[2] = amax2(cm[2], e.z);
            cm[3] = amax2(cm[3], e.w);
        }
        // rows beyond the tile, kept in L2 (evict_last) for the conversion's second read
        if (W == 64 && COL_MAJOR) {  // (inline: a call here costs this instance a spill)
            const uint64_t keep = l2_policy_evict_last();
            for (int64_t rg = start + r_cap + rl; rg < end; rg += N_RL) {
                if (v == 0 && rg + PG_OVF_PF_STEPS * N_RL < end) prefetch_l2(x + (rg + PG_OVF_PF_STEPS * N_RL) * K + c);
                const uint4 e = ld_nc_v4_hint(x + rg * K + c, keep);
                cm[0] = amax2(cm[0], e.x);
                cm[1] = amax2(cm[1], e.y);
                cm[2] = amax2(cm[2], e.z);
                cm[3] = amax2(cm[3], e.w);
            }
        } else if (start + r_cap < end) {
            const uint4 m = overflow_maxima(x, start + r_cap + rl, end, N_RL, K, c, make_uint4(cm[0], cm[1], cm[2], cm[3]),
                                            v == 0);
            cm[0] = m.x;
            cm[1] = m.y;
            cm[2] = m.z;
            cm[3] = m.w;
        }
    }
#pragma unroll
    for (int sh = L; sh < 32; sh <<= 1)
#pragma unroll
        for (int w = 0; w < 4; ++w) cm[w] = amax2(cm[w], __shfl_xor_sync(FULL_MASK, cm[w], sh));
    if (lane < L)
#pragma unroll
        for (int w = 0; w < 4; ++w) red[warp][lane * 4 + w] = cm[w];
    __syncthreads();
    uint32_t m = 0;
    if (tid < W / 2) {
#pragma unroll
        for (int w = 0; w < N_WARPS; ++w) m = amax2(m, red[w][tid]);
    }
    if (CL > 1) {
        // exchange of the partial maxima: each CTA pushes its W/2 words into slot `rank`
        // of every CTA's parts[] with st.async, each completing on the receiver's xbar;
        // a CTA reads parts[] once its xbar has seen all CL * W/2 words, plus one skip
        // word from every CTA (bounded wait)
        cluster_wait();  // every CTA's xbar is initialised
        if (tid < W / 2) {
#pragma unroll
            for (int r = 0; r < CL; ++r)
                st_async_u32(cluster_map(&parts[rank][tid], (uint32_t)r), m, cluster_map(&xbar, (uint32_t)r));
        } else if (tid == W / 2) {
#pragma unroll
            for (int r = 0; r < CL; ++r)
                st_async_u32(cluster_map(&skips[rank], (uint32_t)r), skip ? 1u : 0u, cluster_map(&xbar, (uint32_t)r));
        }
        cluster_arrive_relaxed();  // matched by the wait at the end: no CTA exits early
        const bool got = mbar_wait_bounded(&xbar, 0, wait_ns);
        if (__syncthreads_or(!got)) {
            drain_after_give_up(&xbar);
            gave_up = skip = true;
        } else {
            uint32_t any = 0;
#pragma unroll
            for (int r = 0; r < CL; ++r) any |= skips[r];
            skip = any != 0u;
        }
        if (tid < W / 2 && !skip)
#pragma unroll
            for (int r = 0; r < CL; ++r) m = amax2(m, parts[r][tid]);
    }
    if (gave_up && tid == 0) atomicAdd(&g_wait_timeouts, 1u);
    if (tid < W / 2) {
        m = mag2(m);
        // word tid = columns 8*(tid/4) + 2*(tid%4) + {0, 1} of the slab
        const int col0 = 8 * (tid >> 2) + 2 * (tid & 3);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float sv = group_scale(h ? (m >> 16) : (m & 0xFFFFu));
            sc[col0 + h] = sv;
            if (rank == 0 && !skip && k0 + col0 + h < K) scales[(int64_t)g * K + k0 + col0 + h] = sv;
        }
    }
    __syncthreads();
    if (cv && !skip) {
        // column-major codes of a batched tensor: group g's (K, rows_per_group) matrix
        uint8_t* qg = (COL_MAJOR && rows_per_group > 0) ? q + (int64_t)g * rows_per_group * (K - 1) : q;
        const int64_t col_stride = (COL_MAJOR && rows_per_group > 0) ? rows_per_group : M;
        convert_tile<COL_MAJOR, W>(tile, x, start, end, rows, res, r_cap, sc, qg, col_stride, K, c, v, rl);
    }
    if (CL > 1) cluster_wait();
}

// ---------------------------------------------------------------------------------------
// Column-major output, small groups: one CTA per pair of neighbouring groups (2p, 2p+1)
// and 64-column slab; grid (n_slabs64, ceil(G / 2)).  The pair shares one TMA tile, and
// the octet holding the boundary between its two groups is assembled from both groups'
// codes and stored with whole 8-byte column words, so only the pair's outer boundaries
// are cut (a group boundary otherwise costs up to three piece stores per column).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(PG_TILE_THREADS, pg_min_blocks(true, 64)) per_group_pair_col_kernel(
    const __grid_constant__ CUtensorMap xmap, const uint16_t* __restrict__ x, int64_t M, int64_t K,
    const int32_t* __restrict__ offs, int32_t G, uint8_t* __restrict__ q, float* __restrict__ scales, int r_cap,
    uint64_t wait_ns, int rows_per_group) {
    constexpr int W = 64, L = 8;
    constexpr int BOX_R = pg_box_rows(W), ALIGN_R = pg_align_rows(W), ROW_B = 2 * W;
    constexpr int N_WARPS = PG_TILE_THREADS / 32, N_RL = PG_TILE_THREADS / L;
    __shared__ uint64_t bar;
    __shared__ uint32_t red[2][N_WARPS][W / 2];
    __shared__ __align__(16) float sc[2][W];
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* tile = align128(dyn_smem);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid % L, rl = tid / L;
    const int gA = 2 * (int)blockIdx.y, gB = gA + 1;
    const bool hasB = gB < G;
    const int64_t k0 = (int64_t)blockIdx.x * W;
    const int64_t c = k0 + 8 * v;
    const bool cv = c < K;
    if (tid == 0) mbar_init(&bar, 1);

    // bounds of the two groups (the clamp rule): start, mid (end of A), end (end of B)
    int pm = 0;
    for (int i = lane; i < gA; i += 32) pm = max(pm, end_offset(offs, i, rows_per_group));
#pragma unroll
    for (int sh = 16; sh; sh >>= 1) pm = max(pm, __shfl_xor_sync(FULL_MASK, pm, sh));
    const int pmA = max(pm, end_offset(offs, gA, rows_per_group));
    const int64_t start = min((int64_t)pm, M);
    const int64_t mid = min((int64_t)pmA, M);
    const int64_t end = hasB ? min((int64_t)max(pmA, end_offset(offs, gB, rows_per_group)), M) : mid;
    const int64_t rows = end - start;
    int res = (int)min(rows, (int64_t)r_cap);
    __syncthreads();

    if (tid == 0 && res > 0) {
        const uint64_t pol = l2_policy_evict_first();
        const int n_box = (res + BOX_R - 1) / BOX_R;
        mbar_arrive_expect_tx(&bar, (uint32_t)(n_box * PG_TILE_BOX_BYTES));
        for (int b = 0; b < n_box; ++b) {
            const int y = (b == n_box - 1 && b > 0) ? (res - BOX_R + ALIGN_R - 1) / ALIGN_R * ALIGN_R : b * BOX_R;
            tma_load_2d(tile + y * ROW_B, &xmap, (int)k0, (int)(start + y), &bar, pol);
        }
    }
    bool skip = false;  // gave up on the tile: neither codes nor scales of the pair are written
    if (res > 0) {
        const bool landed = mbar_wait_bounded(&bar, 0, wait_ns);
        if (__syncthreads_or(!landed)) {
            if (tid == 0) atomicAdd(&g_wait_timeouts, 1u);
            drain_after_give_up(&bar);
            skip = true;
            res = 0;
        }
    }

    // ---- column maxima of both groups: tile rows [0, mrel) are A's, [mrel, res) B's
    const int mrel = (int)min(mid - start, (int64_t)res);
    uint32_t ca[4] = {0, 0, 0, 0}, cb[4] = {0, 0, 0, 0};
    if (cv && !skip) {
        const uint8_t* sp = tile + 16 * v;
        int r = rl;
        for (; r < mrel; r += N_RL) {
            const uint4 e = lds_v4(sp + r * ROW_B);
            ca[0] = amax2(ca[0], e.x); ca[1] = amax2(ca[1], e.y); ca[2] = amax2(ca[2], e.z); ca[3] = amax2(ca[3], e.w);
        }
        for (; r < res; r += N_RL) {
            const uint4 e = lds_v4(sp + r * ROW_B);
            cb[0] = amax2(cb[0], e.x); cb[1] = amax2(cb[1], e.y); cb[2] = amax2(cb[2], e.z); cb[3] = amax2(cb[3], e.w);
        }
        for (int64_t rg = start + r_cap + rl; rg < end; rg += N_RL) {  // rows beyond the tile
            const uint4 e = ld_nc_v4(x + rg * K + c);
            uint32_t* cm = rg < mid ? ca : cb;
            cm[0] = amax2(cm[0], e.x); cm[1] = amax2(cm[1], e.y); cm[2] = amax2(cm[2], e.z); cm[3] = amax2(cm[3], e.w);
        }
    }
#pragma unroll
    for (int sh = L; sh < 32; sh <<= 1)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            ca[w] = amax2(ca[w], __shfl_xor_sync(FULL_MASK, ca[w], sh));
            cb[w] = amax2(cb[w], __shfl_xor_sync(FULL_MASK, cb[w], sh));
        }
    if (lane < L)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            red[0][warp][lane * 4 + w] = ca[w];
            red[1][warp][lane * 4 + w] = cb[w];
        }
    __syncthreads();
    if (tid < W) {  // thread = (group tid / 32, word tid % 32)
        const int grp = tid >> 5, wd = tid & 31;
        uint32_t m = 0;
#pragma unroll
        for (int w = 0; w < N_WARPS; ++w) m = amax2(m, red[grp][w][wd]);
        m = mag2(m);
        const int col0 = 8 * (wd >> 2) + 2 * (wd & 3);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float sv = group_scale(h ? (m >> 16) : (m & 0xFFFFu));
            sc[grp][col0 + h] = sv;
            if ((grp == 0 || hasB) && !skip && k0 + col0 + h < K) scales[(int64_t)(gA + grp) * K + k0 + col0 + h] = sv;
        }
    }
    __syncthreads();
    if (!cv || skip) return;

    // ---- conversion: octets of rows base + 8k .. +7 (base = start rounded down to 32)
    const uint64_t drop = l2_policy_evict_first();
    const bool aligned8 = (M & 7) == 0;
    const int64_t base = start & ~(int64_t)31;
    const int rel0 = (int)(start - base);
    const int rel_end = rel0 + res;
    const int mb = rel0 + mrel;  // first row of B, relative to base
    for (int k = rl; 8 * k < rel_end; k += N_RL) {
        const int lo = max(0, rel0 - 8 * k), hi = min(8, rel_end - 8 * k);
        if (lo >= hi) continue;
        uint4 e[8];
#pragma unroll
        for (int t = 0; t < 8; ++t)
            e[t] = (t >= lo && t < hi) ? lds_v4(tile + (8 * k + t - rel0) * ROW_B + 16 * v) : make_uint4(0, 0, 0, 0);
        uint8_t* dst = q + c * M + base + 8 * k;
        const int split = mb - 8 * k;  // rows t < split are A's
        if (split >= 8 || split <= 0) {
            const float* fs = &sc[split >= 8 ? 0 : 1][8 * v];
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] = fs[j];
#pragma unroll
            for (int j = 0; j < 8; ++j, dst += M) {
                const uint2 w = octet_column_codes(e, f, j);
                store_word_range(dst, ((uint64_t)w.y << 32) | w.x, lo, hi, aligned8, drop);
            }
        } else {
            const uint64_t keep_a = (1ull << (8 * split)) - 1;  // bytes of A's rows
#pragma unroll
            for (int j = 0; j < 8; ++j, dst += M) {
                const uint2 wa = octet_column_codes_s(e, sc[0][8 * v + j], j);
                const uint2 wb = octet_column_codes_s(e, sc[1][8 * v + j], j);
                const uint64_t w = ((((uint64_t)wa.y << 32) | wa.x) & keep_a) | ((((uint64_t)wb.y << 32) | wb.x) & ~keep_a);
                store_word_range(dst, w, lo, hi, aligned8, drop);
            }
        }
    }
    if (rows > r_cap) {  // rows beyond the tile, from global memory, split at mid
        const int64_t lo_r = start + r_cap;
        if (lo_r < mid) convert_rows_col_major<1>(x, lo_r, mid, rl, N_RL, &sc[0][8 * v], q, M, K, c);
        if (max(lo_r, mid) < end) convert_rows_col_major<1>(x, max(lo_r, mid), end, rl, N_RL, &sc[1][8 * v], q, M, K, c);
    }
}

// ---------------------------------------------------------------------------------------
// Large groups: grid (n_slabs32, G), 512 threads, two streaming passes over the tile.
// ---------------------------------------------------------------------------------------
template <bool COL_MAJOR>
__global__ void __launch_bounds__(PG_BIG_THREADS, 1) per_group_big_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, const int32_t* __restrict__ offs,
    uint8_t* __restrict__ q, float* __restrict__ scales, bool vec_col_store, int rows_per_group) {
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
    const GroupRows gr = group_rows(offs, g, M, scratch, rows_per_group);
    // column-major codes of a batched tensor: group g's (K, rows_per_group) matrix
    uint8_t* qg = (COL_MAJOR && rows_per_group > 0) ? q + (int64_t)g * rows_per_group * (K - 1) : q;
    const int64_t col_stride = (COL_MAJOR && rows_per_group > 0) ? rows_per_group : M;
    // column-major: a warp's eight octets start on a 64-row boundary (two aligned
    // sectors per column per store)
    const int64_t ob = COL_MAJOR ? (gr.start >> 6) << 3 : gr.start >> 3;
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
            store_octet<COL_MAJOR, true>(d, f, qg, oc * 8, lo, hi, col_stride, K, c, vec_col_store, drop);
        }
    }
}

// ---- host side ---------------------------------------------------------------------------

namespace {

template <bool COL_MAJOR, int W, int CL>
cudaError_t launch_tile(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs, int32_t G, uint8_t* q,
                        float* scales, int r_cap, int rows_per_group, cudaStream_t stream) {
    CUtensorMap xmap;
    std::memset(&xmap, 0, sizeof(xmap));
    if (M > 0 &&  // with M == 0 every group is empty and the kernel never reads the map
        !encode_bf16_tile_map(&xmap, x, (uint64_t)K, (uint64_t)M, (uint32_t)W, (uint32_t)pg_box_rows(W)))
        return cudaErrorInvalidValue;
    const int smem = pg_tile_smem(r_cap, W);
    auto kernel = per_group_tile_kernel<COL_MAJOR, W, CL>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((K + W - 1) / W * CL), (unsigned)G);
    cfg.blockDim = dim3(PG_TILE_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = CL > 1 ? 1 : 0;
    // each CTA prefetches into L2 the tile of the CTA PG_PF_WAVES waves later; resident
    // CTAs per SM from the shared memory (228 KB per SM, 1 KB of it reserved per CTA)
    // and the register cap; 32-bit index arithmetic in the kernel: grids below 2^31 CTAs
    const int64_t n_cta = (int64_t)cfg.gridDim.x * cfg.gridDim.y;
    const int per_sm = std::min(pg_min_blocks(COL_MAJOR, W), 228 * 1024 / (smem + 1024));
    // (16-column column-major tiles measured up to 14% slower with the prefetch: off there)
    const bool prefetch = n_cta < ((int64_t)1 << 31) && !(COL_MAJOR && W == 16);
    const uint32_t pf_ahead = prefetch ? (uint32_t)(PG_PF_WAVES * sm_count() * per_sm) : 0u;
    return cudaLaunchKernelEx(&cfg, kernel, xmap, x, M, K, offs, q, scales, r_cap, pf_ahead, g_wait_limit_ns.load(),
                              rows_per_group);
}

cudaError_t launch_pair_col(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs, int32_t G, uint8_t* q,
                            float* scales, int r_cap, cudaStream_t stream) {
    constexpr int W = 64;
    CUtensorMap xmap;
    std::memset(&xmap, 0, sizeof(xmap));
    if (M > 0 && !encode_bf16_tile_map(&xmap, x, (uint64_t)K, (uint64_t)M, (uint32_t)W, (uint32_t)pg_box_rows(W)))
        return cudaErrorInvalidValue;
    const int smem = pg_tile_smem(r_cap, W);
    if (smem > 48 * 1024) {
        const cudaError_t e =
            cudaFuncSetAttribute(per_group_pair_col_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    cudaFuncSetAttribute(per_group_pair_col_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    const dim3 grid((unsigned)((K + W - 1) / W), (unsigned)((G + 1) / 2));
    per_group_pair_col_kernel<<<grid, PG_TILE_THREADS, smem, stream>>>(xmap, x, M, K, offs, G, q, scales, r_cap,
                                                                       g_wait_limit_ns.load(), 0);
    return cudaGetLastError();
}

template <bool COL_MAJOR, int W>
cudaError_t launch_tile_cluster(int cl, const uint16_t* x, int64_t M, int64_t K, const int32_t* offs, int32_t G,
                                uint8_t* q, float* scales, int r_cap, int rpg, cudaStream_t stream) {
    switch (cl) {
        case 1: return launch_tile<COL_MAJOR, W, 1>(x, M, K, offs, G, q, scales, r_cap, rpg, stream);
        case 2: return launch_tile<COL_MAJOR, W, 2>(x, M, K, offs, G, q, scales, r_cap, rpg, stream);
        case 4: return launch_tile<COL_MAJOR, W, 4>(x, M, K, offs, G, q, scales, r_cap, rpg, stream);
        default: return launch_tile<COL_MAJOR, W, 8>(x, M, K, offs, G, q, scales, r_cap, rpg, stream);
    }
}

}  // namespace

unsigned int read_wait_timeouts() {
    unsigned int n = 0;
    if (cudaMemcpyFromSymbol(&n, g_wait_timeouts, sizeof(n)) != cudaSuccess) return 0xFFFFFFFFu;
    return n;
}

unsigned int read_wait_abandoned() {
    unsigned int n = 0;
    if (cudaMemcpyFromSymbol(&n, g_wait_abandoned, sizeof(n)) != cudaSuccess) return 0xFFFFFFFFu;
    return n;
}

void set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

// Tile shapes (slab width W, cluster size CL) of the TMA tile kernel, in the order they
// are tried (each order measured against the alternatives on the per-group shapes).
// Row-major output: whole 128-byte rows on one or two CTAs, then 64-byte rows on one,
// then 128-byte rows over larger clusters; 16-column tiles would store half sectors of
// a row.  A single-CTA 128-byte-row tile, and the 8-CTA clusters, may take up to 80 KB
// (three CTAs per SM): measured at 65536 rows x 16 groups, 128-byte rows over 8 CTAs
// beat 64-byte rows by 17%; at 16640 x 32 groups one CTA per tile beat a 2-CTA cluster
// by 5%; and 8192-row groups stay in the TMA tile kernel instead of the two-pass one
// (+27%).  The 2- and 4-CTA shapes keep 48 KB: a 2-CTA 76 KB tile lost 11% to a 4-CTA
// 41 KB one at 16640 x 16 groups.
// Column-major output: 16-column slabs before clusters of more than two CTAs, but
// 32-column slabs over 4 or 8 CTAs before 16-column ones over 4 or 8: 68 -> 73% of the
// copy peak at 65536 rows x 16 groups (32-column slabs over 8 CTAs in place of
// 16-column slabs over 4).
struct TileShape {
    int w, cl, max_bytes;
};
constexpr int PG_TILE_BIG_BYTES = 80 * 1024;
constexpr TileShape PG_ROW_ORDER[] = {{64, 1, PG_TILE_BIG_BYTES},   {64, 2, PG_TILE_TARGET_BYTES},
                                      {32, 1, PG_TILE_TARGET_BYTES}, {64, 4, PG_TILE_TARGET_BYTES},
                                      {64, 8, PG_TILE_BIG_BYTES},   {32, 2, PG_TILE_TARGET_BYTES},
                                      {32, 4, PG_TILE_TARGET_BYTES}, {32, 8, PG_TILE_BIG_BYTES}};
constexpr TileShape PG_COL_ORDER[] = {{64, 1, PG_TILE_TARGET_BYTES}, {32, 1, PG_TILE_TARGET_BYTES},
                                      {32, 2, PG_TILE_TARGET_BYTES}, {16, 1, PG_TILE_TARGET_BYTES},
                                      {16, 2, PG_TILE_TARGET_BYTES}, {32, 4, PG_TILE_TARGET_BYTES},
                                      {32, 8, PG_TILE_TARGET_BYTES}, {16, 4, PG_TILE_TARGET_BYTES},
                                      {16, 8, PG_TILE_TARGET_BYTES}};

// Kernel choice from the average group size n = M / G.
//  * The TMA tile kernel: a (group, slab) tile is split among a cluster of CL CTAs
//    (1, 2, 4 or 8) and each CTA holds rows/CL + PG_TILE_SIGMAS sqrt(n)/CL + 16 rows
//    (+32 for the split at multiples of 32 rows) -- multinomial group sizes stay below
//    that; a larger group's extra rows take a slower path, never a wrong one.  The
//    first shape of the layout's order whose tile stays within that shape's bound
//    (48 KB, four or more CTAs per SM, or 80 KB for the shapes marked above).
//    Column-major output with 64-column tiles takes two neighbouring groups per CTA
//    when their joint tile fits within 48 KB too.
//  * Groups too large for eight CTAs: the two-pass streaming kernel with 512, 256 or
//    128 threads per CTA (one, two or four CTAs per SM at up to 128 registers): the most
//    CTAs per SM whose resident tiles -- each one's second pass must still find it in
//    L2 -- fit the budget, tiles estimated from the average group plus 15%.
PerGroupPlan plan_per_group(int64_t M, int64_t K, int32_t G, bool col_major, int n_sm, bool batched) {
    PerGroupPlan p{PG_PLAN_NONE, 0, 0, 0, 0};
    if (K == 0 || G == 0) return p;
    const double n = (double)((M + G - 1) / G);
    const double spread = PG_TILE_SIGMAS * std::sqrt(n);
    if (M < ((int64_t)1 << 31) - 4096) {
        const TileShape* order = col_major ? PG_COL_ORDER : PG_ROW_ORDER;
        const int n_shapes = col_major ? (int)(sizeof(PG_COL_ORDER) / sizeof(TileShape))
                                       : (int)(sizeof(PG_ROW_ORDER) / sizeof(TileShape));
        for (int i = 0; i < n_shapes; ++i) {
            const int w = order[i].w, cl = order[i].cl;
            const int r_cap = ((int)std::ceil((n + spread) / cl + (cl > 1 ? 32.0 : 0.0) + 16.0) + 15) / 16 * 16;
            if (r_cap * 2 * w > order[i].max_bytes) continue;
            if (w == 64 && col_major && cl == 1 && G >= 2 && !batched) {
                // two neighbouring groups per CTA when their tile still fits
                const int r_cap2 = ((int)std::ceil(2 * n + PG_TILE_SIGMAS * std::sqrt(2 * n) + 16.0) + 15) / 16 * 16;
                if (r_cap2 * 2 * 64 <= PG_TILE_TARGET_BYTES) return {PG_PLAN_PAIR, 64, 1, r_cap2, PG_TILE_THREADS};
            }
            return {PG_PLAN_TILE, w, cl, r_cap, PG_TILE_THREADS};
        }
    }
    const double want = std::max(1.0, n * 1.3);
    const double tile_bytes = want / 1.3 * 1.15 * PG_BIG_COLS * 2;
    const double per_sm = PG_RESIDENT_BUDGET / ((double)std::max(n_sm, 1) * tile_bytes);
    return {PG_PLAN_STREAM, PG_BIG_COLS, 1, 0, per_sm >= 4.0 ? 128 : per_sm >= 2.0 ? 256 : PG_BIG_THREADS};
}

cudaError_t launch_per_group(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, bool col_major, uint8_t* q, float* scales,
                             cudaStream_t stream, int rows_per_group) {
    const int rpg = rows_per_group;
    const PerGroupPlan p = plan_per_group(M, K, G, col_major, sm_count(), rpg > 0);
    switch (p.kind) {
        case PG_PLAN_NONE:
            return cudaSuccess;
        case PG_PLAN_PAIR:
            return launch_pair_col(x, M, K, offs, G, q, scales, p.r_cap, stream);
        case PG_PLAN_TILE:
            if (p.w == 64)
                return col_major ? launch_tile_cluster<true, 64>(p.cl, x, M, K, offs, G, q, scales, p.r_cap, rpg, stream)
                                 : launch_tile_cluster<false, 64>(p.cl, x, M, K, offs, G, q, scales, p.r_cap, rpg, stream);
            if (p.w == 32)
                return col_major ? launch_tile_cluster<true, 32>(p.cl, x, M, K, offs, G, q, scales, p.r_cap, rpg, stream)
                                 : launch_tile_cluster<false, 32>(p.cl, x, M, K, offs, G, q, scales, p.r_cap, rpg, stream);
            return launch_tile_cluster<true, 16>(p.cl, x, M, K, offs, G, q, scales, p.r_cap, rpg, stream);
        default: {
            const bool vec_col_store = ((rpg > 0 ? rpg : M) % 8) == 0;
            const dim3 grid((unsigned)((K + PG_BIG_COLS - 1) / PG_BIG_COLS), (unsigned)G);
            if (col_major)
                per_group_big_kernel<true><<<grid, p.threads, 0, stream>>>(x, M, K, offs, q, scales, vec_col_store,
                                                                           rpg);
            else
                per_group_big_kernel<false><<<grid, p.threads, 0, stream>>>(x, M, K, offs, q, scales, vec_col_store,
                                                                            rpg);
            return cudaGetLastError();
        }
    }
}

}  // namespace mxq
