// per_group.cu -- per-group rowwise FP8 scaling kernel (sm_100a).
//
// Operation (torchao "[moe training] fix uncoalesced global accesses in per group
// rowwise scaling kernel", Summary and Performance): a bf16 (M, K) tensor of expert
// tokens, split into G contiguous row groups by int32 end offsets; for every
// (group g, feature k): amax over the group's rows, fp32 scale s = 448 / max(amax,
// fp32(1e-12)) (IEEE divide), and E4M3 codes q = satRNE_E4M3(fp32(x * s)), written
// row-major (M, K) -- the left operand of the scaled grouped GEMM -- or column-major.
//
// The page's Triton kernel lost its time in uncoalesced row-major stores.  Here both
// layouts store full 32-byte sectors.  The whole group must be reduced before any
// byte of it is written, so the design is built around reading X from DRAM once and
// keeping loads in flight while earlier work is converted:
//
//  * Work unit = (group g, 64-column slab), handled by a thread-block cluster of CS
//    CTAs (CS in {1, 2, 4, 8}); the CS CTAs split the group's rows (in 8-row octets,
//    aligned to absolute row multiples of 8) into contiguous shares.
//  * The kernel is persistent: cluster c takes units c, c + n_clusters, ... (units in
//    group-major, slab-minor order, so clusters running side by side read adjacent
//    columns of the same rows).
//  * Each CTA keeps a ring of NBUF shared-memory buffers and issues the rows of the
//    next NBUF-1 units as 16-byte cp.async copies (a warp's 32 copies = 4 rows x
//    128 B) before it reduces and converts the current unit, so DRAM reads of later
//    units overlap the reduction, conversion and stores of earlier ones.
//  * Reduction: per-column maxima from shared memory, shuffles over the lanes of a
//    column, shared memory over the 16 warps, then distributed shared memory over the
//    cluster.  One split cluster barrier per unit (hardware barrier.cluster arrive /
//    wait): a CTA publishes unit k+1's maxima and arrives, converts unit k, and only
//    then waits, so the exchange overlaps the conversion.  Maxima and scale slots are
//    double-buffered by unit parity.  No spin loops, no global scratch.
//  * Conversion from shared memory.  Row-major: each lane writes 8 codes of one row
//    (8 lanes = 64 contiguous bytes).  Column-major: each lane packs the 8 rows of one
//    column into one 8-byte store (4 lanes = 32 contiguous bytes); octets cut by a
//    group boundary fall back to byte stores.
//  * Rows beyond a CTA's buffer capacity (only in groups far above the average size)
//    stream through registers for the maxima and are read again for the conversion.
//  * Group bounds come from the device offsets without a host sync: the clamp rule
//    end_g = min(max(offs[g], end_{g-1}), M) equals min(M, max(0, offs[0..g])), a
//    running maximum each CTA computes once into shared memory (G <= 4096).
//
// CS, the buffer capacity and NBUF are chosen on the host from the average group size.

#include <algorithm>
#include <cmath>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int PG_THREADS = 512;
constexpr int PG_WARPS = PG_THREADS / 32;
constexpr int PG_OCT_STRIDE = PG_THREADS / 8;  // octets covered by one pass of the CTA
constexpr int PG_COLS = 64;
constexpr int PG_MAX_G = 4096;
constexpr int PG_SMEM_BUDGET = 200 * 1024;  // dynamic shared memory the plan may use

struct GroupRange {
    int64_t start, end;      // the group's rows
    int64_t oct_lo, oct_hi;  // this CTA's octets
};

__device__ __forceinline__ void load_octet(uint4 (&d)[8], const uint16_t* __restrict__ x,
                                           int64_t oct, const GroupRange& gr, int64_t K,
                                           int64_t c, bool cv) {
    const bool ov = cv && oct < gr.oct_hi;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = oct * 8 + i;
        d[i] = (ov && r >= gr.start && r < gr.end) ? ld_nc_v4(x + r * K + c) : make_uint4(0, 0, 0, 0);
    }
}

__device__ __forceinline__ uint32_t word_of(const uint4& a, int w) {
    return w == 0 ? a.x : w == 1 ? a.y : w == 2 ? a.z : a.w;
}

// Convert one octet (8 rows) x this lane's 8 columns and store it.  `r0` is the
// octet's first row; rows r0 + i with lo <= i < hi belong to the group (lo = 0, hi = 8
// for an octet fully inside it).
template <bool COL_MAJOR>
__device__ __forceinline__ void store_octet(const uint4 (&d)[8], const float (&f)[8],
                                            uint8_t* __restrict__ q, int64_t r0, int lo, int hi,
                                            int64_t M, int64_t K, int64_t c, bool vec_col_store) {
    if (!COL_MAJOR) {
        uint8_t* dst = q + r0 * K + c;
        const bool full = lo == 0 && hi == 8;
#pragma unroll
        for (int i = 0; i < 8; ++i, dst += K) {
            if (!full && (i < lo || i >= hi)) continue;
            uint2 out;
            out.x = cvt_e4m3x2(__fmul_rn(bf16_lo(d[i].x), f[0]), __fmul_rn(bf16_hi(d[i].x), f[1])) |
                    (cvt_e4m3x2(__fmul_rn(bf16_lo(d[i].y), f[2]), __fmul_rn(bf16_hi(d[i].y), f[3])) << 16);
            out.y = cvt_e4m3x2(__fmul_rn(bf16_lo(d[i].z), f[4]), __fmul_rn(bf16_hi(d[i].z), f[5])) |
                    (cvt_e4m3x2(__fmul_rn(bf16_lo(d[i].w), f[6]), __fmul_rn(bf16_hi(d[i].w), f[7])) << 16);
            *reinterpret_cast<uint2*>(dst) = out;
        }
    } else {
        const bool full = vec_col_store && lo == 0 && hi == 8;
        uint8_t* dst = q + c * M + r0;
#pragma unroll
        for (int j = 0; j < 8; ++j, dst += M) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t w = word_of(d[i], j >> 1);
                v[i] = __fmul_rn((j & 1) ? bf16_hi(w) : bf16_lo(w), f[j]);
            }
            uint2 out;
            out.x = cvt_e4m3x2(v[0], v[1]) | (cvt_e4m3x2(v[2], v[3]) << 16);
            out.y = cvt_e4m3x2(v[4], v[5]) | (cvt_e4m3x2(v[6], v[7]) << 16);
            if (full) {
                *reinterpret_cast<uint2*>(dst) = out;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i >= lo && i < hi) dst[i] = (uint8_t)(((i < 4 ? out.x : out.y) >> (8 * (i & 3))) & 0xFFu);
            }
        }
    }
}

// Rows of octet `oct` that belong to the group: [lo, hi) within 0..8.
__device__ __forceinline__ void octet_bounds(const GroupRange& gr, int64_t oct, int* lo, int* hi) {
    const int64_t r0 = oct * 8;
    *lo = (int)max((int64_t)0, min((int64_t)8, gr.start - r0));
    *hi = (int)max((int64_t)0, min((int64_t)8, gr.end - r0));
}

// Rows of group g and the octet share of CTA `rank` of the cluster.
template <int CS>
__device__ __forceinline__ GroupRange unit_range(const int* ends, int g, uint32_t rank) {
    GroupRange gr;
    gr.start = g ? ends[g - 1] : 0;
    gr.end = ends[g];
    const int64_t ob = gr.start >> 3;
    const int64_t oe = gr.end > gr.start ? (gr.end + 7) >> 3 : ob;
    const int64_t per = (oe - ob + CS - 1) / CS;
    gr.oct_lo = ob + (int64_t)rank * per;
    gr.oct_hi = min(oe, gr.oct_lo + per);
    return gr;
}

// Issue the cp.async copies of the staged part of a unit into `buf`; rows outside the
// group in the first / last octet are zeroed instead.
__device__ __forceinline__ void issue_unit(uint4* buf, const uint16_t* __restrict__ x,
                                           const GroupRange& gr, int cap_oct, int64_t K,
                                           int64_t k0, int tid) {
    const int64_t n_oct = gr.oct_hi > gr.oct_lo ? gr.oct_hi - gr.oct_lo : 0;
    const int on_chip = (int)min(n_oct, (int64_t)cap_oct);
    const int vv = tid & 7;
    const int64_t col = k0 + 8 * vv;
    const int64_t R_lo = gr.oct_lo * 8;
    const int lo_l = (int)(gr.start - R_lo) > 0 ? (int)(gr.start - R_lo) : 0;  // < 8
    const int64_t hi64 = gr.end - R_lo;
    const int n_rows = on_chip * 8;
    const int hi_l = hi64 < n_rows ? (int)hi64 : n_rows;
    int rl = tid >> 3;
    uint4* dst = buf + rl * 8 + vv;
    if (col >= K) {  // this lane's vector lies past the last column: zeros
        for (; rl < n_rows; rl += PG_THREADS / 8, dst += PG_THREADS) *dst = make_uint4(0, 0, 0, 0);
        return;
    }
    const uint16_t* src = x + (R_lo + rl) * K + col;
    const int64_t step = (int64_t)(PG_THREADS / 8) * K;
    for (; rl < n_rows; rl += PG_THREADS / 8, src += step, dst += PG_THREADS) {
        if (rl >= lo_l && rl < hi_l)
            cp_async16(dst, src);
        else
            *dst = make_uint4(0, 0, 0, 0);
    }
}

// Per-column maxima (4 words = 8 columns as u16x2) of the staged rows of one unit,
// plus its overflow rows streamed from global memory.
__device__ __forceinline__ void unit_maxima(const uint4* buf, const uint16_t* __restrict__ x,
                                            const GroupRange& gr, int on_chip, int64_t K, int64_t c,
                                            bool cv, int o, int v, uint32_t (&cm)[4]) {
    cm[0] = cm[1] = cm[2] = cm[3] = 0;
    for (int ol = o; ol < on_chip; ol += PG_OCT_STRIDE) {
        const uint4* src = buf + ol * 64 + v;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 w = src[i * 8];
            cm[0] = amax2(cm[0], w.x);
            cm[1] = amax2(cm[1], w.y);
            cm[2] = amax2(cm[2], w.z);
            cm[3] = amax2(cm[3], w.w);
        }
    }
    uint4 d[8];
    for (int64_t oct = gr.oct_lo + on_chip + o; oct < gr.oct_hi; oct += PG_OCT_STRIDE) {
        load_octet(d, x, oct, gr, K, c, cv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            cm[0] = amax2(cm[0], d[i].x);
            cm[1] = amax2(cm[1], d[i].y);
            cm[2] = amax2(cm[2], d[i].z);
            cm[3] = amax2(cm[3], d[i].w);
        }
    }
}

// Unit index -> (group, slab), walked incrementally (no 64-bit division per unit).
struct UnitCursor {
    int64_t u;
    int g, slab;
};

__device__ __forceinline__ void cursor_advance(UnitCursor& cu, int step_g, int step_s, int n_slabs,
                                               int64_t step_u) {
    cu.u += step_u;
    cu.g += step_g;
    cu.slab += step_s;
    if (cu.slab >= n_slabs) {
        cu.slab -= n_slabs;
        cu.g += 1;
    }
}

// Schedule of one CTA (cluster rank `rank`), units k = 0, 1, ... of its cluster:
//   prologue: issue units 0..nbuf-2; maxima(0); publish; arrive
//   iteration k: wait(k) -> cluster maxima of unit k -> scales(k) -> CTA barrier
//                -> issue unit k+nbuf-1 -> copies of unit k+1 landed -> maxima(k+1)
//                -> publish; arrive -> convert + store unit k
// The split cluster barrier (arrive ... wait) brackets the conversion of unit k, so the
// exchange of unit k+1's maxima and the release of earlier stores overlap real work.
// Scales and maxima slots are double-buffered by unit parity.
template <int CS, bool COL_MAJOR>
__global__ void __launch_bounds__(PG_THREADS, 1) per_group_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, const int32_t* __restrict__ offs, int G,
    uint8_t* __restrict__ q, float* __restrict__ scales, int cap_oct, int nbuf, int64_t n_units,
    int n_slabs, bool vec_col_store) {
    extern __shared__ uint4 dyn[];  // nbuf x [cap_oct * 8 rows][8 vectors], then ends[G]
    int* ends = reinterpret_cast<int*>(dyn + (size_t)nbuf * cap_oct * 64);
    __shared__ uint32_t red[PG_WARPS][32];
    __shared__ uint32_t amax_cta[2][32];
    __shared__ float sc[2][PG_COLS];
    __shared__ int scan[PG_WARPS];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid & 7, o = tid >> 3;
    const uint32_t rank = CS > 1 ? cluster_ctarank() : 0u;
    const int64_t cid = blockIdx.x / CS;
    const int64_t n_clusters = gridDim.x / CS;
    const int step_g = (int)(n_clusters / n_slabs), step_s = (int)(n_clusters % n_slabs);

    // ---- group ends: ends[g] = min(M, max(0, offs[0..g])), a block-wide prefix max
    {
        const int per = (G + PG_THREADS - 1) / PG_THREADS;  // <= 8 for G <= 4096
        const int base = tid * per;
        int run = 0;
        for (int j = 0; j < per; ++j) {
            const int i = base + j;
            if (i < G) run = max(run, offs[i]);
        }
        int incl = run;  // inclusive prefix max over the lanes of the warp
#pragma unroll
        for (int sh = 1; sh < 32; sh <<= 1) {
            const int t = __shfl_up_sync(FULL_MASK, incl, sh);
            if (lane >= sh) incl = max(incl, t);
        }
        if (lane == 31) scan[warp] = incl;
        __syncthreads();
        int before = 0;  // max over all earlier threads (floored at 0)
        for (int w = 0; w < warp; ++w) before = max(before, scan[w]);
        const int prev_lane = __shfl_up_sync(FULL_MASK, incl, 1);
        if (lane > 0) before = max(before, prev_lane);
        int r2 = before;
        for (int j = 0; j < per; ++j) {
            const int i = base + j;
            if (i < G) {
                r2 = max(r2, offs[i]);
                ends[i] = (int)min((int64_t)r2, M);
            }
        }
        __syncthreads();
    }
    if (cid >= n_units) return;  // cluster-uniform: no unit for this cluster, no barrier used

    // cursors: `cur` = unit k, `nxt` = unit k+1, `iss` = next unit to issue
    UnitCursor cur{cid, (int)(cid / n_slabs), (int)(cid % n_slabs)};
    UnitCursor iss = cur;
    for (int p = 0; p < nbuf - 1; ++p) {
        if (iss.u < n_units)
            issue_unit(dyn + (size_t)p * cap_oct * 64, x, unit_range<CS>(ends, iss.g, rank), cap_oct, K,
                       (int64_t)iss.slab * PG_COLS, tid);
        cp_async_commit();
        cursor_advance(iss, step_g, step_s, n_slabs, n_clusters);
    }

    // maxima of unit 0, published for the cluster
    {
        const int64_t c = (int64_t)cur.slab * PG_COLS + 8 * v;
        const GroupRange gr = unit_range<CS>(ends, cur.g, rank);
        const int64_t n_oct = gr.oct_hi > gr.oct_lo ? gr.oct_hi - gr.oct_lo : 0;
        cp_async_wait_pending(nbuf - 2);
        __syncthreads();
        uint32_t cm[4];
        unit_maxima(dyn, x, gr, (int)min(n_oct, (int64_t)cap_oct), K, c, c < K, o, v, cm);
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
#pragma unroll
            for (int w = 0; w < PG_WARPS; ++w) m = amax2(m, red[w][tid]);
            m = mag2(m);
            amax_cta[0][tid] = m;
        }
        if (CS > 1) cluster_arrive_release();
    }

    int it = 0;
    for (; cur.u < n_units; ++it) {
        const int par = it & 1;
        // ---- cluster maxima and scales of unit `it`
        if (CS > 1) cluster_wait_acquire();
        if (tid < 32) {
            uint32_t m = 0;
            if (CS > 1) {
#pragma unroll
                for (int r = 0; r < CS; ++r) m = amax2(m, dsmem_ld_u32(&amax_cta[par][tid], (uint32_t)r));
                m = mag2(m);
            } else {
                m = amax_cta[par][tid];
            }
            // word tid = columns 8*(tid/4) + 2*(tid%4) + {0, 1} of the slab
            const int col0 = 8 * (tid >> 2) + 2 * (tid & 3);
            const int64_t k0 = (int64_t)cur.slab * PG_COLS;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t ab = h ? (m >> 16) : (m & 0xFFFFu);
                const float s = ab >= 0x7F80u ? __uint_as_float(0x7FC00000u)
                                              : __fdiv_rn(448.0f, fmaxf(__uint_as_float(ab << 16), 1e-12f));
                sc[par][col0 + h] = s;
                if (rank == 0 && k0 + col0 + h < K) scales[(int64_t)cur.g * K + k0 + col0 + h] = s;
            }
        }
        __syncthreads();  // scales visible; unit it-1 fully converted (its buffer is free)

        // ---- keep nbuf-1 units in flight
        if (iss.u < n_units)
            issue_unit(dyn + (size_t)((it + nbuf - 1) % nbuf) * cap_oct * 64, x,
                       unit_range<CS>(ends, iss.g, rank), cap_oct, K, (int64_t)iss.slab * PG_COLS, tid);
        cp_async_commit();
        cursor_advance(iss, step_g, step_s, n_slabs, n_clusters);

        // ---- maxima of unit it+1, published before converting unit it
        UnitCursor nxt = cur;
        cursor_advance(nxt, step_g, step_s, n_slabs, n_clusters);
        if (nxt.u < n_units) {
            const int64_t c = (int64_t)nxt.slab * PG_COLS + 8 * v;
            const GroupRange gr = unit_range<CS>(ends, nxt.g, rank);
            const int64_t n_oct = gr.oct_hi > gr.oct_lo ? gr.oct_hi - gr.oct_lo : 0;
            cp_async_wait_pending(nbuf - 2);  // unit it+1's copies have landed
            __syncthreads();
            uint32_t cm[4];
            unit_maxima(dyn + (size_t)((it + 1) % nbuf) * cap_oct * 64, x, gr,
                        (int)min(n_oct, (int64_t)cap_oct), K, c, c < K, o, v, cm);
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
#pragma unroll
                for (int w = 0; w < PG_WARPS; ++w) m = amax2(m, red[w][tid]);
            m = mag2(m);
                amax_cta[par ^ 1][tid] = m;
            }
        }
        if (CS > 1) cluster_arrive_release();
        // (CS == 1: the next iteration's reader of amax_cta is the thread that wrote it)

        // ---- convert and store unit it
        {
            const int64_t c = (int64_t)cur.slab * PG_COLS + 8 * v;
            const bool cv = c < K;
            const GroupRange gr = unit_range<CS>(ends, cur.g, rank);
            const int64_t n_oct = gr.oct_hi > gr.oct_lo ? gr.oct_hi - gr.oct_lo : 0;
            const int on_chip = (int)min(n_oct, (int64_t)cap_oct);
            const uint4* buf = dyn + (size_t)(it % nbuf) * cap_oct * 64;
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] = sc[par][8 * v + j];
            if (cv) {
                uint4 d[8];
                for (int ol = o; ol < on_chip; ol += PG_OCT_STRIDE) {
                    const int64_t oct = gr.oct_lo + ol;
                    int lo, hi;
                    octet_bounds(gr, oct, &lo, &hi);
                    const uint4* src = buf + ol * 64 + v;
#pragma unroll
                    for (int i = 0; i < 8; ++i) d[i] = src[i * 8];
                    store_octet<COL_MAJOR>(d, f, q, oct * 8, lo, hi, M, K, c, vec_col_store);
                }
                for (int64_t oct = gr.oct_lo + on_chip + o; oct < gr.oct_hi; oct += PG_OCT_STRIDE) {
                    int lo, hi;
                    octet_bounds(gr, oct, &lo, &hi);
                    load_octet(d, x, oct, gr, K, c, cv);
                    store_octet<COL_MAJOR>(d, f, q, oct * 8, lo, hi, M, K, c, vec_col_store);
                }
            }
        }
        cur = nxt;
    }
    cp_async_wait_all();
    if (CS > 1) cluster_wait_acquire();  // matches the last arrive; then nobody reads our slots
}

// ---- host side ---------------------------------------------------------------------------

struct PgPlan {
    int cs, cap_oct, nbuf;
};

// From the average group size: clusters of up to 8 CTAs with at most ~768 rows each per
// unit (15% headroom for multinomial spread, one extra octet for a cut edge), and as
// many buffers as fit the shared-memory budget to keep >= ~96 KB of reads in flight.
static PgPlan per_group_plan(int64_t M, int32_t G) {
    const double want = (double)((M + G - 1) / G) * 1.15;
    PgPlan p;
    p.cs = 1;
    while (p.cs < 8 && want / p.cs > 768.0) p.cs *= 2;
    int64_t cap = (int64_t)std::ceil(want / p.cs / 8.0) + 1;
    const int64_t max_cap = (PG_SMEM_BUDGET - (int64_t)G * 4) / 2 / 1024;  // two buffers at least
    cap = std::max<int64_t>(1, std::min(cap, max_cap));
    p.cap_oct = (int)cap;
    const int64_t unit_bytes = cap * 1024;
    int nbuf = (int)std::max<int64_t>(2, (96 * 1024 + unit_bytes - 1) / unit_bytes + 1);
    nbuf = std::min(nbuf, 8);
    while (nbuf > 2 && nbuf * unit_bytes + (int64_t)G * 4 > PG_SMEM_BUDGET) --nbuf;
    p.nbuf = nbuf;
    return p;
}

template <int CS, bool COL_MAJOR>
static cudaError_t launch_cs(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, uint8_t* q, float* scales, const PgPlan& plan,
                             cudaStream_t stream) {
    auto kern = per_group_kernel<CS, COL_MAJOR>;
    const size_t smem = (size_t)plan.nbuf * plan.cap_oct * 1024 + (size_t)G * 4;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cache = dev >= 0 && dev < 64;
    static int attr_smem[64] = {0};
    if (!cache || attr_smem[dev] < (int)smem) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (cache) attr_smem[dev] = (int)smem;
    }
    const int64_t n_slabs = (K + PG_COLS - 1) / PG_COLS;
    const int64_t n_units = n_slabs * G;

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(PG_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = CS > 1 ? 1 : 0;

    // persistent grid: as many clusters as can be resident at once (cached per device
    // and shared-memory size), never more than there are units
    static int occ_smem[64] = {0}, occ_clusters[64] = {0};
    int max_clusters = 0;
    if (cache && occ_smem[dev] == (int)smem && occ_clusters[dev] > 0) {
        max_clusters = occ_clusters[dev];
    } else {
        cfg.gridDim = dim3(CS, 1, 1);
        if (cudaOccupancyMaxActiveClusters(&max_clusters, (const void*)kern, &cfg) != cudaSuccess ||
            max_clusters <= 0) {
            (void)cudaGetLastError();
            max_clusters = std::max(1, sm_count() / CS);
        }
        if (cache) {
            occ_smem[dev] = (int)smem;
            occ_clusters[dev] = max_clusters;
        }
    }
    const int64_t n_clusters = std::min<int64_t>(n_units, max_clusters);
    cfg.gridDim = dim3((unsigned)(n_clusters * CS), 1, 1);
    const bool vec_col_store = (M % 8) == 0;
    return cudaLaunchKernelEx(&cfg, kern, x, M, K, offs, (int)G, q, scales, plan.cap_oct, plan.nbuf,
                              n_units, (int)n_slabs, vec_col_store);
}

cudaError_t launch_per_group(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, bool col_major, uint8_t* q, float* scales,
                             cudaStream_t stream) {
    if (K == 0 || G == 0) return cudaSuccess;
    if (G > PG_MAX_G) return cudaErrorInvalidValue;
    const PgPlan plan = per_group_plan(M, G);
#define MXQ_PG_CASE(N)                                                                        \
    case N:                                                                                   \
        return col_major ? launch_cs<N, true>(x, M, K, offs, G, q, scales, plan, stream)     \
                         : launch_cs<N, false>(x, M, K, offs, G, q, scales, plan, stream);
    switch (plan.cs) {
        MXQ_PG_CASE(1)
        MXQ_PG_CASE(2)
        MXQ_PG_CASE(4)
        MXQ_PG_CASE(8)
        default:
            return cudaErrorInvalidValue;
    }
#undef MXQ_PG_CASE
}

}  // namespace mxq
