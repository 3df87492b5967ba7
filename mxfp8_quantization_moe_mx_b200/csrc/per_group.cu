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
// byte of it is written; the design reads X from DRAM once and keeps it in registers:
//
//  * Work unit = (group g, 64-column slab), handled by a thread-block cluster of CS
//    CTAs (CS up to 16, a non-portable cluster size, falling back to 8).  The CS CTAs
//    split the group's rows in 8-row octets (aligned to absolute row multiples of 8).
//  * A CTA has one thread per row of its share: thread (o = tid/8, v = tid%8) holds
//    octet o (rows 8o..8o+7) x columns 8v..8v+7 of the slab as eight 16-byte loads
//    issued all at once (a warp's load = 4 rows x 128 B).  The host sizes the CTA (a
//    multiple of 32 threads) and CS from the average group size, so the whole tile
//    sits in registers across the cluster, with several CTAs per SM to hide latency.
//  * Reduction: packed bf16 magnitude maxima in registers, shuffles over the lanes of
//    a column, shared memory over the warps, then distributed shared memory over the
//    cluster between two hardware cluster barriers (no spin loops, no global scratch).
//  * Conversion straight from registers.  Row-major: each lane writes 8 codes of one
//    row (8 lanes = 64 contiguous bytes).  Column-major: each lane packs the 8 rows of
//    one column into one 8-byte store (4 lanes = 32 contiguous bytes); octets cut by a
//    group boundary fall back to byte stores.
//  * Rows beyond the cluster's capacity (only in groups far above the average size)
//    are streamed twice: once for the maxima, once for the conversion.
//  * Group bounds come from the device offsets without a host sync: the clamp rule
//    end_g = min(max(offs[g], end_{g-1}), M) equals min(M, max(0, offs[0..g])), a
//    running maximum each CTA reduces itself.

#include <algorithm>
#include <cmath>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int PG_COLS = 64;
constexpr int PG_MAX_THREADS = 512;
constexpr int PG_MAX_G = 4096;

struct GroupRange {
    int64_t start, end;      // the group's rows
    int64_t oct_lo, oct_hi;  // this CTA's octets
};

// Rows r0 + i (i in [lo, hi)) of an octet belong to the group.
__device__ __forceinline__ void octet_bounds(const GroupRange& gr, int64_t r0, int* lo, int* hi) {
    *lo = (int)max((int64_t)0, min((int64_t)8, gr.start - r0));
    *hi = (int)max((int64_t)0, min((int64_t)8, gr.end - r0));
}

__device__ __forceinline__ void load_octet(uint4 (&d)[8], const uint16_t* __restrict__ x, int64_t r0,
                                           int lo, int hi, int64_t K, int64_t c) {
    const uint16_t* src = x + r0 * K + c;
#pragma unroll
    for (int i = 0; i < 8; ++i, src += K) d[i] = (i >= lo && i < hi) ? ld_nc_v4(src) : make_uint4(0, 0, 0, 0);
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

// Convert one octet x this lane's 8 columns (scales f[0..7]) and store it.
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
            float p[8];
            fmul2(bf16_lo(d[i].x), bf16_hi(d[i].x), f[0], f[1], p[0], p[1]);
            fmul2(bf16_lo(d[i].y), bf16_hi(d[i].y), f[2], f[3], p[2], p[3]);
            fmul2(bf16_lo(d[i].z), bf16_hi(d[i].z), f[4], f[5], p[4], p[5]);
            fmul2(bf16_lo(d[i].w), bf16_hi(d[i].w), f[6], f[7], p[6], p[7]);
            uint2 out;
            out.x = cvt4_e4m3(p[0], p[1], p[2], p[3]);
            out.y = cvt4_e4m3(p[4], p[5], p[6], p[7]);
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
                *reinterpret_cast<uint2*>(dst) = out;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i >= lo && i < hi) dst[i] = (uint8_t)(((i < 4 ? out.x : out.y) >> (8 * (i & 3))) & 0xFFu);
            }
        }
    }
}

template <int CS, bool COL_MAJOR>
__global__ void __launch_bounds__(PG_MAX_THREADS) per_group_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, const int32_t* __restrict__ offs,
    uint8_t* __restrict__ q, float* __restrict__ scales, bool vec_col_store) {
    __shared__ uint32_t red[PG_MAX_THREADS / 32][32];
    __shared__ uint32_t amax_cta[32];
    __shared__ float sc[PG_COLS];
    __shared__ int bnd[PG_MAX_THREADS / 32];

    const int T = blockDim.x, n_warps = T >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid & 7, o = tid >> 3, oct_per_cta = T >> 3;
    const int g = blockIdx.y;
    const uint32_t rank = CS > 1 ? cluster_ctarank() : 0u;
    const int64_t k0 = (int64_t)(blockIdx.x / CS) * PG_COLS;
    const int64_t c = k0 + 8 * v;
    const bool cv = c < K;

    // ---- group bounds: running maximum of offs[0..g-1] (floored at 0), then offs[g]
    int pm = 0;
    for (int i = tid; i < g; i += T) pm = max(pm, offs[i]);
#pragma unroll
    for (int sh = 16; sh; sh >>= 1) pm = max(pm, __shfl_xor_sync(FULL_MASK, pm, sh));
    if (lane == 0) bnd[warp] = pm;
    __syncthreads();
    pm = 0;
    for (int w = 0; w < n_warps; ++w) pm = max(pm, bnd[w]);
    GroupRange gr;
    gr.start = min((int64_t)pm, M);
    gr.end = min((int64_t)max(pm, offs[g]), M);
    {
        const int64_t ob = gr.start >> 3;
        const int64_t oe = gr.end > gr.start ? (gr.end + 7) >> 3 : ob;
        const int64_t per = (oe - ob + CS - 1) / CS;
        gr.oct_lo = ob + (int64_t)rank * per;
        gr.oct_hi = min(oe, gr.oct_lo + per);
    }

    // ---- the resident octet: all eight row loads in flight at once
    const int64_t oct = gr.oct_lo + o;
    const bool have = cv && oct < gr.oct_hi;
    int lo = 0, hi = 0;
    if (have) octet_bounds(gr, oct * 8, &lo, &hi);
    uint4 d[8];
    load_octet(d, x, oct * 8, lo, hi, K, c);  // lo == hi == 0 loads nothing

    // ---- maxima: the resident octet, then any octets beyond the CTA's capacity
    uint32_t cm[4] = {0, 0, 0, 0};
    amax_octet(d, cm);
    if (cv) {  // one row at a time: the resident octet stays live in d
        for (int64_t ox = gr.oct_lo + oct_per_cta + o; ox < gr.oct_hi; ox += oct_per_cta) {
            int l2, h2;
            octet_bounds(gr, ox * 8, &l2, &h2);
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

    // ---- reduce: lanes of a column (xor 8, 16), warps (shared), CTAs (DSMEM)
#pragma unroll
    for (int sh = 8; sh <= 16; sh <<= 1)
#pragma unroll
        for (int w = 0; w < 4; ++w) cm[w] = amax2(cm[w], __shfl_xor_sync(FULL_MASK, cm[w], sh));
    if (lane < 8)
#pragma unroll
        for (int w = 0; w < 4; ++w) red[warp][lane * 4 + w] = cm[w];
    __syncthreads();
    uint32_t m = 0;
    if (tid < 32) {
        for (int w = 0; w < n_warps; ++w) m = amax2(m, red[w][tid]);
        m = mag2(m);
    }
    if (CS > 1) {
        if (tid < 32) amax_cta[tid] = m;
        cluster_arrive_release();
        cluster_wait_acquire();
        if (tid < 32) {
#pragma unroll
            for (int r = 0; r < CS; ++r) m = amax2(m, dsmem_ld_u32(&amax_cta[tid], (uint32_t)r));
            m = mag2(m);
        }
        cluster_arrive_release();  // done reading the other CTAs' shared memory
    }
    if (tid < 32) {
        // word tid = columns 8*(tid/4) + 2*(tid%4) + {0, 1} of the slab
        const int col0 = 8 * (tid >> 2) + 2 * (tid & 3);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t ab = h ? (m >> 16) : (m & 0xFFFFu);
            const float s = ab >= 0x7F80u ? __uint_as_float(0x7FC00000u)
                                          : __fdiv_rn(448.0f, fmaxf(__uint_as_float(ab << 16), 1e-12f));
            sc[col0 + h] = s;
            if (rank == 0 && k0 + col0 + h < K) scales[(int64_t)g * K + k0 + col0 + h] = s;
        }
    }
    __syncthreads();

    // ---- convert and store
    if (cv) {
        float f[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = sc[8 * v + j];
        if (have) store_octet<COL_MAJOR>(d, f, q, oct * 8, lo, hi, M, K, c, vec_col_store);
        for (int64_t ox = gr.oct_lo + oct_per_cta + o; ox < gr.oct_hi; ox += oct_per_cta) {
            int l2, h2;
            octet_bounds(gr, ox * 8, &l2, &h2);
            load_octet(d, x, ox * 8, l2, h2, K, c);
            store_octet<COL_MAJOR>(d, f, q, ox * 8, l2, h2, M, K, c, vec_col_store);
        }
    }
    if (CS > 1) cluster_wait_acquire();  // keep this CTA's shared memory alive for the others
}

// ---- host side ---------------------------------------------------------------------------

struct PgPlan {
    int cs, threads;
};

// One thread per row of a CTA's share.  From the average group size (15% headroom for
// multinomial spread), the smallest cluster (up to max_cs) whose CTAs need at most 384
// threads each; beyond that the CTAs grow up to 512 threads and the rest of a group
// streams twice.
static PgPlan per_group_plan(int64_t M, int32_t G, int max_cs) {
    const double want = std::max(1.0, (double)((M + G - 1) / G) * 1.15);
    PgPlan p;
    p.cs = 1;
    while (p.cs < max_cs && want / p.cs > 384.0) p.cs *= 2;
    int64_t t = (int64_t)std::ceil(want / p.cs);
    t = (t + 31) / 32 * 32;
    p.threads = (int)std::min<int64_t>(std::max<int64_t>(t, 32), PG_MAX_THREADS);
    return p;
}

template <int CS, bool COL_MAJOR>
static cudaError_t launch_cs(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, uint8_t* q, float* scales, int threads, cudaStream_t stream) {
    auto kern = per_group_kernel<CS, COL_MAJOR>;
    if (CS > 8) {
        static bool attr_set[64] = {false};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 64 || !attr_set[dev]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) attr_set[dev] = true;
        }
    }
    const int64_t n_slabs = (K + PG_COLS - 1) / PG_COLS;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n_slabs * CS), (unsigned)G, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = CS > 1 ? 1 : 0;
    const bool vec_col_store = (M % 8) == 0;
    return cudaLaunchKernelEx(&cfg, kern, x, M, K, offs, q, scales, vec_col_store);
}

static cudaError_t launch_plan(const PgPlan& p, bool col_major, const uint16_t* x, int64_t M, int64_t K,
                               const int32_t* offs, int32_t G, uint8_t* q, float* scales,
                               cudaStream_t stream) {
#define MXQ_PG_CASE(N)                                                                          \
    case N:                                                                                     \
        return col_major ? launch_cs<N, true>(x, M, K, offs, G, q, scales, p.threads, stream)  \
                         : launch_cs<N, false>(x, M, K, offs, G, q, scales, p.threads, stream);
    switch (p.cs) {
        MXQ_PG_CASE(1)
        MXQ_PG_CASE(2)
        MXQ_PG_CASE(4)
        MXQ_PG_CASE(8)
        MXQ_PG_CASE(16)
        default:
            return cudaErrorInvalidValue;
    }
#undef MXQ_PG_CASE
}

cudaError_t launch_per_group(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, bool col_major, uint8_t* q, float* scales,
                             cudaStream_t stream) {
    if (K == 0 || G == 0) return cudaSuccess;
    if (G > PG_MAX_G) return cudaErrorInvalidValue;
    PgPlan p = per_group_plan(M, G, 16);
    cudaError_t e = launch_plan(p, col_major, x, M, K, offs, G, q, scales, stream);
    if (e != cudaSuccess && p.cs > 8) {
        // a 16-CTA cluster is a non-portable size; retry with the portable maximum
        (void)cudaGetLastError();
        p = per_group_plan(M, G, 8);
        e = launch_plan(p, col_major, x, M, K, offs, G, q, scales, stream);
    }
    return e;
}

}  // namespace mxq
