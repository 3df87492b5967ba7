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
// layouts store full 32-byte sectors, and the whole group must be reduced before any
// byte is written, so the design is built around reading X from DRAM once:
//
//  * Work unit = (group g, 64-column slab): grid (n_slabs * CS, G), launched as
//    thread-block clusters of CS CTAs (CS up to 16, a non-portable cluster size, with
//    a fallback to 8).  The CS CTAs split the group's rows (in 8-row octets, aligned
//    to absolute row multiples of 8) into contiguous ranges.
//  * Pass 1: each CTA issues its whole row range at once as 16-byte cp.async copies
//    into shared memory (a warp's 32 copies = 4 rows x 128 B), so the CTA has its
//    entire share in flight; then it takes per-column maxima from shared memory.
//    Rows beyond the on-chip capacity -- only in groups far above the average size --
//    stream through registers for the maxima and are read again in pass 2 (from L2
//    when it still holds them).
//  * Reduction: shuffles over the lanes of a column, shared memory over the 8 warps,
//    then distributed shared memory over the CS CTAs of the cluster between two
//    cluster barriers (hardware barriers: no spin loops, no global scratch).
//  * Pass 2: scale, convert from shared memory, store.  Row-major: each lane writes
//    8 codes of one row (8 lanes = 64 contiguous bytes).  Column-major: each lane
//    packs the 8 rows of one column into one 8-byte store (4 lanes = 32 contiguous
//    bytes); octets cut by a group boundary fall back to byte stores.
//  * Group bounds come straight from the device offsets (no host sync): the clamp
//    rule end_g = min(max(offs[g], end_{g-1}), M) equals min(M, max(0, offs[0..g])),
//    a running maximum each CTA reduces itself.  Empty groups still write scales.
//
// CS and the staging capacity are chosen on the host from the average group size M / G.

#include <algorithm>
#include <cmath>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int PG_THREADS = 256;
constexpr int PG_COLS = 64;
constexpr int PG_TARGET_ROWS = 384;  // rows per CTA the plan aims at
constexpr int PG_MAX_CAP_OCT = 200;  // 200 octets x 1 KB = 200 KB of staged rows at most

struct GroupRange {
    int64_t start, end;    // the group's rows
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

template <bool COL_MAJOR>
__device__ __forceinline__ void store_octet(const uint4 (&d)[8], const float (&f)[8],
                                            uint8_t* __restrict__ q, int64_t oct,
                                            const GroupRange& gr, int64_t M, int64_t K,
                                            int64_t c, bool cv, bool vec_col_store) {
    if (!cv || oct >= gr.oct_hi) return;
    const int64_t r0 = oct * 8;
    if (!COL_MAJOR) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t r = r0 + i;
            if (r < gr.start || r >= gr.end) continue;
            uint2 out;
            out.x = cvt_e4m3x2(__fmul_rn(bf16_lo(d[i].x), f[0]), __fmul_rn(bf16_hi(d[i].x), f[1])) |
                    (cvt_e4m3x2(__fmul_rn(bf16_lo(d[i].y), f[2]), __fmul_rn(bf16_hi(d[i].y), f[3])) << 16);
            out.y = cvt_e4m3x2(__fmul_rn(bf16_lo(d[i].z), f[4]), __fmul_rn(bf16_hi(d[i].z), f[5])) |
                    (cvt_e4m3x2(__fmul_rn(bf16_lo(d[i].w), f[6]), __fmul_rn(bf16_hi(d[i].w), f[7])) << 16);
            *reinterpret_cast<uint2*>(q + r * K + c) = out;
        }
    } else {
        const bool full = vec_col_store && r0 >= gr.start && r0 + 8 <= gr.end;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t w = word_of(d[i], j >> 1);
                v[i] = __fmul_rn((j & 1) ? bf16_hi(w) : bf16_lo(w), f[j]);
            }
            uint2 out;
            out.x = cvt_e4m3x2(v[0], v[1]) | (cvt_e4m3x2(v[2], v[3]) << 16);
            out.y = cvt_e4m3x2(v[4], v[5]) | (cvt_e4m3x2(v[6], v[7]) << 16);
            uint8_t* dst = q + (c + j) * M + r0;
            if (full) {
                *reinterpret_cast<uint2*>(dst) = out;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int64_t r = r0 + i;
                    if (r >= gr.start && r < gr.end)
                        dst[i] = (uint8_t)(((i < 4 ? out.x : out.y) >> (8 * (i & 3))) & 0xFFu);
                }
            }
        }
    }
}

template <int CS, bool COL_MAJOR>
__global__ void __launch_bounds__(PG_THREADS, 3) per_group_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, const int32_t* __restrict__ offs,
    uint8_t* __restrict__ q, float* __restrict__ scales, int cap_oct, bool vec_col_store) {
    extern __shared__ uint4 stage[];  // [cap_oct * 8 rows][8 vectors of 8 columns]
    __shared__ uint32_t red[8][32];
    __shared__ uint32_t amax_cta[32];
    __shared__ float sc[PG_COLS];
    __shared__ int bnd[8];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid & 7, o = tid >> 3;
    const int g = blockIdx.y;
    const uint32_t rank = CS > 1 ? cluster_ctarank() : 0u;
    const int64_t k0 = (int64_t)(blockIdx.x / CS) * PG_COLS;
    const int64_t c = k0 + 8 * v;
    const bool cv = c < K;

    // ---- group bounds: running maximum of offs[0..g-1] (floored at 0), then offs[g]
    int pm = 0;
    for (int i = tid; i < g; i += PG_THREADS) pm = max(pm, offs[i]);
#pragma unroll
    for (int sh = 16; sh; sh >>= 1) pm = max(pm, __shfl_xor_sync(FULL_MASK, pm, sh));
    if (lane == 0) bnd[warp] = pm;
    __syncthreads();
    pm = bnd[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) pm = max(pm, bnd[w]);
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
    const int64_t n_oct = gr.oct_hi > gr.oct_lo ? gr.oct_hi - gr.oct_lo : 0;
    const int on_chip = (int)min(n_oct, (int64_t)cap_oct);  // octets staged in shared memory

    // ---- pass 1a: issue every staged row at once (cp.async, 16 B per copy); rows outside
    // the group (the edges of the first and last octet) are zeroed instead
    const int n_chunks = on_chip * 64;  // 8 rows x 8 vectors per octet
    for (int idx = tid; idx < n_chunks; idx += PG_THREADS) {
        const int vv = idx & 7;
        const int64_t r = gr.oct_lo * 8 + (idx >> 3);
        const int64_t col = k0 + 8 * vv;
        if (col < K && r >= gr.start && r < gr.end)
            cp_async16(&stage[idx], x + r * K + col);
        else
            stage[idx] = make_uint4(0, 0, 0, 0);
    }
    cp_async_commit();

    // ---- pass 1b: rows beyond the on-chip capacity stream through registers meanwhile
    uint32_t cm0 = 0, cm1 = 0, cm2 = 0, cm3 = 0;
    uint4 d[8];
    for (int64_t oct = gr.oct_lo + on_chip + o; oct < gr.oct_hi; oct += 32) {
        load_octet(d, x, oct, gr, K, c, cv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            cm0 = vmax2(cm0, abs2(d[i].x));
            cm1 = vmax2(cm1, abs2(d[i].y));
            cm2 = vmax2(cm2, abs2(d[i].z));
            cm3 = vmax2(cm3, abs2(d[i].w));
        }
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- pass 1c: column maxima of the staged rows
    for (int ol = o; ol < on_chip; ol += 32) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 w = stage[(ol * 8 + i) * 8 + v];
            cm0 = vmax2(cm0, abs2(w.x));
            cm1 = vmax2(cm1, abs2(w.y));
            cm2 = vmax2(cm2, abs2(w.z));
            cm3 = vmax2(cm3, abs2(w.w));
        }
    }

    // ---- reduce: lanes of a column (xor 8, 16), warps (shared), CTAs (DSMEM)
#pragma unroll
    for (int sh = 8; sh <= 16; sh <<= 1) {
        cm0 = vmax2(cm0, __shfl_xor_sync(FULL_MASK, cm0, sh));
        cm1 = vmax2(cm1, __shfl_xor_sync(FULL_MASK, cm1, sh));
        cm2 = vmax2(cm2, __shfl_xor_sync(FULL_MASK, cm2, sh));
        cm3 = vmax2(cm3, __shfl_xor_sync(FULL_MASK, cm3, sh));
    }
    if (lane < 8) {
        red[warp][lane * 4 + 0] = cm0;
        red[warp][lane * 4 + 1] = cm1;
        red[warp][lane * 4 + 2] = cm2;
        red[warp][lane * 4 + 3] = cm3;
    }
    __syncthreads();
    uint32_t m = 0;
    if (tid < 32) {
#pragma unroll
        for (int w = 0; w < 8; ++w) m = vmax2(m, red[w][tid]);
    }
    if (CS > 1) {
        if (tid < 32) amax_cta[tid] = m;
        cluster_arrive_release();
        cluster_wait_acquire();
        if (tid < 32) {
            m = 0;
#pragma unroll
            for (int r = 0; r < CS; ++r) m = vmax2(m, dsmem_ld_u32(&amax_cta[tid], (uint32_t)r));
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

    // ---- pass 2: convert and store (staged rows from shared memory, the overflow rows
    // read again from global memory)
    float f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = sc[8 * v + j];
    for (int ol = o; ol < on_chip; ol += 32) {
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = stage[(ol * 8 + i) * 8 + v];
        store_octet<COL_MAJOR>(d, f, q, gr.oct_lo + ol, gr, M, K, c, cv, vec_col_store);
    }
    for (int64_t oct = gr.oct_lo + on_chip + o; oct < gr.oct_hi; oct += 32) {
        load_octet(d, x, oct, gr, K, c, cv);
        store_octet<COL_MAJOR>(d, f, q, oct, gr, M, K, c, cv, vec_col_store);
    }
    if (CS > 1) cluster_wait_acquire();  // keep this CTA's shared memory alive for the others
}

template <int CS, bool COL_MAJOR>
static cudaError_t launch_cs(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, uint8_t* q, float* scales, int cap_oct,
                             cudaStream_t stream) {
    auto kern = per_group_kernel<CS, COL_MAJOR>;
    const size_t smem = (size_t)cap_oct * 8 * 8 * sizeof(uint4);
    // function attributes are per device; remember the largest shared-memory size set
    static int attr_smem[64] = {0};
    static bool attr_cluster[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cache = dev >= 0 && dev < 64;
    if (!cache || attr_smem[dev] < (int)smem) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (cache) attr_smem[dev] = (int)smem;
    }
    if (CS > 8 && (!cache || !attr_cluster[dev])) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        if (cache) attr_cluster[dev] = true;
    }
    const int64_t n_slabs = (K + PG_COLS - 1) / PG_COLS;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n_slabs * CS), (unsigned)G, 1);
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
    const bool vec_col_store = (M % 8) == 0;
    return cudaLaunchKernelEx(&cfg, kern, x, M, K, offs, q, scales, cap_oct, vec_col_store);
}

// Cluster size and on-chip capacity from the average group size: about PG_TARGET_ROWS
// rows per CTA (15% headroom for multinomial spread), clusters of up to `max_cs` CTAs,
// shared memory for the CTA's whole share plus one octet for a cut edge.
void per_group_plan(int64_t M, int32_t G, int max_cs, int* cs_out, int* cap_oct_out) {
    const double want = (double)((M + G - 1) / G) * 1.15;
    int cs = 1;
    while (cs < max_cs && want / cs > (double)PG_TARGET_ROWS) cs *= 2;
    const int64_t per_cta_rows = (int64_t)std::ceil(want / cs);
    int64_t cap = (per_cta_rows + 7) / 8 + 1;
    if (cap > PG_MAX_CAP_OCT) cap = PG_MAX_CAP_OCT;
    *cs_out = cs;
    *cap_oct_out = (int)cap;
}

static cudaError_t launch_with(int cs, bool col_major, const uint16_t* x, int64_t M, int64_t K,
                               const int32_t* offs, int32_t G, uint8_t* q, float* scales,
                               int cap_oct, cudaStream_t stream) {
#define MXQ_PG_CASE(N)                                                                           \
    case N:                                                                                      \
        return col_major ? launch_cs<N, true>(x, M, K, offs, G, q, scales, cap_oct, stream)     \
                         : launch_cs<N, false>(x, M, K, offs, G, q, scales, cap_oct, stream);
    switch (cs) {
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
    int cs, cap_oct;
    per_group_plan(M, G, 16, &cs, &cap_oct);
    cudaError_t e = launch_with(cs, col_major, x, M, K, offs, G, q, scales, cap_oct, stream);
    if (e != cudaSuccess && cs > 8) {
        // a 16-CTA cluster is a non-portable size; fall back to the portable maximum
        (void)cudaGetLastError();
        per_group_plan(M, G, 8, &cs, &cap_oct);
        e = launch_with(cs, col_major, x, M, K, offs, G, q, scales, cap_oct, stream);
    }
    return e;
}

}  // namespace mxq
