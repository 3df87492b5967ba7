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
// layouts store full 32-byte sectors.  The hard part is the dependency: a group's
// whole column must be reduced before any of its bytes is written, and groups run
// from a few rows to tens of thousands.  The design:
//
//  * Tile = (group g, 64-column slab); a tile is cut into chunks of up to T rows (T =
//    the CTA size, a multiple of 32; whole 8-row octets aligned to absolute row
//    multiples of 8).  Chunk i of the work list = (group, slab, chunk), in group-major,
//    slab, chunk order; the list is built on the device from the offsets (no host
//    sync) and every CTA derives it into shared memory.
//  * A persistent grid of co-resident CTAs (cooperative launch) walks the list in
//    rounds: CTA b takes items b, b + N, b + 2N, ...  In round k a CTA
//      1. prefetches the rows of item k into L2 (cp.async.bulk.prefetch, one 128-byte
//         row segment per thread),
//      2. converts item k-1: waits until every chunk of that tile has published its
//         maxima (a counter in the workspace -- normally already complete, because
//         the tile's chunks ran in the previous round on neighbouring CTAs), turns
//         the tile maxima into scales, reads the rows again (they are still in L2)
//         and stores E4M3 codes,
//      3. reduces item k: thread (o = tid/8, v = tid%8) loads octet o x columns
//         8v..8v+7 (eight 16-byte loads, a warp load = 4 rows x 128 B), packed bf16
//         magnitude maxima, shuffles and shared memory across the CTA, then atomicMax
//         per column into the tile's slot and one counter increment.
//    DRAM sees each input byte once (the prefetch) and each output byte once; the
//    second read of a chunk comes from L2 one round later.
//  * The wait on a tile counter is bounded (about half a second); if it ever runs out
//    the kernel records the failure in a device error word (mxq_device_error), later
//    waits give up at once, and the kernel finishes.
//    Deadlock cannot arise: all CTAs are resident (cooperative launch), a tile has at
//    most N chunks (larger chunks for huge groups), and a CTA only waits for chunks
//    of earlier rounds or of lower-numbered CTAs in the same round.
//  * The workspace (per tile: 64 column maxima + 1 counter, 260 bytes) is cleared on
//    the caller's stream before the launch (cudaMemsetAsync, no allocation).
//  * Group bounds come straight from the device offsets: the clamp rule
//    end_g = min(max(offs[g], end_{g-1}), M) equals min(M, max(0, offs[0..g])).

#include <algorithm>
#include <cmath>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int PG_COLS = 64;
constexpr int PG_MAX_THREADS = 256;
constexpr int PG_MAX_G = 4096;
constexpr uint32_t PG_SPIN_LIMIT = 1u << 22;  // x ~128 ns sleep ~ 0.5 s

__device__ unsigned int g_pg_error = 0;  // bit 0: a tile wait gave up

// One work item: rows [start, end) of the group, this chunk's octets, tile id.
struct Chunk {
    int64_t start, end, oct_lo, oct_hi;
    int64_t tile;
    int g, s, r, n_chunks;
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Rows r0 + i (i in [lo, hi)) of an octet belong to the group.
__device__ __forceinline__ void octet_bounds(const Chunk& ch, int64_t r0, int* lo, int* hi) {
    *lo = (int)max((int64_t)0, min((int64_t)8, ch.start - r0));
    *hi = (int)max((int64_t)0, min((int64_t)8, ch.end - r0));
}

__device__ __forceinline__ void load_octet(uint4 (&d)[8], const uint16_t* __restrict__ x, int64_t r0,
                                           int lo, int hi, int64_t K, int64_t c) {
    const uint16_t* src = x + r0 * K + c;
#pragma unroll
    for (int i = 0; i < 8; ++i, src += K) d[i] = (i >= lo && i < hi) ? ld_nc_v4(src) : make_uint4(0, 0, 0, 0);
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

// Item index -> chunk (binary search over the per-group item prefix).
__device__ __forceinline__ Chunk decode_item(int64_t i, const int* ends, const int64_t* base,
                                             const int* octs_per_chunk, int G, int n_slabs) {
    int lo = 0, hi = G - 1;  // largest g with base[g] <= i
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (base[mid] <= i) lo = mid;
        else hi = mid - 1;
    }
    Chunk ch;
    ch.g = lo;
    ch.start = lo ? ends[lo - 1] : 0;
    ch.end = ends[lo];
    const int64_t ob = ch.start >> 3;
    const int64_t oe = ch.end > ch.start ? (ch.end + 7) >> 3 : ob;
    const int opc = octs_per_chunk[lo];
    ch.n_chunks = (int)max((int64_t)1, (oe - ob + opc - 1) / opc);
    const int64_t local = i - base[lo];
    ch.s = (int)(local / ch.n_chunks);
    ch.r = (int)(local - (int64_t)ch.s * ch.n_chunks);
    ch.oct_lo = ob + (int64_t)ch.r * opc;
    ch.oct_hi = min(oe, ch.oct_lo + opc);
    ch.tile = (int64_t)ch.g * n_slabs + ch.s;
    return ch;
}

template <bool COL_MAJOR>
__global__ void __launch_bounds__(PG_MAX_THREADS) per_group_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, const int32_t* __restrict__ offs, int G,
    uint8_t* __restrict__ q, float* __restrict__ scales, uint32_t* __restrict__ ws_amax,
    uint32_t* __restrict__ ws_count, int n_slabs, bool vec_col_store) {
    extern __shared__ int64_t dyn64[];  // base[G + 1] (int64), then ends[G], opc[G] (int)
    int64_t* base = dyn64;
    int* ends = reinterpret_cast<int*>(base + G + 1);
    int* opc = ends + G;
    __shared__ uint32_t red[PG_MAX_THREADS / 32][32];
    __shared__ float sc[PG_COLS];
    __shared__ int64_t scan64[PG_MAX_THREADS / 32];
    __shared__ int scan32[PG_MAX_THREADS / 32];

    const int T = blockDim.x, n_warps = T >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int v = tid & 7, o = tid >> 3, oct_per_cta = T >> 3;
    const int64_t N = gridDim.x;

    // ---- per-group tables: ends (prefix max of the offsets), octets per chunk (a
    // tile may have at most N chunks, so huge groups get bigger chunks), item prefix
    {
        const int per = (G + T - 1) / T;
        const int first = tid * per;
        int run = 0;
        for (int j = 0; j < per; ++j)
            if (first + j < G) run = max(run, offs[first + j]);
        int incl = run;
#pragma unroll
        for (int sh = 1; sh < 32; sh <<= 1) {
            const int t = __shfl_up_sync(FULL_MASK, incl, sh);
            if (lane >= sh) incl = max(incl, t);
        }
        if (lane == 31) scan32[warp] = incl;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before = max(before, scan32[w]);
        const int prev_lane = __shfl_up_sync(FULL_MASK, incl, 1);
        if (lane > 0) before = max(before, prev_lane);
        int r2 = before;
        for (int j = 0; j < per; ++j)
            if (first + j < G) {
                r2 = max(r2, offs[first + j]);
                ends[first + j] = (int)min((int64_t)r2, M);
            }
        __syncthreads();
        // items per group and their exclusive prefix
        int64_t cnt = 0;
        for (int j = 0; j < per; ++j) {
            const int g = first + j;
            if (g >= G) break;
            const int64_t st = g ? ends[g - 1] : 0, en = ends[g];
            const int64_t ob = st >> 3, oe = en > st ? (en + 7) >> 3 : ob;
            const int64_t n_oct = oe - ob;
            int64_t o_pc = oct_per_cta;
            if ((n_oct + o_pc - 1) / o_pc > N) o_pc = (n_oct + N - 1) / N;
            opc[g] = (int)o_pc;
            const int64_t n_ch = max((int64_t)1, (n_oct + o_pc - 1) / o_pc);
            base[g] = n_ch * n_slabs;  // items of group g (turned into a prefix below)
            cnt += n_ch * n_slabs;
        }
        int64_t incl64 = cnt;
#pragma unroll
        for (int sh = 1; sh < 32; sh <<= 1) {
            const int64_t t = __shfl_up_sync(FULL_MASK, incl64, sh);
            if (lane >= sh) incl64 += t;
        }
        if (lane == 31) scan64[warp] = incl64;
        __syncthreads();
        int64_t excl = incl64 - cnt;
        for (int w = 0; w < warp; ++w) excl += scan64[w];
        for (int j = 0; j < per; ++j) {
            const int g = first + j;
            if (g >= G) break;
            const int64_t items = base[g];
            base[g] = excl;
            excl += items;
        }
        if (tid == T - 1) base[G] = excl;  // the last thread's running sum is the total
        __syncthreads();
    }
    const int64_t total = base[G];

    Chunk prev;
    bool have_prev = false;
    for (int64_t i = blockIdx.x;; i += N) {
        const bool have_cur = i < total;
        Chunk cur;
        // ---- 1. prefetch this round's rows into L2
        if (have_cur) {
            cur = decode_item(i, ends, base, opc, G, n_slabs);
            const int64_t k0 = (int64_t)cur.s * PG_COLS;
            const uint32_t bytes = (uint32_t)(min((int64_t)PG_COLS, K - k0) * 2);
            for (int64_t r = cur.oct_lo * 8 + tid; r < cur.oct_hi * 8; r += T)
                if (r >= cur.start && r < cur.end) prefetch_l2(x + r * K + k0, bytes);
        }

        // ---- 2. convert the previous round's chunk
        if (have_prev) {
            if (tid == 0) {
                uint32_t spins = 0;
                while (ld_acquire_u32(&ws_count[prev.tile]) < (uint32_t)prev.n_chunks) {
                    // give up after the bound, or at once if some wait already gave up
                    if (++spins > PG_SPIN_LIMIT || *(volatile unsigned int*)&g_pg_error) {
                        atomicOr(&g_pg_error, 1u);
                        break;
                    }
                    __nanosleep(128);
                }
            }
            __syncthreads();
            const int64_t k0 = (int64_t)prev.s * PG_COLS;
            if (tid < PG_COLS) {
                const bool colv = k0 + tid < K;
                const uint32_t ab = colv ? ld_relaxed_u32(&ws_amax[prev.tile * PG_COLS + tid]) : 0u;
                const float s = ab >= 0x7F80u ? __uint_as_float(0x7FC00000u)
                                              : __fdiv_rn(448.0f, fmaxf(__uint_as_float(ab << 16), 1e-12f));
                sc[tid] = s;
                if (prev.r == 0 && colv) scales[(int64_t)prev.g * K + k0 + tid] = s;
            }
            __syncthreads();
            const int64_t c = k0 + 8 * v;
            if (c < K) {
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] = sc[8 * v + j];
                uint4 d[8];
                for (int64_t oc = prev.oct_lo + o; oc < prev.oct_hi; oc += oct_per_cta) {
                    int lo, hi;
                    octet_bounds(prev, oc * 8, &lo, &hi);
                    load_octet(d, x, oc * 8, lo, hi, K, c);
                    store_octet<COL_MAJOR>(d, f, q, oc * 8, lo, hi, M, K, c, vec_col_store);
                }
            }
        }
        if (!have_cur) break;

        // ---- 3. reduce this round's chunk and publish its maxima
        {
            const int64_t k0 = (int64_t)cur.s * PG_COLS;
            const int64_t c = k0 + 8 * v;
            uint32_t cm[4] = {0, 0, 0, 0};
            if (c < K) {
                uint4 d[8];
                for (int64_t oc = cur.oct_lo + o; oc < cur.oct_hi; oc += oct_per_cta) {
                    int lo, hi;
                    octet_bounds(cur, oc * 8, &lo, &hi);
                    load_octet(d, x, oc * 8, lo, hi, K, c);
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        cm[0] = amax2(cm[0], d[r].x);
                        cm[1] = amax2(cm[1], d[r].y);
                        cm[2] = amax2(cm[2], d[r].z);
                        cm[3] = amax2(cm[3], d[r].w);
                    }
                }
            }
#pragma unroll
            for (int sh = 8; sh <= 16; sh <<= 1)
#pragma unroll
                for (int w = 0; w < 4; ++w) cm[w] = amax2(cm[w], __shfl_xor_sync(FULL_MASK, cm[w], sh));
            if (lane < 8)
#pragma unroll
                for (int w = 0; w < 4; ++w) red[warp][lane * 4 + w] = cm[w];
            __syncthreads();
            if (warp == 0) {
                uint32_t m = 0;
                for (int w = 0; w < n_warps; ++w) m = amax2(m, red[w][lane]);
                m = mag2(m);
                // word `lane` = columns 8*(lane/4) + 2*(lane%4) + {0, 1} of the slab
                const int col0 = 8 * (lane >> 2) + 2 * (lane & 3);
                uint32_t* slot = ws_amax + cur.tile * PG_COLS;
                if (k0 + col0 < K) atomicMax(slot + col0, m & 0xFFFFu);
                if (k0 + col0 + 1 < K) atomicMax(slot + col0 + 1, m >> 16);
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(&ws_count[cur.tile], 1u);
            }
        }
        prev = cur;
        have_prev = true;
    }
}

// ---- host side ---------------------------------------------------------------------------

size_t per_group_workspace_bytes(int64_t K, int32_t G) {
    const int64_t n_tiles = (int64_t)G * ((K + PG_COLS - 1) / PG_COLS);
    return (size_t)n_tiles * (PG_COLS + 1) * sizeof(uint32_t);
}

// CTA size = rows per chunk: the average group size with 30% headroom, in multiples of
// 32, between 64 and 256.
static int per_group_threads(int64_t M, int32_t G) {
    const double want = (double)((M + G - 1) / G) * 1.3;
    int t = (int)std::ceil(want / 32.0) * 32;
    return std::max(64, std::min(PG_MAX_THREADS, t));
}

template <bool COL_MAJOR>
static cudaError_t launch_layout(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                                 int32_t G, uint8_t* q, float* scales, uint32_t* ws, int threads,
                                 cudaStream_t stream) {
    auto kern = per_group_kernel<COL_MAJOR>;
    const size_t smem = (size_t)(G + 1) * sizeof(int64_t) + (size_t)G * 2 * sizeof(int);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cache = dev >= 0 && dev < 64;
    static int attr_smem[64] = {0};
    if (smem > 48 * 1024 && (!cache || attr_smem[dev] < (int)smem)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (cache) attr_smem[dev] = (int)smem;
    }
    // persistent grid: every CTA resident at once (cooperative launch); the occupancy
    // query is cached per device for the last (threads, shared memory) pair
    static int occ_threads[64] = {0}, occ_smem[64] = {0}, occ_per_sm[64] = {0};
    int per_sm = 0;
    if (cache && occ_threads[dev] == threads && occ_smem[dev] == (int)smem) {
        per_sm = occ_per_sm[dev];
    } else {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
        if (e != cudaSuccess) return e;
        if (cache) {
            occ_threads[dev] = threads;
            occ_smem[dev] = (int)smem;
            occ_per_sm[dev] = per_sm;
        }
    }
    if (per_sm <= 0) return cudaErrorInvalidConfiguration;
    const int grid = per_sm * sm_count();
    const int64_t n_slabs = (K + PG_COLS - 1) / PG_COLS;
    const int64_t n_tiles = (int64_t)G * n_slabs;
    uint32_t* ws_amax = ws;
    uint32_t* ws_count = ws + n_tiles * PG_COLS;
    e = cudaMemsetAsync(ws, 0, per_group_workspace_bytes(K, G), stream);
    if (e != cudaSuccess) return e;
    int g_int = (int)G, ns = (int)n_slabs;
    bool vec_col_store = (M % 8) == 0;
    void* args[] = {(void*)&x, (void*)&M, (void*)&K, (void*)&offs, (void*)&g_int, (void*)&q,
                    (void*)&scales, (void*)&ws_amax, (void*)&ws_count, (void*)&ns, (void*)&vec_col_store};
    return cudaLaunchCooperativeKernel((const void*)kern, dim3((unsigned)grid), dim3((unsigned)threads), args,
                                       smem, stream);
}

cudaError_t launch_per_group(const uint16_t* x, int64_t M, int64_t K, const int32_t* offs,
                             int32_t G, bool col_major, uint8_t* q, float* scales, void* workspace,
                             cudaStream_t stream) {
    if (K == 0 || G == 0) return cudaSuccess;
    if (G > PG_MAX_G) return cudaErrorInvalidValue;
    const int threads = per_group_threads(M, G);
    uint32_t* ws = static_cast<uint32_t*>(workspace);
    return col_major ? launch_layout<true>(x, M, K, offs, G, q, scales, ws, threads, stream)
                     : launch_layout<false>(x, M, K, offs, G, q, scales, ws, threads, stream);
}

cudaError_t read_and_clear_device_error(unsigned int* out, cudaStream_t stream) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_pg_error, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_pg_error, &zero, sizeof(unsigned int));
}

}  // namespace mxq
