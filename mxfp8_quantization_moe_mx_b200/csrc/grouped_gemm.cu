// grouped_gemm.cu -- MXFP8 grouped GEMM on the 5th-generation tensor cores (sm_100a).
//
// Operation (torchtitan "[mxfp8 MoE training] Support mxfp8 all to all in expert
// parallel", Performance: the "+ MXFP8 Grouped GEMMs" rows; torchao "[moe training] fix
// uncoalesced global accesses in per group rowwise scaling kernel", Summary: the
// quantized expert tokens are the left operand of the scaled grouped GEMM): for the
// rows m of expert group g (the offsets' clamp rule),
//     out[m][n] = sum_k  A[m][k] 2^(sa[m][k/32]-127)  *  B[g][n][k] 2^(sb[g][n][k/32]-127)
// with A (M, K) and B (G, N, K) E4M3 codes in the 1x32 row layout of mx_quantize and
// their E8M0 scales in the 128 x 4 blocked layout of mx_scales_to_blocked (A per
// group, B per expert matrix).  fp32 accumulation in tensor memory, bf16 output.
//
// One CTA per (128-row M tile of a group, 256-column N tile); the M tiles of the
// groups are numbered in the padded order of the blocked scales, so a CTA's tile index
// is also its scale-tile index.  128 threads:
//   warp 0, one lane   -- producer: per 128-element K block, TMA loads of the A tile
//                         (128 x 128 B) and the B tile (256 x 128 B), both 128-byte
//                         swizzled, and bulk copies of the three 512-byte scale tiles,
//                         into a 4-stage shared-memory ring (full/empty mbarriers);
//   warp 1, one lane   -- MMA issuer: tcgen05.cp of the scale tiles into tensor memory
//                         (32x128b.warpx4: each 512-byte tile lands in 4 columns, copied
//                         to all four lane quarters), then four
//                         tcgen05.mma.kind::mxf8f6f4.block_scale of K = 32 (scale
//                         byte k of each column selected by the descriptor's scale
//                         ids), and tcgen05.commit to release the stage;
//   warp 2             -- allocates (and at the end frees) 512 tensor-memory columns:
//                         the 128 x 256 fp32 accumulator and the scale slots of the ring;
//   all four warps     -- epilogue: tcgen05.ld of their 32 accumulator lanes (rows),
//                         32 columns at a time, rounded to bf16, 64-byte row stores;
//                         rows past the group's end are not stored.
// Every mbarrier wait is bounded (2 s).  A CTA that gives up counts it
// (mxq_wait_timeouts), skips its stores, and still waits (20 s bound) for its copies
// and MMAs in flight before it frees tensor memory and exits.

#include <cstring>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int GG_BM = 128, GG_BN = 256, GG_BK = 128;  // tile rows, tile columns, K elements (= bytes) per stage
constexpr int GG_STAGES = 4;
constexpr int GG_A_BYTES = GG_BM * GG_BK;              // 16 KB
constexpr int GG_B_BYTES = GG_BN * GG_BK;              // 32 KB
constexpr int GG_SF_BYTES = 512;                       // one 128 x 4 scale tile
constexpr int GG_OFF_B = GG_STAGES * GG_A_BYTES;
constexpr int GG_OFF_SFA = GG_OFF_B + GG_STAGES * GG_B_BYTES;
constexpr int GG_OFF_SFB = GG_OFF_SFA + GG_STAGES * GG_SF_BYTES;
constexpr int GG_SMEM = GG_OFF_SFB + GG_STAGES * 2 * GG_SF_BYTES + 1024;  // + alignment slack
constexpr uint32_t GG_STAGE_TX = GG_A_BYTES + GG_B_BYTES + 3 * GG_SF_BYTES;
constexpr uint32_t GG_TMEM_COLS = 512;
constexpr uint32_t GG_TMEM_SFA = 256;                  // 4 columns per stage
constexpr uint32_t GG_TMEM_SFB = 256 + 4 * GG_STAGES;  // 8 columns per stage
constexpr uint64_t GG_WAIT_NS = 2000000000ull, GG_DRAIN_NS = 20000000000ull;

__device__ unsigned int g_gemm_timeouts = 0;  // CTAs that gave up a bounded wait

// ---- tcgen05 / bulk-copy wrappers -------------------------------------------------------

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes
// apart (rows of 128 bytes), Blackwell descriptor version 1.
__device__ __forceinline__ uint64_t desc_sw128(const void* p) {
    const uint64_t a = (smem_addr(p) & 0x3FFFFu) >> 4;
    return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Descriptor of a dense 32-row x 16-byte block (a 512-byte scale tile): no swizzle,
// 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(const void* p) {
    const uint64_t a = (smem_addr(p) & 0x3FFFFu) >> 4;
    return a | (8ull << 32) | (1ull << 46);
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 tensor-memory lanes (one row per lane).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Instruction descriptor of kind::mxf8f6f4 with E4M3 A and B, E8M0 scales, K-major A
// and B, M = 128, N = 256; scale byte `k` of the A and B scale columns.
__device__ __forceinline__ uint32_t idesc_mxf8(uint32_t k) {
    constexpr uint32_t base = (uint32_t)(GG_BN >> 3) << 17 | 1u << 23 | (uint32_t)(GG_BM >> 4) << 24;
    return base | k << 4 | k << 29;
}

// ---- the kernel -----------------------------------------------------------------------------

__global__ void __launch_bounds__(128, 1) mx_grouped_gemm_kernel(
    const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
    const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb, const int32_t* __restrict__ offs, int32_t G,
    int64_t M, int64_t N, int64_t K, uint16_t* __restrict__ out) {
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[GG_STAGES], empty[GG_STAGES], acc_full;
    __shared__ uint32_t tmem_base_s;
    __shared__ int64_t tile_info[3];  // first row of the tile, valid rows, group
    __shared__ int abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t n0 = (int64_t)blockIdx.x * GG_BN;
    const int64_t tile = blockIdx.y;
    const int64_t k_blocks = K / GG_BK;

    // ---- which group and rows this M tile covers (the padded order of the blocked scales)
    if (warp == 0) {
        int run = 0;
        int64_t padded = 0;
        bool found = false;
        for (int h0 = 0; h0 < G && !found; h0 += 32) {
            const int h = h0 + lane;
            int e = h < G ? max(offs[h], 0) : 0;
#pragma unroll
            for (int sh = 1; sh < 32; sh <<= 1) {
                const int o = __shfl_up_sync(FULL_MASK, e, sh);
                if (lane >= sh) e = max(e, o);
            }
            e = max(e, run);
            const int up = __shfl_up_sync(FULL_MASK, e, 1);
            const int prev_e = lane == 0 ? run : up;
            const int64_t end = min((int64_t)e, M), start = min((int64_t)prev_e, M);
            const int64_t n_tiles = h < G ? (end - start + GG_BM - 1) / GG_BM : 0;
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
                tile_info[0] = start + (tile - first) * GG_BM;
                tile_info[1] = min((int64_t)GG_BM, end - tile_info[0]);
                tile_info[2] = h;
            }
            found = who != 0;
            padded += __shfl_sync(FULL_MASK, inc, 31);
            run = __shfl_sync(FULL_MASK, e, 31);
        }
        if (!found && lane == 0) tile_info[1] = -1;
        if (lane == 0) {
            abort_s = 0;
            for (int s = 0; s < GG_STAGES; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            mbar_init(&acc_full, 1);
        }
    }
    __syncthreads();
    const int64_t row0 = tile_info[0], valid = tile_info[1];
    const int g = (int)tile_info[2];
    if (valid < 0) return;  // past the last used tile (uniform across the CTA, before any allocation)

    if (warp == 2) tmem_alloc(&tmem_base_s, GG_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;

    if (warp == 0 && lane == 0) {
        // ---- producer
        const int64_t n_tiles_b = N / 128, col_tiles = K / 128;
        const uint8_t* sfa_tile = sfa + tile * col_tiles * GG_SF_BYTES;
        const uint8_t* sfb_tile0 = sfb + ((int64_t)g * n_tiles_b + n0 / 128) * col_tiles * GG_SF_BYTES;
        const uint8_t* sfb_tile1 = sfb_tile0 + col_tiles * GG_SF_BYTES;
        const uint64_t pol = l2_policy_evict_last();
        int64_t armed = 0;
        for (int64_t it = 0; it < k_blocks; ++it) {
            const int s = (int)(it % GG_STAGES);
            const uint32_t r = (uint32_t)(it / GG_STAGES);
            if (!mbar_wait_bounded(&empty[s], (r & 1) ^ 1, GG_WAIT_NS)) {
                atomicExch(&abort_s, 1);
                break;
            }
            if (*(volatile int*)&abort_s) break;
            mbar_arrive_expect_tx(&full[s], GG_STAGE_TX);
            tma_load_2d(sm + s * GG_A_BYTES, &amap, (int)(it * GG_BK), (int)row0, &full[s], pol);
            tma_load_2d(sm + GG_OFF_B + s * GG_B_BYTES, &bmap, (int)(it * GG_BK), (int)((int64_t)g * N + n0), &full[s],
                        pol);
            bulk_copy_g2s(sm + GG_OFF_SFA + s * GG_SF_BYTES, sfa_tile + it * GG_SF_BYTES, GG_SF_BYTES, &full[s]);
            bulk_copy_g2s(sm + GG_OFF_SFB + s * 2 * GG_SF_BYTES, sfb_tile0 + it * GG_SF_BYTES, GG_SF_BYTES, &full[s]);
            bulk_copy_g2s(sm + GG_OFF_SFB + s * 2 * GG_SF_BYTES + GG_SF_BYTES, sfb_tile1 + it * GG_SF_BYTES,
                          GG_SF_BYTES, &full[s]);
            armed = it + 1;
        }
        // every copy this thread started has landed before the CTA can exit
        for (int64_t it = armed - GG_STAGES < 0 ? 0 : armed - GG_STAGES; it < armed; ++it)
            if (!mbar_wait_bounded(&full[it % GG_STAGES], (uint32_t)(it / GG_STAGES) & 1, GG_DRAIN_NS))
                atomicExch(&abort_s, 1);
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer
        for (int64_t it = 0; it < k_blocks; ++it) {
            const int s = (int)(it % GG_STAGES);
            const uint32_t r = (uint32_t)(it / GG_STAGES);
            if (!mbar_wait_bounded(&full[s], r & 1, GG_WAIT_NS)) {
                atomicExch(&abort_s, 1);
                break;
            }
            if (*(volatile int*)&abort_s) break;
            tc_fence_after();
            const uint32_t t_sfa = tmem + GG_TMEM_SFA + 4 * s, t_sfb = tmem + GG_TMEM_SFB + 8 * s;
            tmem_cp_sf(t_sfa, desc_sf(sm + GG_OFF_SFA + s * GG_SF_BYTES));
            tmem_cp_sf(t_sfb, desc_sf(sm + GG_OFF_SFB + s * 2 * GG_SF_BYTES));
            tmem_cp_sf(t_sfb + 4, desc_sf(sm + GG_OFF_SFB + s * 2 * GG_SF_BYTES + GG_SF_BYTES));
            const uint64_t a0 = desc_sw128(sm + s * GG_A_BYTES), b0 = desc_sw128(sm + GG_OFF_B + s * GG_B_BYTES);
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k)  // K = 32 per MMA: 32 bytes further along the swizzled rows
                mma_mxf8(tmem, a0 + 2 * k, b0 + 2 * k, idesc_mxf8(k), t_sfa | k << 30, t_sfb | k << 30,
                         (it > 0 || k > 0) ? 1u : 0u);
            mma_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        mma_commit(&acc_full);  // arrives when every MMA issued above has completed
    }
    __syncwarp();

    // ---- epilogue: warp w reads accumulator lanes (rows) 32w .. 32w+31
    const bool done = mbar_wait_bounded(&acc_full, 0, GG_WAIT_NS) || mbar_wait_bounded(&acc_full, 0, GG_DRAIN_NS);
    if (!done) atomicExch(&abort_s, 1);
    tc_fence_after();
    __syncthreads();  // abort_s is final here
    const bool skip = abort_s != 0;
    if (!skip && done) {
        const int r = 32 * warp + lane;
        uint16_t* orow = out + (row0 + r) * N + n0;
#pragma unroll 1
        for (int c0 = 0; c0 < GG_BN; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, v);
            if (r < valid) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 w;
                    w.x = cvt_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                    w.y = cvt_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                    w.z = cvt_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                    w.w = cvt_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                    *reinterpret_cast<uint4*>(orow + c0 + 8 * q) = w;
                }
            }
        }
    }
    if (skip && tid == 0) atomicAdd(&g_gemm_timeouts, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 2) tmem_dealloc(tmem, GG_TMEM_COLS);
}

// ---- host side -------------------------------------------------------------------------------

unsigned int read_gemm_timeouts() {
    unsigned int n = 0;
    if (cudaMemcpyFromSymbol(&n, g_gemm_timeouts, sizeof(n)) != cudaSuccess) return 0xFFFFFFFFu;
    return n;
}

cudaError_t launch_mx_grouped_gemm(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb, const uint8_t* sfb,
                                   const int32_t* offs, int32_t G, int64_t M, int64_t N, int64_t K, uint16_t* out,
                                   cudaStream_t stream) {
    const int64_t m_tiles = (M + (int64_t)(GG_BM - 1) * G) / GG_BM;  // bound on the groups' padded tiles
    if (m_tiles <= 0 || N == 0 || K == 0) return cudaSuccess;
    if (m_tiles > 65535 || N / GG_BN > 0x7FFFFFFFLL || M > 0x7FFFFFFFLL || (int64_t)G * N > 0x7FFFFFFFLL)
        return cudaErrorInvalidConfiguration;
    CUtensorMap amap, bmap;
    std::memset(&amap, 0, sizeof(amap));
    std::memset(&bmap, 0, sizeof(bmap));
    if (!encode_u8_tile_map_sw128(&amap, qa, (uint64_t)K, (uint64_t)M, GG_BK, GG_BM) ||
        !encode_u8_tile_map_sw128(&bmap, qb, (uint64_t)K, (uint64_t)G * N, GG_BK, GG_BN))
        return cudaErrorInvalidValue;
    const cudaError_t e =
        cudaFuncSetAttribute(mx_grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GG_SMEM);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(N / GG_BN), (unsigned)m_tiles);
    mx_grouped_gemm_kernel<<<grid, 128, GG_SMEM, stream>>>(amap, bmap, sfa, sfb, offs, G, M, N, K, out);
    return cudaGetLastError();
}

}  // namespace mxq
