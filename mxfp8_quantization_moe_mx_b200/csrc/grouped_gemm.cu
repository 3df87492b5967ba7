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
// Work unit: 256 rows of one group (two consecutive 128-row M tiles of the group, in the
// padded order of the blocked scales) x 256 columns, computed by a pair of CTAs (a
// 2-CTA cluster) with the paired MMA (tcgen05 .cta_group::2, M = 256, N = 256): each CTA
// stages its own 128 rows of A and its own half (128 rows) of the B tile, and the MMA
// reads B from both.  Per CTA that is 32 KB of operands per 128-element K block instead
// of 48 KB for a 128 x 256 tile on one SM, and six stages fit in shared memory.  A group
// with an odd number of M tiles leaves the second CTA of its last unit without rows: it
// computes on filler and stores nothing.
//
// Persistent: each cluster walks the units c, c + clusters, ... (M pairs major, the 256-
// column N tiles inner), 192 threads per CTA in three roles:
//   warp 0, one lane   -- producer (both CTAs): per K block, TMA loads of its A tile
//                         (128 x 128 B) and B half (128 x 128 B), both 128-byte swizzled,
//                         and of the scale tiles (its 512-byte A tile, both 512-byte B
//                         tiles: each CTA's tensor memory holds the scales of all 256
//                         columns), into a 6-stage ring.  All copies of both CTAs
//                         complete on the first CTA's `full` barrier; each CTA's own
//                         `empty` barrier frees its stage;
//   warp 1             -- allocates (and at the end frees) 512 tensor-memory columns in
//                         both CTAs: the 128-lane x 256-column fp32 accumulator (this
//                         CTA's rows) and the scale slots of the ring.  In the first CTA
//                         one lane issues: tcgen05.cp of the scale tiles (each CTA's
//                         shared memory into its own tensor memory), four paired
//                         tcgen05.mma.kind::mxf8f6f4.block_scale of K = 32, and a commit
//                         that releases the stage in both CTAs; a unit's first MMA waits
//                         until both epilogues have read the previous accumulator;
//   warps 2..5         -- epilogue (both CTAs): each reads its quarter of the
//                         accumulator lanes (rows) with tcgen05.ld, rounds the row to
//                         bf16 in registers, releases the accumulator (an arrival on the
//                         first CTA's barrier) and then stores, so the stores overlap the
//                         next unit's MMAs; rows past the group's end are not stored.
// Every mbarrier wait is bounded (2 s).  A CTA that gives up counts it
// (mxq_wait_timeouts) and skips its remaining stores; before the pair frees tensor memory
// and exits, the copies both CTAs started are accounted on the first CTA's barriers and
// awaited there, and the MMAs in flight too (20 s bounds).

#include <algorithm>
#include <cstring>

#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int GG_BM = 128;                             // rows per CTA (the paired MMA: 256)
constexpr int GG_BN = 256, GG_BK = 128;                // tile columns, K elements (= bytes) per stage
constexpr int GG_STAGES = 6;
constexpr int GG_A_BYTES = GG_BM * GG_BK;              // 16 KB
constexpr int GG_B_BYTES = (GG_BN / 2) * GG_BK;        // this CTA's half of the B tile, 16 KB
constexpr int GG_SF_BYTES = 512;                       // one 128 x 4 scale tile
constexpr int GG_OFF_B = GG_STAGES * GG_A_BYTES;
constexpr int GG_OFF_SFA = GG_OFF_B + GG_STAGES * GG_B_BYTES;
constexpr int GG_OFF_SFB = GG_OFF_SFA + GG_STAGES * GG_SF_BYTES;
constexpr int GG_SMEM = GG_OFF_SFB + GG_STAGES * 2 * GG_SF_BYTES + 1024;  // + alignment slack
constexpr uint32_t GG_CTA_TX = GG_A_BYTES + GG_B_BYTES + 3 * GG_SF_BYTES;  // one CTA's bytes per stage
constexpr uint32_t GG_TMEM_COLS = 512;
constexpr uint32_t GG_TMEM_SFA = 256;                  // 4 columns per stage
constexpr uint32_t GG_TMEM_SFB = 256 + 4 * GG_STAGES;  // 8 columns per stage
constexpr uint64_t GG_WAIT_NS = 2000000000ull, GG_DRAIN_NS = 20000000000ull;
static_assert(GG_TMEM_SFB + 8 * GG_STAGES <= GG_TMEM_COLS, "tensor-memory columns");
static_assert(GG_SMEM <= 227 * 1024, "shared memory per CTA");

__device__ unsigned int g_gemm_timeouts = 0;  // CTAs that gave up a bounded wait

// ---- tcgen05 / cluster wrappers (paired forms) -----------------------------------------------

// TMA 2-D tile load into this CTA's shared memory that completes on an mbarrier of either
// CTA of the pair (`bar` a cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* tmap, int x, int y, uint32_t bar,
                                                 uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(bar), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Count `bytes` as arrived on the current phase's transaction count (no arrival).
__device__ __forceinline__ void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Whole-cluster barrier with release / acquire (every thread of both CTAs).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
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

// Paired copy: each CTA's 512-byte scale tile at this shared-memory offset into 4 columns
// of its own tensor memory (copied to all four lane quarters).
__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Arrives (once) on the mbarrier at this shared-memory offset in both CTAs of the pair
// when every tcgen05 operation this thread issued before it has completed.
__device__ __forceinline__ void mma_commit_both(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_addr(bar)),
        "h"((uint16_t)3)
        : "memory");
}

// ... on this CTA's mbarrier only.
__device__ __forceinline__ void mma_commit_own(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
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
// and B, M = 256 (the pair), N = 256; scale byte `k` of the A and B scale columns.
__device__ __forceinline__ uint32_t idesc_mxf8(uint32_t k) {
    constexpr uint32_t base = (uint32_t)(GG_BN >> 3) << 17 | 1u << 23 | (uint32_t)((2 * GG_BM) >> 4) << 24;
    return base | k << 4 | k << 29;
}

// ---- the kernel -----------------------------------------------------------------------------

struct PairTile {
    int64_t row0;    // first row of the unit (the first CTA's rows; the second's start 128 later)
    int64_t valid0;  // rows of the group in the first CTA's 128 (>= 1)
    int64_t valid1;  // ... in the second CTA's 128 (<= 0: none)
    int64_t mt0;     // padded M-tile index of the first CTA's rows (its scale tile)
    int g;           // the group (expert)
};

// Run by a whole warp: M pair `pair` -- the groups' padded M tiles taken two at a time
// within each group, groups in order -- returned to every lane.  With pair < 0 only the
// number of pairs is computed (into *total).
__device__ void gg_find_pair(const int32_t* __restrict__ offs, int32_t G, int64_t M, int64_t pair, PairTile* pt,
                             int64_t* total) {
    const int lane = threadIdx.x & 31;
    int run = 0;
    int64_t tiles_before = 0, pairs_before = 0;
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
        const int64_t n_pairs = (n_tiles + 1) / 2;
        int64_t inc_t = n_tiles, inc_p = n_pairs;
#pragma unroll
        for (int sh = 1; sh < 32; sh <<= 1) {
            const int64_t ot = __shfl_up_sync(FULL_MASK, inc_t, sh);
            const int64_t op = __shfl_up_sync(FULL_MASK, inc_p, sh);
            if (lane >= sh) {
                inc_t += ot;
                inc_p += op;
            }
        }
        const int64_t first_t = tiles_before + inc_t - n_tiles, first_p = pairs_before + inc_p - n_pairs;
        const bool mine = pair >= 0 && h < G && pair >= first_p && pair < first_p + n_pairs;
        const unsigned who = __ballot_sync(FULL_MASK, mine);
        if (who) {
            const int src = __ffs(who) - 1;
            const int64_t j = 2 * (pair - first_p);
            const int64_t my_r0 = start + j * GG_BM;
            pt->row0 = __shfl_sync(FULL_MASK, my_r0, src);
            pt->valid0 = __shfl_sync(FULL_MASK, min((int64_t)GG_BM, end - my_r0), src);
            pt->valid1 = __shfl_sync(FULL_MASK, min((int64_t)GG_BM, end - my_r0 - GG_BM), src);
            pt->mt0 = __shfl_sync(FULL_MASK, first_t + j, src);
            pt->g = __shfl_sync(FULL_MASK, h, src);
            found = true;
        }
        tiles_before += __shfl_sync(FULL_MASK, inc_t, 31);
        pairs_before += __shfl_sync(FULL_MASK, inc_p, 31);
        run = __shfl_sync(FULL_MASK, e, 31);
    }
    if (total) *total = pairs_before;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1) mx_grouped_gemm_kernel(
    const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
    const __grid_constant__ CUtensorMap sfamap, const __grid_constant__ CUtensorMap sfbmap,
    const int32_t* __restrict__ offs, int32_t G, int64_t M, int64_t N, int64_t K, uint16_t* __restrict__ out) {
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[GG_STAGES], empty[GG_STAGES], acc_full, acc_empty, drained;
    __shared__ uint32_t tmem_base_s;
    __shared__ uint32_t issued_s[2];  // stages each CTA's producer armed / issued (exchanged at the end)
    __shared__ int64_t n_work_s;
    __shared__ int abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const bool first = rank == 0;
    const int64_t cl = blockIdx.x >> 1, n_cl = gridDim.x >> 1;
    const int64_t n_tiles_n = N / GG_BN;
    const int64_t k_blocks = K / GG_BK;
    const int64_t col_tiles = K / 128;

    if (warp == 0) {
        PairTile pt;
        int64_t total;
        gg_find_pair(offs, G, M, -1, &pt, &total);
        if (lane == 0) {
            n_work_s = total * n_tiles_n;
            abort_s = 0;
            issued_s[0] = issued_s[1] = 0;
            for (int s = 0; s < GG_STAGES; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            mbar_init(&acc_full, 1);
            mbar_init(&acc_empty, 8);  // the epilogue warps of both CTAs
            mbar_init(&drained, 1);
        }
    }
    if (warp == 1) tmem_alloc_pair(&tmem_base_s, GG_TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const int64_t n_work = n_work_s;
    const uint32_t full0 = cluster_map(&full[0], 0);  // the first CTA's `full` ring (8 bytes apart)
    const uint32_t acc_empty0 = cluster_map(&acc_empty, 0);

    uint32_t it_prod = 0;
    if (warp == 0) {
        // ---- producer (both CTAs)
        const uint64_t pol = l2_policy_evict_last();
        bool stop = false;
        for (int64_t w = cl; w < n_work && !stop; w += n_cl) {
            const int64_t p = w / n_tiles_n, n0 = (w % n_tiles_n) * GG_BN;
            PairTile pt;
            gg_find_pair(offs, G, M, p, &pt, nullptr);
            if (lane == 0) {
                const int64_t my_row = pt.row0 + (int64_t)rank * GG_BM;
                const int64_t my_mt = (rank == 1 && pt.valid1 > 0) ? pt.mt0 + 1 : pt.mt0;  // filler: any real tile
                const int64_t sfa_row = 2 * my_mt * col_tiles;
                const int64_t sfb_row = 2 * ((int64_t)pt.g * (N / 128) + n0 / 128) * col_tiles;
                const int b_row = (int)((int64_t)pt.g * N + n0 + (int64_t)rank * (GG_BN / 2));
                for (int64_t kb = 0; kb < k_blocks; ++kb, ++it_prod) {
                    const int s = (int)(it_prod % GG_STAGES);
                    const uint32_t r = it_prod / GG_STAGES;
                    if (!mbar_wait_bounded(&empty[s], (r & 1) ^ 1, GG_WAIT_NS) || *(volatile int*)&abort_s) {
                        atomicExch(&abort_s, 1);
                        stop = true;
                        break;
                    }
                    if (first) mbar_arrive_expect_tx(&full[s], 2 * GG_CTA_TX);
                    const uint32_t bar = full0 + 8u * (uint32_t)s;
                    tma_load_2d_pair(sm + s * GG_A_BYTES, &amap, (int)(kb * GG_BK), (int)my_row, bar, pol);
                    tma_load_2d_pair(sm + GG_OFF_B + s * GG_B_BYTES, &bmap, (int)(kb * GG_BK), b_row, bar, pol);
                    tma_load_2d_pair(sm + GG_OFF_SFA + s * GG_SF_BYTES, &sfamap, 0, (int)(sfa_row + 2 * kb), bar,
                                     pol);
                    tma_load_2d_pair(sm + GG_OFF_SFB + s * 2 * GG_SF_BYTES, &sfbmap, 0, (int)(sfb_row + 2 * kb), bar,
                                     pol);
                    tma_load_2d_pair(sm + GG_OFF_SFB + s * 2 * GG_SF_BYTES + GG_SF_BYTES, &sfbmap, 0,
                                     (int)(sfb_row + 2 * col_tiles + 2 * kb), bar, pol);
                }
            }
            stop = __shfl_sync(FULL_MASK, stop ? 1 : 0, 0) != 0;
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMA issuer (the first CTA)
        if (first && lane == 0) {
            uint32_t it = 0;
            int64_t i = 0;
            for (int64_t w = cl; w < n_work; w += n_cl, ++i) {
                if (i > 0 && !mbar_wait_bounded(&acc_empty, (uint32_t)((i - 1) & 1), GG_WAIT_NS)) {
                    atomicExch(&abort_s, 1);
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int64_t kb = 0; kb < k_blocks; ++kb, ++it) {
                    const int s = (int)(it % GG_STAGES);
                    const uint32_t r = it / GG_STAGES;
                    if (!mbar_wait_bounded(&full[s], r & 1, GG_WAIT_NS) || *(volatile int*)&abort_s) {
                        atomicExch(&abort_s, 1);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t t_sfa = tmem + GG_TMEM_SFA + 4 * s, t_sfb = tmem + GG_TMEM_SFB + 8 * s;
                    tmem_cp_sf_pair(t_sfa, desc_sf(sm + GG_OFF_SFA + s * GG_SF_BYTES));
                    tmem_cp_sf_pair(t_sfb, desc_sf(sm + GG_OFF_SFB + s * 2 * GG_SF_BYTES));
                    tmem_cp_sf_pair(t_sfb + 4, desc_sf(sm + GG_OFF_SFB + s * 2 * GG_SF_BYTES + GG_SF_BYTES));
                    const uint64_t a0 = desc_sw128(sm + s * GG_A_BYTES), b0 = desc_sw128(sm + GG_OFF_B + s * GG_B_BYTES);
#pragma unroll
                    for (uint32_t k = 0; k < 4; ++k)  // K = 32 per MMA: 32 bytes further along the swizzled rows
                        mma_mxf8_pair(tmem, a0 + 2 * k, b0 + 2 * k, idesc_mxf8(k), t_sfa | k << 30, t_sfb | k << 30,
                                      (kb > 0 || k > 0) ? 1u : 0u);
                    mma_commit_both(&empty[s]);  // the stage is free in both CTAs once these MMAs have read it
                }
                if (!ok) break;              // a partial accumulator is never handed to the epilogues
                mma_commit_both(&acc_full);  // the unit's accumulators are complete once its MMAs are
            }
            // every tcgen05 operation issued above (and its arrivals) is done before the pair
            // frees tensor memory or leaves
            mma_commit_own(&drained);
            if (!mbar_wait_bounded(&drained, 0, GG_DRAIN_NS)) atomicExch(&abort_s, 1);
        }
        __syncwarp();
    } else {
        // ---- epilogue (both CTAs): warp w reads accumulator lanes (rows) 32 (w % 4) .. + 31
        const int quarter = warp & 3;
        const int r = 32 * quarter + lane;
        int64_t i = 0;
        for (int64_t w = cl; w < n_work; w += n_cl, ++i) {
            const int64_t p = w / n_tiles_n, n0 = (w % n_tiles_n) * GG_BN;
            PairTile pt;
            gg_find_pair(offs, G, M, p, &pt, nullptr);
            const bool done = mbar_wait_bounded(&acc_full, (uint32_t)(i & 1), GG_WAIT_NS);
            if (!done) atomicExch(&abort_s, 1);
            if (__any_sync(FULL_MASK, !done) || *(volatile int*)&abort_s) break;
            tc_fence_after();
            // the whole row, rounded to bf16 in registers, so the accumulator is released
            // before the stores and the next unit's MMAs overlap them
            uint32_t v16[GG_BN / 2];
#pragma unroll
            for (int c0 = 0; c0 < GG_BN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0, v);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    v16[c0 / 2 + j] = cvt_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0);  // this warp's quarter is read
            const int64_t valid = rank == 0 ? pt.valid0 : pt.valid1;
            if (r < valid) {
                uint4* orow = reinterpret_cast<uint4*>(out + (pt.row0 + (int64_t)rank * GG_BM + r) * N + n0);
#pragma unroll
                for (int q = 0; q < GG_BN / 8; ++q)
                    orow[q] = make_uint4(v16[4 * q], v16[4 * q + 1], v16[4 * q + 2], v16[4 * q + 3]);
            }
        }
    }

    // ---- leaving: account every copy either producer started on the first CTA's `full`
    // barriers and wait for them there, so neither CTA's shared memory is still a copy's
    // destination (or a barrier still to be signalled) when the pair exits
    if (warp == 0 && lane == 0) {
        issued_s[rank] = it_prod;
        st_cluster_u32(cluster_map(&issued_s[rank], rank ^ 1u), it_prod);
    }
    tc_fence_before();
    cluster_sync();
    if (first && warp == 0 && lane == 0) {
        const uint32_t i0 = issued_s[0], i1 = issued_s[1];
        // stages the second CTA filled but this one never armed: arm them for its bytes;
        // stages armed for both but filled only here: count the missing bytes as arrived
        for (uint32_t i = i0; i < i1; ++i) mbar_arrive_expect_tx(&full[i % GG_STAGES], GG_CTA_TX);
        for (uint32_t i = i1; i < i0; ++i) mbar_complete_tx(&full[i % GG_STAGES], GG_CTA_TX);
        const uint32_t hi = max(i0, i1);
        for (uint32_t i = hi > (uint32_t)GG_STAGES ? hi - GG_STAGES : 0u; i < hi; ++i)
            if (!mbar_wait_bounded(&full[i % GG_STAGES], (i / GG_STAGES) & 1, GG_DRAIN_NS)) atomicExch(&abort_s, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (abort_s && tid == 0) atomicAdd(&g_gemm_timeouts, 1u);
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, GG_TMEM_COLS);
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
    const int64_t col_tiles = K / 128;
    const int64_t sfa_rows = 2 * m_tiles * col_tiles, sfb_rows = 2 * (int64_t)G * (N / 128) * col_tiles;
    if (M + GG_BM > 0x7FFFFFFFLL || (int64_t)G * N > 0x7FFFFFFFLL || sfa_rows > 0x7FFFFFFFLL ||
        sfb_rows > 0x7FFFFFFFLL)
        return cudaErrorInvalidConfiguration;
    CUtensorMap amap, bmap, sfamap, sfbmap;
    std::memset(&amap, 0, sizeof(amap));
    std::memset(&bmap, 0, sizeof(bmap));
    std::memset(&sfamap, 0, sizeof(sfamap));
    std::memset(&sfbmap, 0, sizeof(sfbmap));
    // the scale arrays as rows of 256 bytes: one 512-byte scale tile is a 2-row box
    if (!encode_u8_tile_map_sw128(&amap, qa, (uint64_t)K, (uint64_t)M, GG_BK, GG_BM) ||
        !encode_u8_tile_map_sw128(&bmap, qb, (uint64_t)K, (uint64_t)G * N, GG_BK, GG_BN / 2) ||
        !encode_u8_map_plain(&sfamap, sfa, 256, (uint64_t)sfa_rows, 256, 2) ||
        !encode_u8_map_plain(&sfbmap, sfb, 256, (uint64_t)sfb_rows, 256, 2))
        return cudaErrorInvalidValue;
    const cudaError_t e =
        cudaFuncSetAttribute(mx_grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GG_SMEM);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (about 202 KB of shared memory each), in pairs, at most one
    // pair per unit (the pair count bounds the units from above)
    const int64_t units = (m_tiles + G) / 2 * (N / GG_BN);
    const int64_t pairs = std::max<int64_t>(1, std::min<int64_t>(units, sm_count() / 2));
    mx_grouped_gemm_kernel<<<(unsigned)(2 * pairs), 192, GG_SMEM, stream>>>(amap, bmap, sfamap, sfbmap, offs, G, M, N,
                                                                           K, out);
    return cudaGetLastError();
}

}  // namespace mxq
