// mxq_device.cuh -- device helpers shared by the sm_100a kernels of libmxq.
//
// Number formats (OCP FP8 / MX): E4M3 = 1 sign, 4 exponent bits (bias 7), 3 mantissa
// bits, max 448, NaN = S.1111.111; E8M0 = biased exponent b, value 2^(b-127), 0xFF NaN;
// bf16 = upper half of an IEEE binary32.
//
// Build rule: no fast-math.  Subnormal bf16 inputs are fp32 subnormals after widening
// and must survive the multiply by 2^(127-b) (a flush to zero would change the result),
// and the per-group scale needs the IEEE divide.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxq {

constexpr unsigned FULL_MASK = 0xFFFFFFFFu;

// ---- loads / stores ----------------------------------------------------------------

// 16-byte read-only load that does not allocate in L1 (each byte is read once).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
    uint2 r;
    asm("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_nc_u8(const void* p) {
    unsigned short r;
    asm("ld.global.nc.u8 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// L2 prefetch of the line holding p, with evict_last priority so that it stays until the
// load that wants it (issued part of a wave of CTAs, or one loop step, later) arrives
// (measured: a normal-priority prefetch gained about half as much).
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}

// ---- L2 eviction-priority hints --------------------------------------------------------
// For data that is read twice with other traffic in between: the first read carries an
// evict_last policy so the line outlives the streaming traffic around it, the second
// read (and stores that are not read again) evict_first, which also demotes the line.

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint4 ld_nc_v4_hint(const void* p, uint64_t pol) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p), "l"(pol));
    return r;
}

__device__ __forceinline__ void st_v2_hint(void* p, uint2 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.u32 [%0], {%1, %2}, %3;"
                 :: "l"(p), "r"(v.x), "r"(v.y), "l"(pol) : "memory");
}

// ---- conversions ---------------------------------------------------------------------

// Two fp32 values -> two E4M3 codes, round to nearest even, saturating to +-448
// (PTX cvt ... .satfinite.e4m3x2.f32: first source goes to the upper byte).
// Result: `lo` in bits 0..7, `hi` in bits 8..15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return (uint32_t)r;
}

// Four fp32 values -> four E4M3 codes in one word (a in bits 0..7 ... d in 24..31),
// same convert; the two 16-bit halves are joined inside the asm block.
__device__ __forceinline__ uint32_t cvt4_e4m3(float a, float b, float c, float d) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "f"(a), "f"(b), "f"(c), "f"(d));
    return r;
}

// Two fp32 products at once (PTX mul.rn.f32x2, sm_100): (a0*b0, a1*b1), each rounded
// to nearest even, subnormals kept (no .ftz).
__device__ __forceinline__ void fmul2(float a0, float a1, float b0, float b1, float& r0, float& r1) {
    unsigned long long x, y, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b0), "f"(b1));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(x), "l"(y));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}

// The same two products as two scalar multiplies (measured faster than the packed form
// where fewer values are live).
__device__ __forceinline__ void fmul2s(float a0, float a1, float b0, float b1, float& r0, float& r1) {
    r0 = __fmul_rn(a0, b0);
    r1 = __fmul_rn(a1, b1);
}

// Two fp32 values -> bf16x2, round to nearest even (subnormals kept); `lo` in bits 0..15.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// The two bf16 halves of a 32-bit word as fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Running maximum of magnitudes, two bf16 lanes at once: max.NaN.xorsign.abs.bf16x2
// returns max(|a|, |b|) per half (one instruction, absolute values taken inside) with
// the sign bit set to the XOR of the input signs, and a NaN if either input is NaN.
// Only magnitudes are kept, so callers clear the sign bits once after the reduction
// (mag2).  For non-negative bf16 values the float order equals the order of the bit
// patterns, so the result's bits are exactly the largest magnitude's bits (a NaN
// anywhere gives 0x7FFF, which every consumer treats like Inf: >= 0x7F80).
__device__ __forceinline__ uint32_t amax2(uint32_t acc, uint32_t w) {
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w));
    return r;
}
__device__ __forceinline__ uint32_t mag2(uint32_t w) { return w & 0x7FFF7FFFu; }

// ---- MX scale ---------------------------------------------------------------------------

// E8M0 byte of a block from the bf16 bit pattern of its amax (sign cleared).
// For finite amax with biased exponent E: floor(log2 amax) - 8 + 127 = E - 8, clamped at
// 0 (subnormal and zero amax land there too); the top clamp (254) cannot bind since
// E <= 254.  E == 255 (Inf/NaN in the block) gives the NaN scale 0xFF.
__device__ __forceinline__ uint32_t e8m0_of_amax(uint32_t amax_bits) {
    const uint32_t E = amax_bits >> 7;
    return E == 255u ? 255u : (E > 8u ? E - 8u : 0u);
}

// The same for an amax known to be finite (E <= 254): E - 8 clamped at 0.
__device__ __forceinline__ uint32_t e8m0_of_finite_amax(uint32_t amax_bits) {
    return (uint32_t)max((int)(amax_bits >> 7) - 8, 0);
}

// 2^(127-b) as fp32 (exponent field 254-b, a normal number for b <= 246).
__device__ __forceinline__ float mx_mult(uint32_t b) { return __uint_as_float((254u - b) << 23); }

// 2^(b-127) as fp32: normal for b >= 1, the subnormal 2^-127 for b == 0.
__device__ __forceinline__ float e8m0_value(uint32_t b) {
    return b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

// Four bf16 values (two words) times an exact power of two -> four E4M3 codes.
__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, float m) {
    float p0, p1, p2, p3;
    fmul2(bf16_lo(w0), bf16_hi(w0), m, m, p0, p1);
    fmul2(bf16_lo(w1), bf16_hi(w1), m, m, p2, p3);
    return cvt4_e4m3(p0, p1, p2, p3);
}

// NaN codes (0x7F with each element's sign) for four bf16 values: the reading for a
// block whose scale is NaN.
__device__ __forceinline__ uint32_t nan4(uint32_t w0, uint32_t w1) {
    const uint32_t s = ((w0 >> 8) & 0x80u) | ((w0 >> 16) & 0x8000u) |
                       ((w1 << 8) & 0x800000u) | (w1 & 0x80000000u);
    return s | 0x7F7F7F7Fu;
}

// ---- E4M3 -> bf16 -----------------------------------------------------------------------

// The code in bits 24..31 of `t` (other bits zero) becomes an fp32 whose value is the
// E4M3 value times 2^-120: shifting right by 4 (arithmetic) puts eeee into the low four
// exponent bits and mmm at the top of the mantissa, and the mask drops the copies of
// the sign bit.  E4M3 subnormals land on fp32 subnormals with the same 2^-120 factor.
// The caller multiplies by 2^120 (exact) to get the value.
__device__ __forceinline__ float e4m3_scaled_from_top_byte(uint32_t t) {
    return __uint_as_float((uint32_t)((int32_t)t >> 4) & 0x87F00000u);
}

// True if any of the four codes in `w` is a NaN code (low seven bits all ones).
__device__ __forceinline__ bool any_e4m3_nan(uint32_t w) {
    return (((w & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u) != 0u;
}

// Two codes -- bytes 0, 1 of w (HI false) or bytes 2, 3 (HI true) -- as fp32, with the
// hardware converter: cvt.rn.f16x2.e4m3x2 widens them to f16 (exact: every E4M3 value is
// an f16 normal or zero; a NaN code gives a NaN), cvt.f32.f16 to fp32 (exact).
template <bool HI>
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t w, float& a, float& b) {
    if (HI)
        asm("{\n\t.reg .b16 c01, c23, h0, h1;\n\t.reg .b32 p;\n\t"
            "mov.b32 {c01, c23}, %2;\n\t"
            "cvt.rn.f16x2.e4m3x2 p, c23;\n\t"
            "mov.b32 {h0, h1}, p;\n\t"
            "cvt.f32.f16 %0, h0;\n\t"
            "cvt.f32.f16 %1, h1;\n\t}"
            : "=f"(a), "=f"(b)
            : "r"(w));
    else
        asm("{\n\t.reg .b16 c01, c23, h0, h1;\n\t.reg .b32 p;\n\t"
            "mov.b32 {c01, c23}, %2;\n\t"
            "cvt.rn.f16x2.e4m3x2 p, c01;\n\t"
            "mov.b32 {h0, h1}, p;\n\t"
            "cvt.f32.f16 %0, h0;\n\t"
            "cvt.f32.f16 %1, h1;\n\t}"
            : "=f"(a), "=f"(b)
            : "r"(w));
}

// Four codes (one word) times 2^(b-127) -> four bf16 (two words), decoded by the hardware
// converter: the exact product with the power-of-two scale and one RNE rounding to bf16.
// Codes must not be NaN (the caller's slow path handles those).
__device__ __forceinline__ uint2 dequant4_cvt(uint32_t w, float sc) {
    float f0, f1, f2, f3;
    e4m3x2_to_f32<false>(w, f0, f1);
    e4m3x2_to_f32<true>(w, f2, f3);
    float p0, p1, p2, p3;
    fmul2(f0, f1, sc, sc, p0, p1);
    fmul2(f2, f3, sc, sc, p2, p3);
    return make_uint2(cvt_bf16x2(p0, p1), cvt_bf16x2(p2, p3));
}

// Slow path for words that hold a NaN code or sit under a NaN scale.
__device__ __forceinline__ uint2 dequant4_nan_aware(uint32_t w, uint32_t b) {
    const float sc = e8m0_value(b);
    uint2 r = dequant4_cvt(w, sc);
    uint32_t h[4] = {r.x & 0xFFFFu, r.x >> 16, r.y & 0xFFFFu, r.y >> 16};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t c = (w >> (8 * i)) & 0xFFu;
        if (b == 255u || (c & 0x7Fu) == 0x7Fu) h[i] = 0x7FC0u;
    }
    return make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
}


// ---- shared memory, mbarriers and TMA ------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint4 lds_v4(const void* p) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(smem_addr(p)));
    return r;
}

// The same load from a 32-bit shared-window address.
__device__ __forceinline__ uint4 lds_v4_at(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(a));
    return r;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
    // make the initialised barrier visible to the async (TMA) proxy
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive once and add `bytes` to the transaction count the current phase waits for.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of the barrier to complete, giving up after `limit_ns`.  A limit
// of 0 gives up at once without looking (the library's wait-limit control uses it to
// exercise the give-up path).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (limit_ns == 0) return false;
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > limit_ns) return false;
    return true;
}

// 2-D TMA tile load (box dimensions from the tensor map) into shared memory, completing
// on `bar` and carrying the L2 policy `pol`.  dst must be 128-byte aligned; x * element
// size must be a multiple of 16 bytes.
// L2 prefetch of one box of a 2-D tensor map at (x, y) (no shared memory, no barrier);
// x * element size must be a multiple of 16 bytes, as for the load.
__device__ __forceinline__ void tma_prefetch_2d(const void* tmap, int x, int y, uint64_t pol) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile.L2::cache_hint [%0, {%1, %2}], %3;" ::"l"(tmap),
                 "r"(x), "r"(y), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar,
                                            uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

// ---- thread-block clusters ------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Cluster-wide barrier halves; every thread of every CTA of the cluster executes both,
// alternating arrive and wait.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t cluster_map(const void* local_smem_ptr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local_smem_ptr)), "r"(rank));
    return remote;
}

// Asynchronous 32-bit store into another CTA's shared memory (cluster addresses from
// cluster_map) that counts 4 bytes toward the transaction count of that CTA's mbarrier.
__device__ __forceinline__ void st_async_u32(uint32_t remote_addr, uint32_t value, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(remote_addr),
                 "r"(value), "r"(remote_bar)
                 : "memory");
}

}  // namespace mxq
