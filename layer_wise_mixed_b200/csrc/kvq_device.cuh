// Device helpers shared by the decode kernels (mma.sync and tcgen05 paths): PTX
// wrappers for shared-memory addresses, mbarriers with bounded waits, bulk copies and
// mma.sync; the exact fp16 unpack of packed code fields; small float helpers; the size
// of a block record.  Everything sits in an unnamed namespace: each translation unit
// gets its own inline copies.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, unsigned bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase), "r"(100000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait: polls until the phase completes or kWaitLimitNs of wall time (the GPU's
// global nanosecond timer) have passed since the first failed poll, then reports
// failure; the caller records kStatusWaitExpired and returns normally.  A copy lands
// in microseconds, so the limit is only reached when something is broken.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned phase) {
    if (mbar_try_wait(bar, phase)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, phase)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

__device__ __forceinline__ void mma16816(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same shape with bf16 operands (the bf16 residual keys of a per-channel layer).
__device__ __forceinline__ void mma16816_bf16(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(orv));
    return d;
}
// (a & m) | (b & ~m) in one LOP3
__device__ __forceinline__ uint32_t lop_sel(uint32_t a, uint32_t b, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
    return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }
__device__ __forceinline__ __half2 bits_h2(uint32_t v) { return *reinterpret_cast<__half2 *>(&v); }
__device__ __forceinline__ uint32_t hsub2_bits(uint32_t x, uint32_t y) {
    return h2_bits(__hsub2(bits_h2(x), bits_h2(y)));
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) { return h2_bits(__floats2half2_rn(lo, hi)); }

// Exact fp16 pair of the two codes of slot p of a word: field p (low half) and field
// p + P (high half), P = 16/BITS.  The masked code bits are OR-ed under an fp16
// exponent M chosen so that one mantissa step of the code is 1.0: the half then
// holds M + c exactly, and subtracting M leaves c (M = 1024, 256, 64 or 16 for code
// bits starting at mantissa bit 0, 2, 4 or 6).
template <int BITS>
__device__ __forceinline__ uint32_t unpack(uint32_t w, int p) {
    if constexpr (BITS == 8) {
        const uint32_t sel = static_cast<uint32_t>(p) | 0x40u | (static_cast<uint32_t>(p + 2) << 8) | 0x4000u;
        return hsub2_bits(prmt(w, 0x64646464u, sel), 0x64006400u);
    } else if constexpr (BITS == 4) {
        const uint32_t src = p < 2 ? w : (w >> 8);
        if ((p & 1) == 0) return hsub2_bits(lop_and_or(src, 0x000F000Fu, 0x64006400u), 0x64006400u);   // 1024 + c
        return hsub2_bits(lop_and_or(src, 0x00F000F0u, 0x54005400u), 0x54005400u);                     // 64 + c
    } else {
        const uint32_t src = p < 4 ? w : (w >> 8);
        const int q = p & 3;
        const uint32_t M = q == 0 ? 0x64006400u : (q == 1 ? 0x5C005C00u : (q == 2 ? 0x54005400u : 0x4C004C00u));
        return hsub2_bits(lop_and_or(src, 0x00030003u << (2 * q), M), M);
    }
}

// hi = value truncated to 11 significant bits (exact in fp16 for normal range),
// lo = exact remainder.
__device__ __forceinline__ float trunc11(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Load a lane's words of one half code area (Wh words, chunked by min(4, Wh)).
template <int WH>
__device__ __forceinline__ void load_lane_words(const uint8_t *half_area, int lane, uint32_t *w) {
    if constexpr (WH >= 4) {
#pragma unroll
        for (int u = 0; u < WH / 4; ++u) {
            const uint4 v = *reinterpret_cast<const uint4 *>(half_area + ((u * 32 + lane) * 4) * 4);
            w[4 * u] = v.x;
            w[4 * u + 1] = v.y;
            w[4 * u + 2] = v.z;
            w[4 * u + 3] = v.w;
        }
    } else if constexpr (WH == 2) {
        const uint2 v = *reinterpret_cast<const uint2 *>(half_area + (lane * 2) * 4);
        w[0] = v.x;
        w[1] = v.y;
    } else {
        w[0] = *reinterpret_cast<const uint32_t *>(half_area + lane * 4);
    }
}

// ------------------------------------------------------------------ kernel
// Exponent-only power of two (exact scaling), e in [-126, 127].
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Largest e with 2^e <= x (x > 0, normal).
__device__ __forceinline__ int floor_log2(float x) { return ((__float_as_int(x) >> 23) & 0xFF) - 127; }

__device__ __forceinline__ float half_lo_f(uint32_t w) { return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFF))); }
__device__ __forceinline__ float half_hi_f(uint32_t w) { return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16))); }

// hi/lo fp16 pair of x*s for a half2 x = xh + xl and a half2 s: hi = rn(xh*s),
// lo = rn(rn_exact(xh*s - hi) + xl*s); the residual xh*s - hi is exact in fp16 (FMA).
__device__ __forceinline__ void mul_hilo(uint32_t xh, uint32_t xl, uint32_t s, uint32_t &hi, uint32_t &lo) {
    const __half2 h = __hmul2(bits_h2(xh), bits_h2(s));
    const __half2 r = __hfma2(bits_h2(xh), bits_h2(s), __hneg2(h));
    lo = h2_bits(__hfma2(bits_h2(xl), bits_h2(s), r));
    hi = h2_bits(h);
}

// Split two floats into three bf16 pairs: hi and mid by 8-bit truncation (exact), lo the
// remainder rounded to bf16; hi + mid + lo carries 24 significant bits (error below
// 2^-24 of |v|), as much as the float itself.
__device__ __forceinline__ void split3_bf16(float a, float b, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
    const float ha = __uint_as_float(__float_as_uint(a) & 0xFFFF0000u);
    const float hb = __uint_as_float(__float_as_uint(b) & 0xFFFF0000u);
    hi = (__float_as_uint(ha) >> 16) | (__float_as_uint(hb) & 0xFFFF0000u);
    const float ra = a - ha, rb = b - hb;   // exact
    const float ma = __uint_as_float(__float_as_uint(ra) & 0xFFFF0000u);
    const float mb = __uint_as_float(__float_as_uint(rb) & 0xFFFF0000u);
    mid = (__float_as_uint(ma) >> 16) | (__float_as_uint(mb) & 0xFFFF0000u);
    const __nv_bfloat162 l = __floats2bfloat162_rn(ra - ma, rb - mb);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Split two floats into fp16 hi (11-bit truncation, exact) and lo (remainder) pairs.
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const float ha = trunc11(a), hb = trunc11(b);
    hi = pack_h2(ha, hb);
    lo = pack_h2(a - ha, b - hb);
}

// Bytes of one unit record: NH 16-token halves of codes, fp16 scales/zeros.
__host__ __device__ constexpr int unit_bytes(int D, int BK, int BV, int KM, int NH) {
    return 2 * NH * D * BK + (KM == 0 ? 4 * D : 2 * NH * D) + 2 * NH * D * BV + 2 * NH * D;
}

}  // namespace
}  // namespace kvq
