// Split-KV decode attention over the packed mixed-precision cache (sm_100a).
//
// Flash-decoding over the sequence with splits merged by log-sum-exp ("TriAxialKV
// per-role mixed-precision KV quantization", Facts: decode path; splits of one layer
// are bitwidth-homogeneous because the layer's precision pair is static, KVTuner
// summary, Approach), with dequantization folded into the tensor-core operands so
// codes never leave registers as anything but exact small integers:
//
//   keys per channel (group scale s_d, zero z_d over 32 tokens):
//     q.k^_t = sum_d (q_d s_d) c_td + sum_d q_d z_d
//     -> A operand = q_d s_d (fp16 hi + lo split, rows 0-7 hi, 8-15 lo), B = codes,
//        plus one per-group constant.
//   keys per token (scale s_tj, zero z_tj per 32 channels j):
//     q.k^_t = sum_j s_tj (sum_{d in j} q_d c_td) + sum_j z_tj (sum_{d in j} q_d)
//     -> A rows = (channel group j, head) with q masked to group j (bf16 q is exact in
//        fp16), the per-token scale applied to the fp32 accumulators.
//   values per token:
//     sum_t p_t v^_td = sum_t (p_t s_tj) c_td + sum_t p_t z_tj
//     -> A = value codes (channels x tokens), B = p_t s_tj (fp16 hi + lo columns).
//
// CTA = 4 warps for one (batch, kv head, split).  Each warp owns every 4th 32-token
// block of the split and streams the 32-token block records into a private ring of
// shared-memory stages with cp.async.bulk + mbarrier (bounded waits).  mma.sync
// m16n8k16 (fp16 in, fp32 accumulate) does both contractions; online softmax in
// base 2.  The last block of a per-channel layer takes its keys from the bf16
// residual.  Warps are combined in shared memory; one split writes the output
// directly, several write fp32 partials for the merge kernel.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int NW = kDecodeWarps;
constexpr float kLog2e = 1.4426950408889634f;

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
        : "r"(smem_u32(bar)), "r"(phase), "r"(1000000u)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after ~2^20 polls (each suspends at most ~1 ms).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned phase) {
    for (int i = 0; i < (1 << 20); ++i)
        if (mbar_try_wait(bar, phase)) return true;
    return false;
}

__device__ __forceinline__ void mma16816(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(orv));
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
__device__ __forceinline__ uint32_t hfma2_bits(uint32_t x, uint32_t m, uint32_t a) {
    return h2_bits(__hfma2(bits_h2(x), bits_h2(m), bits_h2(a)));
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) { return h2_bits(__floats2half2_rn(lo, hi)); }

// Exact fp16 pair of the two codes of slot p of a word: field p (low half) and field
// p + P (high half), P = 16/BITS.  Codes enter the fp16 mantissa under exponent 2^10
// (value 1024 + c, or 1024 + 2^k c) and the offset is removed exactly.
template <int BITS>
__device__ __forceinline__ uint32_t unpack(uint32_t w, int p) {
    constexpr uint32_t kMagic = 0x64006400u;   // (1024, 1024)
    if constexpr (BITS == 8) {
        const uint32_t sel = static_cast<uint32_t>(p) | 0x40u | (static_cast<uint32_t>(p + 2) << 8) | 0x4000u;
        return hsub2_bits(prmt(w, 0x64646464u, sel), kMagic);
    } else if constexpr (BITS == 4) {
        const uint32_t src = p < 2 ? w : (w >> 8);
        if ((p & 1) == 0) return hsub2_bits(lop_and_or(src, 0x000F000Fu, kMagic), kMagic);
        return hfma2_bits(lop_and_or(src, 0x00F000F0u, kMagic), 0x2C002C00u /*1/16*/, 0xD400D400u /*-64*/);
    } else {
        const uint32_t src = p < 4 ? w : (w >> 8);
        const int q = p & 3;
        const uint32_t x = lop_and_or(src, 0x00030003u << (2 * q), kMagic);
        if (q == 0) return hsub2_bits(x, kMagic);
        if (q == 1) return hfma2_bits(x, 0x34003400u /*1/4*/, 0xDC00DC00u /*-256*/);
        if (q == 2) return hfma2_bits(x, 0x2C002C00u /*1/16*/, 0xD400D400u /*-64*/);
        return hfma2_bits(x, 0x24002400u /*1/64*/, 0xCC00CC00u /*-16*/);
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
template <int BK, int BV, int KM, int D, int NT>
__global__ void __launch_bounds__(NW * 32, 3) decode_split_kernel(const DecodeParams p) {
    constexpr int KS = D / 16;     // 16-channel steps (QK) / 16-channel row tiles (PV)
    constexpr int NJ = D / 32;     // channel groups
    constexpr int WHK = D * BK / 64, WHV = D * BV / 64;
    constexpr int PK = 16 / BK, PV = 16 / BV;   // slots per word
    constexpr int KC = 4 * D * BK, KSZ = 4 * D, VC = 4 * D * BV;
    constexpr int REC = KC + KSZ + VC + 4 * D;

    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int b = blockIdx.z, h = blockIdx.y, sp = blockIdx.x;
    const int G = p.G, L = p.L, NS = p.nstage;
    const int nblk = (L + 31) >> 5;
    const int blk0 = sp * p.bps, blk1 = min(nblk, blk0 + p.bps);
    const int rem = L & 31;
    const int tail_blk = rem ? (L >> 5) : -1;

    uint8_t *stages = smem + static_cast<size_t>(warp) * NS * REC;
    const size_t stage_bytes = static_cast<size_t>(NW) * NS * REC;
    const size_t comb_bytes = static_cast<size_t>(NW) * (8 * NT * D + 8 * (2 + NJ)) * 4;
    const size_t bar_off = ((stage_bytes > comb_bytes ? stage_bytes : comb_bytes) + 127) & ~size_t(127);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + bar_off) + warp * NS;
    const uint8_t *unit_rec = p.rec + (static_cast<long long>(b) * p.Hkv + h) * p.cap_blk * REC;

    const int nb = (blk1 - blk0 > warp) ? (blk1 - blk0 - warp + NW - 1) / NW : 0;
    if (lane == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    int issued = 0;
    if (lane == 0) {
        for (; issued < NS && issued < nb; ++issued) {
            mbar_expect_tx(&bars[issued], REC);
            bulk_g2s(stages + issued * REC, unit_rec + static_cast<long long>(blk0 + warp + NW * issued) * REC,
                     REC, &bars[issued]);
        }
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);

    // ---- this thread's query head and channels (16k + 2t + {0, 1, 8, 9}) ----
    const int hh = g % G;
    const uint16_t *qrow = p.q + (static_cast<long long>(b) * p.Hkv * G + h * G + hh) * D;
    float qv[KS][4];
#pragma unroll
    for (int k = 0; k < KS; ++k) {
        const uint32_t a = *reinterpret_cast<const uint32_t *>(qrow + 16 * k + 2 * t);
        const uint32_t c = *reinterpret_cast<const uint32_t *>(qrow + 16 * k + 2 * t + 8);
        qv[k][0] = __uint_as_float(a << 16);
        qv[k][1] = __uint_as_float(a & 0xFFFF0000u);
        qv[k][2] = __uint_as_float(c << 16);
        qv[k][3] = __uint_as_float(c & 0xFFFF0000u);
    }
    const float qscale = kLog2e * rsqrtf(static_cast<float>(D));

    // per-token keys: constant masked A fragments (rows r = j*G + head) and q sums per group
    uint32_t aq[KM == 1 ? KS : 1][4];
    float qsum_g = 0.f, qsum_g8 = 0.f;   // sum of q over the channel group of rows g and g+8
    const int jg = g / G, jg8 = (g + 8) / G;
    const bool row_g = (KM == 1) && (g < G * NJ), row_g8 = (KM == 1) && (g + 8 < G * NJ);
    if constexpr (KM == 1) {
        float part[NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) part[j] = 0.f;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int j = k >> 1;
            part[j] += (qv[k][0] + qv[k][1]) + (qv[k][2] + qv[k][3]);
            const uint32_t lo = pack_h2(qv[k][0], qv[k][1]), hi = pack_h2(qv[k][2], qv[k][3]);
            aq[k][0] = (row_g && jg == j) ? lo : 0u;
            aq[k][1] = (row_g8 && jg8 == j) ? lo : 0u;
            aq[k][2] = (row_g && jg == j) ? hi : 0u;
            aq[k][3] = (row_g8 && jg8 == j) ? hi : 0u;
        }
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            part[j] += __shfl_xor_sync(0xffffffffu, part[j], 1);
            part[j] += __shfl_xor_sync(0xffffffffu, part[j], 2);
            if (j == (jg < NJ ? jg : 0)) qsum_g = part[j];
            if (j == (jg8 < NJ ? jg8 : 0)) qsum_g8 = part[j];
        }
    } else {
#pragma unroll
        for (int k = 0; k < KS; ++k)
#pragma unroll
            for (int c = 0; c < 4; ++c) qv[k][c] *= qscale;
    }

    float m_run = -INFINITY, l_run = 0.f;
    float zacc[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) zacc[j] = 0.f;
    float oacc[KS][NT][4];
#pragma unroll
    for (int m = 0; m < KS; ++m)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) oacc[m][n][c] = 0.f;

    // B-operand column of this thread for P (NT == 1: hi, lo or zero by column)
    const int col_kind = (NT == 1) ? (g < G ? 0 : (g < 2 * G ? 1 : 2)) : (g < G ? 0 : 2);
    const int alpha_src0 = 4 * ((NT == 1) ? ((2 * t) % G) : min(2 * t, 7));
    const int alpha_src1 = 4 * ((NT == 1) ? ((2 * t + 1) % G) : min(2 * t + 1, 7));

    bool failed = false;
    int i = 0;
    for (; i < nb; ++i) {
        const int blk = blk0 + warp + NW * i;
        const int st = i % NS;
        if (!mbar_wait(&bars[st], (i / NS) & 1)) {
            failed = true;
            break;
        }
        const uint8_t *R = stages + st * REC;
        const int valid = (blk == tail_blk) ? rem : 32;

        // ================= scores S^T (rows: heads, columns: 8-token tiles) =================
        float acc[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[n][c] = 0.f;
        float cz = 0.f;
        const bool resid_block = (KM == 0) && (blk == tail_blk);
        if (!resid_block) {
            uint32_t kw[2][WHK];
            load_lane_words<WHK>(R, lane, kw[0]);
            load_lane_words<WHK>(R + 2 * D * BK, lane, kw[1]);
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                uint32_t a[4];
                if constexpr (KM == 0) {
                    const int c0 = 16 * k + 2 * t;
                    const uint2 sz0 = *reinterpret_cast<const uint2 *>(R + KC + 4 * c0);
                    const uint2 sz8 = *reinterpret_cast<const uint2 *>(R + KC + 4 * (c0 + 8));
                    const __half2 s01 = __halves2half2(__ushort_as_half(sz0.x & 0xFFFF), __ushort_as_half(sz0.y & 0xFFFF));
                    const __half2 z01 = __halves2half2(__ushort_as_half(sz0.x >> 16), __ushort_as_half(sz0.y >> 16));
                    const __half2 s89 = __halves2half2(__ushort_as_half(sz8.x & 0xFFFF), __ushort_as_half(sz8.y & 0xFFFF));
                    const __half2 z89 = __halves2half2(__ushort_as_half(sz8.x >> 16), __ushort_as_half(sz8.y >> 16));
                    const float2 fs01 = __half22float2(s01), fz01 = __half22float2(z01);
                    const float2 fs89 = __half22float2(s89), fz89 = __half22float2(z89);
                    const float x0 = qv[k][0] * fs01.x, x1 = qv[k][1] * fs01.y;
                    const float x8 = qv[k][2] * fs89.x, x9 = qv[k][3] * fs89.y;
                    cz = fmaf(qv[k][0], fz01.x, cz);
                    cz = fmaf(qv[k][1], fz01.y, cz);
                    cz = fmaf(qv[k][2], fz89.x, cz);
                    cz = fmaf(qv[k][3], fz89.y, cz);
                    const float h0 = trunc11(x0), h1 = trunc11(x1), h8 = trunc11(x8), h9 = trunc11(x9);
                    a[0] = pack_h2(h0, h1);
                    a[1] = pack_h2(x0 - h0, x1 - h1);
                    a[2] = pack_h2(h8, h9);
                    a[3] = pack_h2(x8 - h8, x9 - h9);
                } else {
                    a[0] = aq[k][0];
                    a[1] = aq[k][1];
                    a[2] = aq[k][2];
                    a[3] = aq[k][3];
                }
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const int s0 = (2 * k + (n & 1)) * 2;
                    const uint32_t w = kw[n >> 1][s0 / PK];
                    mma16816(acc[n], a, unpack<BK>(w, s0 % PK), unpack<BK>(w, s0 % PK + 1));
                }
            }
        } else {
            // bf16 residual keys of the last, incomplete group (per-channel layers)
            const uint16_t *res = p.res + (static_cast<long long>(b) * p.Hkv + h) * 32 * D;
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                const float h0 = trunc11(qv[k][0]), h1 = trunc11(qv[k][1]);
                const float h8 = trunc11(qv[k][2]), h9 = trunc11(qv[k][3]);
                uint32_t a[4] = {pack_h2(h0, h1), pack_h2(qv[k][0] - h0, qv[k][1] - h1), pack_h2(h8, h9),
                                 pack_h2(qv[k][2] - h8, qv[k][3] - h9)};
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const int u = 8 * n + g;
                    uint32_t b0 = 0u, b1 = 0u;
                    if (u < valid) {
                        const uint32_t r0 = *reinterpret_cast<const uint32_t *>(res + u * D + 16 * k + 2 * t);
                        const uint32_t r8 = *reinterpret_cast<const uint32_t *>(res + u * D + 16 * k + 2 * t + 8);
                        b0 = pack_h2(__uint_as_float(r0 << 16), __uint_as_float(r0 & 0xFFFF0000u));
                        b1 = pack_h2(__uint_as_float(r8 << 16), __uint_as_float(r8 & 0xFFFF0000u));
                    }
                    mma16816(acc[n], a, b0, b1);
                }
            }
        }

        float sc[4][2];
        if constexpr (KM == 0) {
            cz += __shfl_xor_sync(0xffffffffu, cz, 1);
            cz += __shfl_xor_sync(0xffffffffu, cz, 2);
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                sc[n][0] = acc[n][0] + acc[n][2] + cz;
                sc[n][1] = acc[n][1] + acc[n][3] + cz;
            }
        } else {
            // per-token key scales, then sum the (group, head) rows of each head
#pragma unroll
            for (int n = 0; n < 4; ++n) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int u = 8 * n + 2 * t + c;
                    float v = 0.f;
                    if (row_g) {
                        const uint32_t e = *reinterpret_cast<const uint32_t *>(R + KC + 4 * (u * NJ + jg));
                        v = fmaf(__half2float(__ushort_as_half(e & 0xFFFF)), acc[n][c],
                                 __half2float(__ushort_as_half(e >> 16)) * qsum_g);
                    }
                    if (row_g8) {
                        const uint32_t e = *reinterpret_cast<const uint32_t *>(R + KC + 4 * (u * NJ + jg8));
                        v += fmaf(__half2float(__ushort_as_half(e & 0xFFFF)), acc[n][2 + c],
                                  __half2float(__ushort_as_half(e >> 16)) * qsum_g8);
                    }
#pragma unroll
                    for (int msk = G; msk < 8; msk <<= 1) v += __shfl_xor_sync(0xffffffffu, v, 4 * msk);
                    sc[n][c] = v * qscale;
                }
            }
        }
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int c = 0; c < 2; ++c)
                if (8 * n + 2 * t + c >= valid) sc[n][c] = -INFINITY;

        // ================= online softmax (base 2) =================
        float mloc = fmaxf(fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1])),
                           fmaxf(fmaxf(sc[2][0], sc[2][1]), fmaxf(sc[3][0], sc[3][1])));
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
        const float m_new = fmaxf(m_run, mloc);
        const float alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
        float pr[4][2];
        float psum = 0.f;
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                pr[n][c] = fast_exp2(sc[n][c] - m_new);
                psum += pr[n][c];
            }
        l_run = fmaf(l_run, alpha, psum);
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
            for (int j = 0; j < NJ; ++j) zacc[j] *= alpha;
            const float a0 = __shfl_sync(0xffffffffu, alpha, alpha_src0);
            const float a1 = __shfl_sync(0xffffffffu, alpha, alpha_src1);
#pragma unroll
            for (int m = 0; m < KS; ++m)
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    oacc[m][n][0] *= a0;
                    oacc[m][n][1] *= a1;
                    oacc[m][n][2] *= a0;
                    oacc[m][n][3] *= a1;
                }
        }

        // ================= O^T += V^T P'^T (two 16-token steps) =================
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            uint32_t vw[WHV];
            load_lane_words<WHV>(R + KC + KSZ + kk * 2 * D * BV, lane, vw);
            const float pt[4] = {pr[2 * kk][0], pr[2 * kk][1], pr[2 * kk + 1][0], pr[2 * kk + 1][1]};
            const int ut[4] = {16 * kk + 2 * t, 16 * kk + 2 * t + 1, 16 * kk + 8 + 2 * t, 16 * kk + 9 + 2 * t};
            uint32_t szv[4][NJ];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint8_t *src = R + KC + KSZ + VC + 4 * (ut[e] * NJ);
                if constexpr (NJ == 4) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(src);
                    szv[e][0] = v.x;
                    szv[e][1] = v.y;
                    szv[e][2] = v.z;
                    szv[e][3] = v.w;
                } else if constexpr (NJ == 2) {
                    const uint2 v = *reinterpret_cast<const uint2 *>(src);
                    szv[e][0] = v.x;
                    szv[e][1] = v.y;
                } else {
#pragma unroll
                    for (int j = 0; j < NJ; ++j) szv[e][j] = reinterpret_cast<const uint32_t *>(src)[j];
                }
            }
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                float pp[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float s = __half2float(__ushort_as_half(szv[e][j] & 0xFFFF));
                    const float z = __half2float(__ushort_as_half(szv[e][j] >> 16));
                    const bool live = pt[e] != 0.0f;
                    pp[e] = live ? pt[e] * s : 0.f;
                    zacc[j] += live ? pt[e] * z : 0.f;
                }
                uint32_t bh0, bh1, bl0 = 0u, bl1 = 0u;
                {
                    const float h0 = trunc11(pp[0]), h1 = trunc11(pp[1]), h2 = trunc11(pp[2]), h3 = trunc11(pp[3]);
                    if constexpr (NT == 1) {
                        const float v0 = col_kind == 0 ? h0 : (col_kind == 1 ? pp[0] - h0 : 0.f);
                        const float v1 = col_kind == 0 ? h1 : (col_kind == 1 ? pp[1] - h1 : 0.f);
                        const float v2 = col_kind == 0 ? h2 : (col_kind == 1 ? pp[2] - h2 : 0.f);
                        const float v3 = col_kind == 0 ? h3 : (col_kind == 1 ? pp[3] - h3 : 0.f);
                        bh0 = pack_h2(v0, v1);
                        bh1 = pack_h2(v2, v3);
                    } else {
                        const bool on = col_kind == 0;
                        bh0 = on ? pack_h2(h0, h1) : 0u;
                        bh1 = on ? pack_h2(h2, h3) : 0u;
                        bl0 = on ? pack_h2(pp[0] - h0, pp[1] - h1) : 0u;
                        bl1 = on ? pack_h2(pp[2] - h2, pp[3] - h3) : 0u;
                    }
                }
#pragma unroll
                for (int mm = 0; mm < 2; ++mm) {
                    const int m = 2 * j + mm;
                    uint32_t a[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int s = 4 * m + r;
                        a[r] = unpack<BV>(vw[s / PV], s % PV);
                    }
                    mma16816(oacc[m][0], a, bh0, bh1);
                    if constexpr (NT == 2) mma16816(oacc[m][NT - 1], a, bl0, bl1);
                }
            }
        }

        __syncwarp();
        if (lane == 0 && issued < nb) {
            fence_proxy_async();
            const int ni = issued++;
            mbar_expect_tx(&bars[st], REC);
            bulk_g2s(stages + st * REC, unit_rec + static_cast<long long>(blk0 + warp + NW * ni) * REC, REC,
                     &bars[st]);
        }
        issued = __shfl_sync(0xffffffffu, issued, 0);
    }
    if (failed) {
        // drain the copies still in flight (bounded), then report
        for (int k = i; k < issued; ++k) mbar_wait(&bars[k % NS], (k / NS) & 1);
        if (lane == 0) atomicOr(p.status, kStatusWaitExpired);
    }

    // ================= combine the warps of this split =================
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        zacc[j] += __shfl_xor_sync(0xffffffffu, zacc[j], 1);
        zacc[j] += __shfl_xor_sync(0xffffffffu, zacc[j], 2);
    }
    __syncthreads();   // every warp is done with its stages
    float *obuf = reinterpret_cast<float *>(smem);                 // [NW][8*NT][D]
    float *mbuf = obuf + NW * 8 * NT * D;                          // [NW][8]
    float *lbuf = mbuf + NW * 8;                                   // [NW][8]
    float *zbuf = lbuf + NW * 8;                                   // [NW][8][NJ]
    {
        float *ob = obuf + warp * 8 * NT * D;
#pragma unroll
        for (int m = 0; m < KS; ++m)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int d0 = 16 * m + g, c0 = 8 * n + 2 * t;
                ob[c0 * D + d0] = oacc[m][n][0];
                ob[(c0 + 1) * D + d0] = oacc[m][n][1];
                ob[c0 * D + d0 + 8] = oacc[m][n][2];
                ob[(c0 + 1) * D + d0 + 8] = oacc[m][n][3];
            }
        if (t == 0 && g < G) {
            mbuf[warp * 8 + g] = (nb > 0 && !failed) ? m_run : -INFINITY;
            lbuf[warp * 8 + g] = l_run;
#pragma unroll
            for (int j = 0; j < NJ; ++j) zbuf[(warp * 8 + g) * NJ + j] = zacc[j];
        }
    }
    __syncthreads();
    const int Hq = p.Hkv * G;
    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
        const int hd = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, mbuf[w * 8 + hd]);
        float val = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float mw = mbuf[w * 8 + hd];
            if (mw == -INFINITY) continue;
            const float wt = fast_exp2(mw - M);
            const float *ob = obuf + w * 8 * NT * D;
            const float o = (NT == 1) ? ob[hd * D + d] + ob[(hd + G) * D + d] : ob[hd * D + d] + ob[(8 + hd) * D + d];
            val = fmaf(wt, o + zbuf[(w * 8 + hd) * NJ + d / 32], val);
            den = fmaf(wt, lbuf[w * 8 + hd], den);
        }
        const long long row = static_cast<long long>(b) * Hq + h * G + hd;
        if (p.S == 1) {
            const float o = val / den;
            if (p.out_fp32) reinterpret_cast<float *>(p.out)[row * D + d] = o;
            else reinterpret_cast<__nv_bfloat16 *>(p.out)[row * D + d] = __float2bfloat16_rn(o);
        } else {
            p.part_acc[(row * kMaxSplits + sp) * D + d] = val;
            if (d == 0) {
                p.part_ml[(row * kMaxSplits + sp) * 2] = M;
                p.part_ml[(row * kMaxSplits + sp) * 2 + 1] = den;
            }
        }
    }
}

// Log-sum-exp merge of the split partials ("merged by online log-sum-exp").
__global__ void merge_kernel(const MergeParams p) {
    const long long row = blockIdx.x;   // b * Hq + hq
    const float *ml = p.part_ml + row * kMaxSplits * 2;
    float M = -INFINITY;
    for (int s = 0; s < p.S; ++s) M = fmaxf(M, ml[2 * s]);
    for (int d = threadIdx.x; d < p.D; d += blockDim.x) {
        float val = 0.f, den = 0.f;
        for (int s = 0; s < p.S; ++s) {
            const float ms = ml[2 * s];
            if (ms == -INFINITY) continue;
            const float wt = fast_exp2(ms - M);
            val = fmaf(wt, p.part_acc[(row * kMaxSplits + s) * p.D + d], val);
            den = fmaf(wt, ml[2 * s + 1], den);
        }
        const float o = val / den;
        if (p.out_fp32) reinterpret_cast<float *>(p.out)[row * p.D + d] = o;
        else reinterpret_cast<__nv_bfloat16 *>(p.out)[row * p.D + d] = __float2bfloat16_rn(o);
    }
}

using KernelFn = void (*)(const DecodeParams);

template <int D, int NT, int KM>
KernelFn pick_bits(int bk, int bv) {
#define KVQ_CASE(BKv, BVv) \
    if (bk == BKv && bv == BVv) return decode_split_kernel<BKv, BVv, KM, D, NT>;
    KVQ_CASE(2, 2) KVQ_CASE(2, 4) KVQ_CASE(2, 8)
    KVQ_CASE(4, 2) KVQ_CASE(4, 4) KVQ_CASE(4, 8)
    KVQ_CASE(8, 2) KVQ_CASE(8, 4) KVQ_CASE(8, 8)
#undef KVQ_CASE
    return nullptr;
}

KernelFn pick_kernel(int D, int bk, int bv, int kmode, int G) {
    const int NT = G <= 4 ? 1 : 2;
    if (G < 1 || G > 8) return nullptr;
    if (kmode == 1) {
        // rows (group, head) must fit one 16-row tile and heads must divide 8
        if (!(G == 1 || G == 2 || G == 4) || G * (D / 32) > 16) return nullptr;
        if (D == 64) return pick_bits<64, 1, 1>(bk, bv);
        if (D == 128) return pick_bits<128, 1, 1>(bk, bv);
        return nullptr;
    }
    if (D == 64) return NT == 1 ? pick_bits<64, 1, 0>(bk, bv) : pick_bits<64, 2, 0>(bk, bv);
    if (D == 128) return NT == 1 ? pick_bits<128, 1, 0>(bk, bv) : pick_bits<128, 2, 0>(bk, bv);
    return nullptr;
}

}  // namespace

int decode_stages(long long rec_bytes) {
    long long ns = 65536 / (NW * rec_bytes);
    if (ns < 2) ns = 2;
    if (ns > 6) ns = 6;
    return static_cast<int>(ns);
}

size_t decode_smem_bytes(long long rec_bytes, int nstage, int D, int G) {
    const int NT = G <= 4 ? 1 : 2;
    const size_t stage = static_cast<size_t>(NW) * nstage * rec_bytes;
    const size_t comb = static_cast<size_t>(NW) * (8 * NT * D + 8 * (2 + D / 32)) * 4;
    const size_t base = ((stage > comb ? stage : comb) + 127) & ~size_t(127);
    return base + static_cast<size_t>(NW) * nstage * 8;
}

cudaError_t decode_occupancy(int D, int bk, int bv, int kmode, int G, long long rec_bytes, int nstage,
                             int *ctas_per_sm) {
    KernelFn fn = pick_kernel(D, bk, bv, kmode, G);
    if (!fn) return cudaErrorInvalidValue;
    const size_t smem = decode_smem_bytes(rec_bytes, nstage, D, G);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, fn, NW * 32, smem);
}

cudaError_t launch_decode(const DecodeParams &p, int D, int bk, int bv, int kmode, cudaStream_t st,
                          int *ctas_per_sm_out) {
    KernelFn fn = pick_kernel(D, bk, bv, kmode, p.G);
    if (!fn) return cudaErrorInvalidValue;
    const size_t smem = decode_smem_bytes(p.rec_bytes, p.nstage, D, p.G);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    (void)ctas_per_sm_out;
    dim3 grid(p.S, p.Hkv, p.B);
    fn<<<grid, NW * 32, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_merge(const MergeParams &p, cudaStream_t st) {
    merge_kernel<<<p.B * p.Hq, p.D, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace kvq
