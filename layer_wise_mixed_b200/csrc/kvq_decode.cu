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
// directly, several write fp32 partials that the (batch, kv head)'s last CTA to finish
// merges by log-sum-exp.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>
#include <type_traits>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_quant.cuh"

namespace kvq {
namespace {

constexpr int NW = kDecodeWarps;
constexpr float kLog2e = 1.4426950408889634f;

// Floats of the per-warp combine buffer: O^T columns [8 NT][D + 4], value zero-point
// terms [D/32][8 NT], running max and sum per head [8] + [8].
__host__ __device__ constexpr int comb_floats(int D, int NT) { return 8 * NT * (D + 4) + (D / 32) * 8 * NT + 16; }

// Per-thread constants of the block body.
struct BodyCtx {
    const uint4 *aq_s;          // q operand fragments in shared memory: [KS][32] fp16 hi/lo,
                                // then (per-channel keys) [KS][32] bf16 hi/mid and [KS][32]
                                // bf16 lo (as uint4 {lo, 0, lo', 0}) for the residual
    const uint16_t *res;        // bf16 residual keys of this (b, h) (per-channel tail) or null
    int lane, g, t, G, jg, jg8, jz, alpha_src0, alpha_src1;
    bool row_g, row_g8;
    uint32_t m_hi;
    float unscale, qsum_g, qsum_g8, pbias;
};

template <int D, int NT>
struct WarpAcc {
    float m_run, l_run;
    float oacc[D / 16][NT][4];
    float zc[NT][4];            // value zero-point term: rows = channel group j (= g)
};

// Query setup: q~ fragments into shared memory (written by warp 0), score scaling.
//  per-channel keys: q~ = q log2(e)/sqrt(D) 2^kq as fp16 hi/lo (rows g: hi, g+8: lo),
//    kq chosen so that q~ s_k < 2^14 and q~ < 2^15; scores = raw * 2^-kq.  The same q~
//    as bf16 hi/mid/lo parts for the bf16 residual keys of the open group (bf16
//    operands take the residual rows as they are, at any magnitude, with no fp16
//    conversion; three parts keep q~'s 24 bits).
//  per-token keys: q~ = q 2^kq with kq chosen so that |q~| < 2^15 (a bf16 value times a
//    power of two is exact in fp16 down to 2^-14 of that bound; smaller entries lose
//    bits far below the largest product), rows (group j, head) masked to group j;
//    scores = raw * log2(e)/sqrt(D) * 2^-kq.
// kq is clamped so that 2^kq and 2^-kq stay normal binary32 numbers.
// Computed by warp 0 only; every lane's scalars (unscale, qsum_g, qsum_g8) go to
// scal_s[lane] for the other warps (load_query_scalars after a CTA barrier).
template <int KM, int D, int NT>
__device__ __forceinline__ void setup_query(const uint16_t *qrow, float smax_k, uint4 *aq_s, float4 *scal_s,
                                            BodyCtx &c, int warp) {
    constexpr int KS = D / 16, NJ = D / 32;
    if (warp != 0) return;
    const int t = c.t;
    float qv[KS][4];
#pragma unroll
    for (int k = 0; k < KS; ++k) {
        const uint32_t a = *reinterpret_cast<const uint32_t *>(qrow + 16 * k + 2 * t);
        const uint32_t b = *reinterpret_cast<const uint32_t *>(qrow + 16 * k + 2 * t + 8);
        qv[k][0] = __uint_as_float(a << 16);
        qv[k][1] = __uint_as_float(a & 0xFFFF0000u);
        qv[k][2] = __uint_as_float(b << 16);
        qv[k][3] = __uint_as_float(b & 0xFFFF0000u);
    }
    const float qscale = kLog2e * rsqrtf(static_cast<float>(D));
    uint32_t aq[KS][4];
    c.qsum_g = c.qsum_g8 = 0.f;
    // the head's largest |q| (times the score scale for per-channel keys): the 4 lanes
    // of a row group hold all D channels of head hh
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < KS; ++k)
#pragma unroll
        for (int x = 0; x < 4; ++x) amax = fmaxf(amax, fabsf(KM == 0 ? qv[k][x] * qscale : qv[k][x]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int kq = 0;
    if (amax > 0.f) {
        kq = 14 - floor_log2(amax);                                                                // q~ < 2^15
        if (KM == 0 && smax_k > 0.f) kq = min(kq, 12 - floor_log2(amax) - floor_log2(smax_k));   // q~ s < 2^14
        kq = max(-120, min(100, kq));
    }
    if constexpr (KM == 0) {
        const float sc = qscale * pow2f(kq);
        c.unscale = pow2f(-kq);
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            split2(qv[k][0] * sc, qv[k][1] * sc, aq[k][0], aq[k][1]);
            split2(qv[k][2] * sc, qv[k][3] * sc, aq[k][2], aq[k][3]);
            uint32_t h0, m0, l0, h2, m2, l2;
            split3_bf16(qv[k][0] * sc, qv[k][1] * sc, h0, m0, l0);
            split3_bf16(qv[k][2] * sc, qv[k][3] * sc, h2, m2, l2);
            if constexpr (NT == 1) {   // one MMA: rows 0-3 hi, 4-7 mid, 8-11 lo (head g % G on every lane)
                aq_s[(KS + k) * 32 + c.lane] = c.g < 4 ? make_uint4(h0, l0, h2, l2) : make_uint4(m0, 0u, m2, 0u);
            } else {        // two MMAs: rows g hi and g + 8 mid, then rows g lo
                aq_s[(KS + k) * 32 + c.lane] = make_uint4(h0, m0, h2, m2);
                aq_s[(2 * KS + k) * 32 + c.lane] = make_uint4(l0, 0u, l2, 0u);
            }
        }
    } else {
        const float sc = pow2f(kq);
#pragma unroll
        for (int k = 0; k < KS; ++k)
#pragma unroll
            for (int x = 0; x < 4; ++x) qv[k][x] *= sc;
        float part[NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) part[j] = 0.f;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int j = k >> 1;
            part[j] += (qv[k][0] + qv[k][1]) + (qv[k][2] + qv[k][3]);
            const uint32_t lo = pack_h2(qv[k][0], qv[k][1]), hi = pack_h2(qv[k][2], qv[k][3]);
            aq[k][0] = (c.row_g && c.jg == j) ? lo : 0u;
            aq[k][1] = (c.row_g8 && c.jg8 == j) ? lo : 0u;
            aq[k][2] = (c.row_g && c.jg == j) ? hi : 0u;
            aq[k][3] = (c.row_g8 && c.jg8 == j) ? hi : 0u;
        }
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            part[j] += __shfl_xor_sync(0xffffffffu, part[j], 1);
            part[j] += __shfl_xor_sync(0xffffffffu, part[j], 2);
            if (j == (c.jg < NJ ? c.jg : 0)) c.qsum_g = part[j];
            if (j == (c.jg8 < NJ ? c.jg8 : 0)) c.qsum_g8 = part[j];
        }
        c.unscale = qscale * pow2f(-kq);
    }
#pragma unroll
    for (int k = 0; k < KS; ++k) aq_s[k * 32 + c.lane] = make_uint4(aq[k][0], aq[k][1], aq[k][2], aq[k][3]);
    scal_s[c.lane] = make_float4(c.unscale, c.qsum_g, c.qsum_g8, 0.f);
}

__device__ __forceinline__ void load_query_scalars(BodyCtx &c, const float4 *scal_s) {
    const float4 v = scal_s[c.lane];
    c.unscale = v.x;
    c.qsum_g = v.y;
    c.qsum_g8 = v.z;
}

// Exponent kp of the power of two carried by p: p * 2^kp * s_v stays below 2^14 in fp16.
__device__ __forceinline__ float value_bias(float smax_v) {
    const int kp = smax_v > 0.f ? max(-24, min(14, 13 - floor_log2(smax_v))) : 14;
    return static_cast<float>(kp);
}

// Thread constants that depend only on the lane, the group size and the layer scales.
template <int KM, int D, int NT>
__device__ __forceinline__ BodyCtx make_ctx(int lane, int G, float smax_v, const uint4 *aq_s) {
    constexpr int NJ = D / 32;
    BodyCtx c{};
    c.aq_s = aq_s;
    c.lane = lane;
    c.g = lane >> 2;
    c.t = lane & 3;
    c.G = G;
    c.jg = c.g / G;
    c.jg8 = (c.g + 8) / G;
    c.row_g = (KM == 1) && (c.g < G * NJ);
    c.row_g8 = (KM == 1) && (c.g + 8 < G * NJ);
    c.jz = c.g < NJ ? c.g : NJ - 1;
    // B-operand column of this thread for P: NT == 1: hi (g < G), else lo (columns 2G..
    // are computed but never read); NT == 2: tile 0 hi, tile 1 lo.
    c.m_hi = (c.g < G) ? 0xFFFFFFFFu : 0u;
    c.alpha_src0 = 4 * ((NT == 1) ? ((2 * c.t) % G) : min(2 * c.t, 7));
    c.alpha_src1 = 4 * ((NT == 1) ? ((2 * c.t + 1) % G) : min(2 * c.t + 1, 7));
    c.pbias = value_bias(smax_v);
    return c;
}

template <int D, int NT>
__device__ __forceinline__ void acc_init(WarpAcc<D, NT> &A) {
    A.m_run = -INFINITY;
    A.l_run = 0.f;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int x = 0; x < 4; ++x) A.zc[n][x] = 0.f;
#pragma unroll
        for (int m = 0; m < D / 16; ++m)
#pragma unroll
            for (int x = 0; x < 4; ++x) A.oacc[m][n][x] = 0.f;
    }
}

// One unit of NH 16-token halves (32-token block record, or 16-token page when NH = 1)
// staged at R, of which the first NHP are processed (NHP = 1: a tail block whose tokens
// all sit in its first half); `valid` tokens are present (TAIL: valid may be < 16 NH; per-channel
// TAIL blocks take their keys from the bf16 residual).
// PAIR: R holds two 16-token pages (per-token keys), one per half, each laid out
// [K codes][K scales/zeros][V codes][V scales/zeros], instead of one 32-token record.
template <int BK, int BV, int KM, int D, int NT, int NH, bool TAIL, bool PAIR = false, int NHP = NH>
__device__ __forceinline__ void process_unit(WarpAcc<D, NT> &A, const uint8_t *R, const int valid,
                                             const BodyCtx &c) {
    constexpr int KS = D / 16;
    constexpr int NJ = D / 32;
    constexpr int NTOK = 16 * NH;        // tokens in the unit
    constexpr int NTI = 2 * NHP;         // 8-token score tiles processed
    static_assert(NHP >= 1 && NHP <= NH && (NHP == NH || TAIL), "a partial unit is a tail");
    constexpr int WHK = D * BK / 64, WHV = D * BV / 64;
    constexpr int PK = 16 / BK, PV = 16 / BV;
    constexpr int KC = 2 * NH * D * BK, KSZ = (KM == 0 ? 4 * D : 2 * NH * D), VC = 2 * NH * D * BV;
    static_assert(KM == 1 || NH == 2, "per-channel keys come in 32-token groups");
    static_assert(!PAIR || (KM == 1 && NH == 2), "page pairs hold per-token keys");
    // areas of half hf (record: the halves share each area; pair: one page per half)
    constexpr int KCH = 2 * D * BK, KSZH = 2 * D, VCH = 2 * D * BV, PAGE = KCH + KSZH + VCH + 2 * D;
    auto kcode = [&](int hf) { return R + (PAIR ? hf * PAGE : hf * KCH); };
    auto ksz_pair = [&](int pi) { return PAIR ? R + (pi >> 3) * PAGE + KCH + 8 * NJ * (pi & 7) : R + KC + 8 * NJ * pi; };
    auto vcode = [&](int kk) { return PAIR ? R + kk * PAGE + KCH + KSZH : R + KC + KSZ + kk * VCH; };
    auto vsz_pair = [&](int kk, int i) {
        return PAIR ? R + kk * PAGE + KCH + KSZH + VCH + 8 * NJ * (i - 8 * kk) : R + KC + KSZ + VC + 8 * NJ * i;
    };
    const int lane = c.lane, g = c.g, t = c.t;

    // ===== scores S^T (rows: heads, columns: 8-token tiles) =====
    float acc[NTI][4];
#pragma unroll
    for (int n = 0; n < NTI; ++n)
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[n][x] = 0.f;
    float czacc[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (KM == 0 && TAIL) {
        // bf16 residual keys of the last, incomplete group: bf16 MMAs with the three bf16
        // query parts (packed into one MMA's rows, or hi/mid then lo), the rows taken as
        // stored
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const uint4 aqv = c.aq_s[(KS + k) * 32 + lane];
            const uint32_t ak[4] = {aqv.x, aqv.y, aqv.z, aqv.w};
            uint32_t al[4] = {0u, 0u, 0u, 0u};
            if constexpr (NT == 2) {
                const uint4 aql = c.aq_s[(2 * KS + k) * 32 + lane];
                al[0] = aql.x;
                al[2] = aql.z;
            }
#pragma unroll
            for (int n = 0; n < NTI; ++n) {
                const int u = 8 * n + g;
                uint32_t b0 = 0u, b1 = 0u;
                if (u < valid) {
                    b0 = *reinterpret_cast<const uint32_t *>(c.res + u * D + 16 * k + 2 * t);
                    b1 = *reinterpret_cast<const uint32_t *>(c.res + u * D + 16 * k + 2 * t + 8);
                }
                mma16816_bf16(acc[n], ak, b0, b1);
                if constexpr (NT == 2) mma16816_bf16(acc[n], al, b0, b1);
            }
        }
    } else {
        // key words of k-step k: slots 4k..4k+3 of each half, lane word (4k + x) / PK
        constexpr int WPK = PK >= 4 ? 1 : 4 / PK;   // words per k-step and half
        constexpr int CH = WHK < 4 ? WHK : 4;        // lane words per chunk
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            uint32_t kw[NHP][WPK];
            const int w0 = (4 * k) / PK;
#pragma unroll
            for (int x = 0; x < WPK; ++x) {
                const int w = w0 + x;
                const int off = (((w / CH) * 32 + lane) * CH + (w % CH)) * 4;
#pragma unroll
                for (int hf = 0; hf < NHP; ++hf) kw[hf][x] = *reinterpret_cast<const uint32_t *>(kcode(hf) + off);
            }
            const uint4 aqv = c.aq_s[k * 32 + lane];
            const uint32_t ak[4] = {aqv.x, aqv.y, aqv.z, aqv.w};
            uint32_t a[4];
            if constexpr (KM == 0) {
                // scales/zeros of channels (16k+2t, +1) and (16k+2t+8, +9) as half2
                const uint4 sz = *reinterpret_cast<const uint4 *>(R + KC + 16 * (4 * k + t));
                mul_hilo(ak[0], ak[1], sz.x, a[0], a[1]);
                mul_hilo(ak[2], ak[3], sz.z, a[2], a[3]);
                mma16816(czacc, ak, sz.y, sz.w);   // sum_d q~_d z_d, same in every column
            } else {
                a[0] = ak[0];
                a[1] = ak[1];
                a[2] = ak[2];
                a[3] = ak[3];
            }
#pragma unroll
            for (int n = 0; n < NTI; ++n) {
                const int s0 = (2 * k + (n & 1)) * 2;
                const int wl = s0 / PK - w0;
                const uint32_t w = kw[n >> 1][wl];
                mma16816(acc[n], a, unpack<BK>(w, s0 % PK), unpack<BK>(w, s0 % PK + 1));
            }
        }
    }

    float raw[NTI][2];
    if constexpr (KM == 0) {
        const float cz = czacc[0] + czacc[2];
#pragma unroll
        for (int n = 0; n < NTI; ++n) {
            raw[n][0] = acc[n][0] + acc[n][2] + cz;
            raw[n][1] = acc[n][1] + acc[n][3] + cz;
        }
        if constexpr (TAIL) {
            if constexpr (NT == 1) {   // rows g (hi, lo) and g ^ 4 (mid) of the packed residual MMA
#pragma unroll
                for (int n = 0; n < NTI; ++n) {
                    raw[n][0] += __shfl_xor_sync(0xffffffffu, raw[n][0], 16);
                    raw[n][1] += __shfl_xor_sync(0xffffffffu, raw[n][1], 16);
                }
            }
        }
    } else {
        // per-token key scales on the (group, head) rows, then sum the rows of a head
#pragma unroll
        for (int n = 0; n < NTI; ++n) {
            const int pi = 4 * n + t;   // token pair (8n + 2t, 8n + 2t + 1)
            const uint8_t *kp = ksz_pair(pi);
            float v0 = 0.f, v1 = 0.f;
            if (c.row_g) {
                const uint32_t sw = *reinterpret_cast<const uint32_t *>(kp + 4 * c.jg);
                const uint32_t zw = *reinterpret_cast<const uint32_t *>(kp + 4 * NJ + 4 * c.jg);
                v0 = fmaf(half_lo_f(sw), acc[n][0], half_lo_f(zw) * c.qsum_g);
                v1 = fmaf(half_hi_f(sw), acc[n][1], half_hi_f(zw) * c.qsum_g);
            }
            if (c.row_g8) {
                const uint32_t sw = *reinterpret_cast<const uint32_t *>(kp + 4 * c.jg8);
                const uint32_t zw = *reinterpret_cast<const uint32_t *>(kp + 4 * NJ + 4 * c.jg8);
                v0 += fmaf(half_lo_f(sw), acc[n][2], half_lo_f(zw) * c.qsum_g8);
                v1 += fmaf(half_hi_f(sw), acc[n][3], half_hi_f(zw) * c.qsum_g8);
            }
#pragma unroll
            for (int msk = c.G; msk < 8; msk <<= 1) {
                v0 += __shfl_xor_sync(0xffffffffu, v0, 4 * msk);
                v1 += __shfl_xor_sync(0xffffffffu, v1, 4 * msk);
            }
            raw[n][0] = v0;
            raw[n][1] = v1;
        }
    }
    if constexpr (TAIL) {
#pragma unroll
        for (int n = 0; n < NTI; ++n)
#pragma unroll
            for (int x = 0; x < 2; ++x)
                if (8 * n + 2 * t + x >= valid) raw[n][x] = -INFINITY;
    }

    // ===== online softmax (base 2; p carries the factor 2^kp) =====
    float mloc = -INFINITY;
#pragma unroll
    for (int n = 0; n < NTI; ++n) mloc = fmaxf(mloc, fmaxf(raw[n][0], raw[n][1]));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
    const float m_new = fmaxf(A.m_run, mloc * c.unscale);
    const float alpha = fast_exp2(A.m_run - m_new);
    A.m_run = m_new;
    const float shift = c.pbias - m_new;
    float pr[NTI][2];
    float psum = 0.f;
#pragma unroll
    for (int n = 0; n < NTI; ++n)
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            pr[n][x] = fast_exp2(fmaf(raw[n][x], c.unscale, shift));
            psum += pr[n][x];
        }
    A.l_run = fmaf(A.l_run, alpha, psum);
    if (__any_sync(0xffffffffu, alpha != 1.0f)) {
        const float a0 = __shfl_sync(0xffffffffu, alpha, c.alpha_src0);
        const float a1 = __shfl_sync(0xffffffffu, alpha, c.alpha_src1);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            A.zc[n][0] *= a0;
            A.zc[n][1] *= a1;
#pragma unroll
            for (int m = 0; m < KS; ++m) {
                A.oacc[m][n][0] *= a0;
                A.oacc[m][n][1] *= a1;
                A.oacc[m][n][2] *= a0;
                A.oacc[m][n][3] *= a1;
            }
        }
    }

    // ===== O^T += V^T P'^T and the zero-point term (16-token steps) =====
#pragma unroll
    for (int kk = 0; kk < NHP; ++kk) {
        uint32_t vw[WHV];
        load_lane_words<WHV>(vcode(kk), lane, vw);
        uint32_t pah, pal, pbh, pbl;   // p of token pairs A (16kk+2t, +1) and B (+8, +9)
        split2(pr[2 * kk][0], pr[2 * kk][1], pah, pal);
        split2(pr[2 * kk + 1][0], pr[2 * kk + 1][1], pbh, pbl);
        const int iA = 8 * kk + t, iB = iA + 4;
        const uint8_t *vsA = vsz_pair(kk, iA), *vsB = vsz_pair(kk, iB);
        uint32_t sA[NJ], sB[NJ];
        if constexpr (NJ == 4) {
            const uint4 xa = *reinterpret_cast<const uint4 *>(vsA);
            const uint4 xb = *reinterpret_cast<const uint4 *>(vsB);
            sA[0] = xa.x; sA[1] = xa.y; sA[2] = xa.z; sA[3] = xa.w;
            sB[0] = xb.x; sB[1] = xb.y; sB[2] = xb.z; sB[3] = xb.w;
        } else {
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                sA[j] = reinterpret_cast<const uint32_t *>(vsA)[j];
                sB[j] = reinterpret_cast<const uint32_t *>(vsB)[j];
            }
        }
        uint32_t zA = *reinterpret_cast<const uint32_t *>(vsA + 4 * NJ + 4 * c.jz);
        uint32_t zB = *reinterpret_cast<const uint32_t *>(vsB + 4 * NJ + 4 * c.jz);
        if constexpr (TAIL) {
            // absent tokens: p = 0 and their scale/zero halves may hold anything
            const int u0 = 16 * kk + 2 * t;
            const uint32_t mA = (u0 < valid ? 0x0000FFFFu : 0u) | (u0 + 1 < valid ? 0xFFFF0000u : 0u);
            const uint32_t mB = (u0 + 8 < valid ? 0x0000FFFFu : 0u) | (u0 + 9 < valid ? 0xFFFF0000u : 0u);
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                sA[j] &= mA;
                sB[j] &= mB;
            }
            zA &= mA;
            zB &= mB;
        }
        // zero-point term: rows j = g of Z^T (tokens as columns) times the P columns
        // (rows g >= NJ load group NJ - 1 and are never read)
        {
            const uint32_t az[4] = {zA, 0u, zB, 0u};
            if constexpr (NT == 1) {
                mma16816(A.zc[0], az, lop_sel(pah, pal, c.m_hi), lop_sel(pbh, pbl, c.m_hi));
            } else {
                mma16816(A.zc[0], az, pah, pbh);
                mma16816(A.zc[1], az, pal, pbl);
            }
        }
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            uint32_t ah, al, bh, bl;
            mul_hilo(pah, pal, sA[j], ah, al);
            mul_hilo(pbh, pbl, sB[j], bh, bl);
            uint32_t b0, b1, c0 = 0u, c1 = 0u;
            if constexpr (NT == 1) {
                b0 = lop_sel(ah, al, c.m_hi);
                b1 = lop_sel(bh, bl, c.m_hi);
            } else {
                b0 = ah;
                b1 = bh;
                c0 = al;
                c1 = bl;
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
                mma16816(A.oacc[m][0], a, b0, b1);
                if constexpr (NT == 2) mma16816(A.oacc[m][NT - 1], a, c0, c1);
            }
        }
    }
    (void)NTOK;
}

// Per-warp ring of NS shared-memory stages filled by cp.async.bulk (one elected lane),
// completion tracked by one mbarrier per stage with bounded waits.
struct WarpPipe {
    uint8_t *stages;
    uint64_t *bars;
    int NS, stage_bytes, lane;
    int issued, st;   // units issued so far; stage of the next unit to consume
    unsigned ph;      // its mbarrier phase
    int ist;          // stage of the next unit to issue
};

__device__ __forceinline__ void pipe_init(WarpPipe &P) {
    if (P.lane == 0) {
        for (int s = 0; s < P.NS; ++s) mbar_init(&P.bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    P.issued = 0;
    P.st = 0;
    P.ph = 0;
    P.ist = 0;
}

// Issue the copy of the next unit (bytes from src, landing `skip` bytes into the stage)
// into the next free stage; stages are refilled in the order they are consumed, so the
// next free stage is P.ist.
__device__ __forceinline__ void pipe_issue(WarpPipe &P, const void *src, unsigned bytes, unsigned skip = 0) {
    const int s = P.ist;
    if (P.lane == 0) {
        fence_proxy_async();
        mbar_expect_tx(&P.bars[s], bytes);
        bulk_g2s(P.stages + static_cast<size_t>(s) * P.stage_bytes + skip, src, bytes, &P.bars[s]);
    }
    ++P.issued;
    if (++P.ist == P.NS) P.ist = 0;
}

__device__ __forceinline__ bool pipe_wait(WarpPipe &P) { return mbar_wait(&P.bars[P.st], P.ph); }

__device__ __forceinline__ const uint8_t *pipe_front(const WarpPipe &P) {
    return P.stages + static_cast<size_t>(P.st) * P.stage_bytes;
}

__device__ __forceinline__ void pipe_pop(WarpPipe &P) {
    __syncwarp();
    if (++P.st == P.NS) {
        P.st = 0;
        P.ph ^= 1u;
    }
}

// After a failed wait: wait (bounded) for the copies still in flight, from `from`.
__device__ __forceinline__ void pipe_drain(WarpPipe &P, int from) {
    for (int k = from; k < P.issued; ++k) mbar_wait(&P.bars[k % P.NS], (k / P.NS) & 1);
}

// Combine the CTA's warps and store either the output (one split) or the split partial;
// with several splits and a counter `arrive`, the unit's last CTA to arrive (it resets
// the counter) merges the S partials by log-sum-exp and stores the output.
template <int D, int NT>
__device__ __forceinline__ void combine_store(WarpAcc<D, NT> &A, const BodyCtx &c, bool has_data, uint8_t *smem,
                                              int warp, long long row0, int sp, int S, int out_fp32, void *out,
                                              float *part_acc, float *part_ml, int sstride, unsigned *arrive) {
    constexpr int KS = D / 16;
    const int g = c.g, t = c.t, G = c.G;
    float l_run = A.l_run;
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    __syncthreads();   // every warp is done with its stages
    // each warp's O^T columns (hi and lo parts, [8 NT][DP]: a store's 32 lanes hit 32
    // banks), its value zero-point terms ([NJ][8 NT]: row j = channel group, on lanes
    // g = j) and per-head m, l; hi + lo + zero term are added while merging
    constexpr int CF = comb_floats(D, NT), DP = D + 4, NJ = D / 32;
    float *base = reinterpret_cast<float *>(smem);
    {
        float *ob = base + warp * CF;
        float *zb = ob + 8 * NT * DP;
        float *ml = zb + NJ * 8 * NT;
#pragma unroll
        for (int m = 0; m < KS; ++m)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int d0 = 16 * m + g, c0 = 8 * n + 2 * t;
                ob[c0 * DP + d0] = A.oacc[m][n][0];
                ob[(c0 + 1) * DP + d0] = A.oacc[m][n][1];
                ob[c0 * DP + d0 + 8] = A.oacc[m][n][2];
                ob[(c0 + 1) * DP + d0 + 8] = A.oacc[m][n][3];
            }
        if (g < NJ) {
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                zb[g * 8 * NT + 8 * n + 2 * t] = A.zc[n][0];
                zb[g * 8 * NT + 8 * n + 2 * t + 1] = A.zc[n][1];
            }
        }
        if (t == 0 && g < G) {
            ml[g] = has_data ? A.m_run : -INFINITY;
            ml[8 + g] = l_run;
        }
    }
    __syncthreads();
    // outputs in groups of 4 channels of one head (16-byte smem reads and global stores);
    // the warps' merge weights once per group
    for (int i4 = threadIdx.x; i4 < G * D / 4; i4 += NW * 32) {
        const int hd = (4 * i4) / D, d = (4 * i4) % D;
        const int chi = hd, clo = (NT == 1) ? hd + G : 8 + hd, j = d >> 5;
        constexpr int MLO = 8 * NT * DP + NJ * 8 * NT;   // m, l offset in a warp's buffer
        float mw[NW], M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            mw[w] = base[w * CF + MLO + hd];
            M = fmaxf(M, mw[w]);
        }
        float den = 0.f;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float *ob = base + w * CF;
            const float *zb = ob + 8 * NT * DP;
            const float wt = (mw[w] == -INFINITY) ? 0.f : fast_exp2(mw[w] - M);
            den = fmaf(wt, ob[MLO + 8 + hd], den);
            const float4 oh = *reinterpret_cast<const float4 *>(ob + chi * DP + d);
            const float4 ol = *reinterpret_cast<const float4 *>(ob + clo * DP + d);
            const float z = zb[j * 8 * NT + chi] + zb[j * 8 * NT + clo];
            val.x = fmaf(wt, oh.x + ol.x + z, val.x);
            val.y = fmaf(wt, oh.y + ol.y + z, val.y);
            val.z = fmaf(wt, oh.z + ol.z + z, val.z);
            val.w = fmaf(wt, oh.w + ol.w + z, val.w);
        }
        const long long row = row0 + hd;
        if (S == 1) {
            const float r = __frcp_rn(den);
            const float4 o = make_float4(val.x * r, val.y * r, val.z * r, val.w * r);
            if (out_fp32) {
                *reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + row * D + d) = o;
            } else {
                const __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y), hi = __floats2bfloat162_rn(o.z, o.w);
                uint2 u;
                u.x = *reinterpret_cast<const uint32_t *>(&lo);
                u.y = *reinterpret_cast<const uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(out) + row * D + d) = u;
            }
        } else {
            *reinterpret_cast<float4 *>(part_acc + (row * sstride + sp) * D + d) = val;
            if (d == 0) {
                part_ml[(row * sstride + sp) * 2] = M - c.pbias;   // den and val carry 2^pbias
                part_ml[(row * sstride + sp) * 2 + 1] = den;
            }
        }
    }
    if (S == 1 || arrive == nullptr) return;
    // split partials: the CTA's stores precede (barrier) thread 0's release-acquire count
    // of the arrival; the last CTA merges (no CTA waits for another)
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned prev;
        asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(prev) : "l"(arrive) : "memory");
        s_last = prev == static_cast<unsigned>(S - 1);
    }
    __syncthreads();
    if (!s_last) return;
    for (int i4 = threadIdx.x; i4 < G * D / 4; i4 += NW * 32) {
        const int hd = (4 * i4) / D, d = (4 * i4) % D;
        const long long row = row0 + hd;
        const float *ml = part_ml + row * sstride * 2;
        float M = -INFINITY;
        for (int s = 0; s < S; ++s) M = fmaxf(M, __ldcg(ml + 2 * s));
        float den = 0.f;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < S; ++s) {
            const float ms = __ldcg(ml + 2 * s);
            if (ms == -INFINITY) continue;
            const float wt = fast_exp2(ms - M);
            den = fmaf(wt, __ldcg(ml + 2 * s + 1), den);
            const float4 a = __ldcg(reinterpret_cast<const float4 *>(part_acc + (row * sstride + s) * D + d));
            val.x = fmaf(wt, a.x, val.x);
            val.y = fmaf(wt, a.y, val.y);
            val.z = fmaf(wt, a.z, val.z);
            val.w = fmaf(wt, a.w, val.w);
        }
        const float r = __frcp_rn(den);
        const float4 o = make_float4(val.x * r, val.y * r, val.z * r, val.w * r);
        if (out_fp32) {
            *reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + row * D + d) = o;
        } else {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y), hi = __floats2bfloat162_rn(o.z, o.w);
            uint2 u;
            u.x = *reinterpret_cast<const uint32_t *>(&lo);
            u.y = *reinterpret_cast<const uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(out) + row * D + d) = u;
        }
    }
    if (threadIdx.x == 0) *arrive = 0u;   // ready for the next launch
}

// Shared-memory carve-up: [stages | combine buffer][barriers][q fragments].
struct SmemParts {
    uint8_t *stages;
    uint64_t *bars;
    uint4 *aq_s;
    float4 *scal_s;
};

// PS: the CTA's stages (all warps).
__host__ __device__ inline size_t smem_bars_off(int PS, int stage_bytes, int D, int NT) {
    const size_t stage = static_cast<size_t>(PS) * stage_bytes;
    const size_t comb = static_cast<size_t>(NW) * comb_floats(D, NT) * 4;
    return ((stage > comb ? stage : comb) + 127) & ~size_t(127);
}

// Bytes after the per-lane scalars: a fused append's token codes (values, keys: 2D), the
// CTA's two scale maxima (16) and the token's fp16 scales/zeros per role and group.
__host__ __device__ constexpr int append_scratch_bytes(int D) { return 2 * D + 16 + 2 * (D / 32) * 2 * 2; }
// Then the prologue area: the CTA's q rows (up to 8 heads), the appended token's K and V
// rows (bf16) and the mbarrier of their bulk copies, issued with the first block copies.
__host__ __device__ constexpr int prologue_bytes(int D) { return 8 * D * 2 + 2 * D * 2 + 16; }

__host__ __device__ inline size_t smem_total(int PS, int stage_bytes, int D, int NT) {
    const size_t bars = static_cast<size_t>(PS) * 8 + 8 * (PS & 1);   // keeps 16-B alignment
    return smem_bars_off(PS, stage_bytes, D, NT) + bars + static_cast<size_t>(D / 16) * 32 * 16 * 3 + 32 * 16 +
           append_scratch_bytes(D) + prologue_bytes(D);
}

__device__ __forceinline__ SmemParts carve(uint8_t *smem, int PS, int stage_bytes, int D, int NT) {
    SmemParts s;
    s.stages = smem;
    const size_t bo = smem_bars_off(PS, stage_bytes, D, NT);
    s.bars = reinterpret_cast<uint64_t *>(smem + bo);
    s.aq_s = reinterpret_cast<uint4 *>(smem + bo + static_cast<size_t>(PS) * 8 + 8 * (PS & 1));
    s.scal_s = reinterpret_cast<float4 *>(s.aq_s + 3 * (D / 16) * 32);
    return s;
}

// ------------------------------------------------------------------ fused append
// Put token e's codes code[0..D) into a 16-token half's code area `area` (global or
// shared memory) with per-code atomic ORs, `step` threads from `tid`.  The first token
// of a half rebuilds the half: its words are zeroed first (stale bytes must read as
// zero); the caller orders the zeroing before the ORs of other threads.
template <int BITS>
__device__ __forceinline__ void zero_half(uint32_t *area, int tid, int step, int D) {
    for (int widx = tid; widx < D * BITS / 2; widx += step) area[widx] = 0u;
}
// Insert token e's codes into a half's code words (one warp): the code fields of the
// token that share a lane word are OR-ed in at once.  Values (role 1): the fields of
// channels 16m + g and 16m + g + 8 are adjacent slots of lane 4g + t, one word (2 codes;
// with 2-bit codes two such pairs share a word).  Keys (role 0): channels
// 16k + 8r + 2t + hb of lane 4 gk + t fill slots 4k + 2i + r, one word (4 codes).
// (e = 8 ch + 2t + hb for values, e = 8i + gk for keys; the positions are those of
// quant::code_place, channel by channel.)
template <int BITS>
__device__ __forceinline__ void or_token_words(uint32_t *area, int role, int e, const uint8_t *code, int lane,
                                               int D) {
    constexpr int P = 16 / BITS;
    const int Wh = D * BITS / 64, c = Wh < 4 ? Wh : 4;
    auto mem_word = [&](int lw, int w) { return ((w / c) * 32 + lw) * c + (w % c); };
    if (role == 1) {
        const int t = (e & 7) >> 1, ch = e >> 3, hb = e & 1;
        for (int pi = lane; pi < D / 2; pi += 32) {
            const int g = pi & 7, m = pi >> 3;
            const int slot = 4 * m + 2 * ch, f = slot % P + hb * P, d = 16 * m + g;
            const uint32_t v = (static_cast<uint32_t>(code[d]) << (f * BITS)) |
                               (static_cast<uint32_t>(code[d + 8]) << ((f + 1) * BITS));
            atomicOr(area + mem_word(4 * g + t, slot / P), v);
        }
    } else {
        const int i = e >> 3, gk = e & 7;
        for (int pi = lane; pi < D / 4; pi += 32) {
            const int t = pi & 3, k = pi >> 2;
            const int slot = 4 * k + 2 * i, f = slot % P, d = 16 * k + 2 * t;
            const uint32_t v = (static_cast<uint32_t>(code[d]) << (f * BITS)) |
                               (static_cast<uint32_t>(code[d + 1]) << ((f + P) * BITS)) |
                               (static_cast<uint32_t>(code[d + 8]) << ((f + 1) * BITS)) |
                               (static_cast<uint32_t>(code[d + 9]) << ((f + 1 + P) * BITS));
            atomicOr(area + mem_word(4 * gk + t, slot / P), v);
        }
    }
}

// Quantize the token appended by a fused launch (token u of its block) in one warp, with
// the append kernel's arithmetic: each 32-channel group of the value row (and, per-token
// keys, of the key row) is held by 32/CPL lanes of CPL channels, so the warp quantizes
// every group at once.  Codes, scales and zeros go to `scratch` (shared memory), from
// which the warp that processes the block patches its staged copy (patch_stage); the
// cache in HBM gets them from append_token_store.  Returns the new scale maxima (keys,
// values; fp16 bits) on every lane.
template <int BK, int BV, int KM, int D>
__device__ __forceinline__ void append_token_quantize(uint8_t *scratch, const uint16_t *kn, const uint16_t *vn,
                                                      int lane, unsigned smax_new[2]) {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    constexpr int NJ = D / 32, CPL = D / 32, LPG = 32 / CPL;
    uint8_t *codes = scratch;                                              // [0, D): values, [D, 2D): keys
    uint16_t *szs = reinterpret_cast<uint16_t *>(scratch + 2 * D + 16);   // [role][j][scale, zero]
    const int j = lane / LPG, d0 = CPL * lane;   // this lane's group and first channel
    smax_new[0] = smax_new[1] = 0u;
    constexpr int NROLE = KM == 1 ? 2 : 1;
#pragma unroll
    for (int r = 0; r < NROLE; ++r) {
        const int role = r == 0 ? 1 : 0;   // values, then (per-token keys) keys
        const int bits = role ? BV : BK;
        const uint16_t *src = (role ? vn : kn) + d0;
        float x[CPL];
        if constexpr (CPL == 4) {
            const uint2 w = *reinterpret_cast<const uint2 *>(src);
            x[0] = __uint_as_float(w.x << 16);
            x[1] = __uint_as_float(w.x & 0xFFFF0000u);
            x[2] = __uint_as_float(w.y << 16);
            x[3] = __uint_as_float(w.y & 0xFFFF0000u);
        } else {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(src);
            x[0] = __uint_as_float(w << 16);
            x[1] = __uint_as_float(w & 0xFFFF0000u);
        }
        float mn = x[0], mx = x[0];
#pragma unroll
        for (int i = 1; i < CPL; ++i) {
            mn = fminf(mn, x[i]);
            mx = fmaxf(mx, x[i]);
        }
#pragma unroll
        for (int o = LPG / 2; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        float sc, z;
        uint16_t s16, z16;
        quant::group_params(mn, mx, bits, sc, z, s16, z16);
        uint32_t packed = 0u;
#pragma unroll
        for (int i = 0; i < CPL; ++i) packed |= static_cast<uint32_t>(quant::group_code(x[i], sc, z, bits)) << (8 * i);
        if constexpr (CPL == 4) *reinterpret_cast<uint32_t *>(codes + (role ? 0 : D) + d0) = packed;
        else *reinterpret_cast<uint16_t *>(codes + (role ? 0 : D) + d0) = static_cast<uint16_t>(packed);
        if (lane % LPG == 0) {
            szs[(role * NJ + j) * 2] = s16;
            szs[(role * NJ + j) * 2 + 1] = z16;
        }
        smax_new[role] = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(s16));
    }
    __syncwarp();
}

// Per-channel keys: the new key row into the residual of unit `unit` (slot u: the host
// takes the two-launch path when the token completes a key group).  One warp.
template <int D>
__device__ __forceinline__ void append_residual_row(const DecodeParams &p, long long unit, int u, const uint16_t *kn,
                                                    int lane) {
    const uint32_t *src = reinterpret_cast<const uint32_t *>(kn);
    uint32_t *dst = reinterpret_cast<uint32_t *>(p.res_w + (unit * 32 + u) * D);
    for (int i = lane; i < D / 2; i += 32) dst[i] = src[i];
    __syncwarp();   // the warp's own later reads of the row (when it holds the block)
}

// The quantized token (append_token_quantize's `scratch`) into the cache in HBM for later
// launches: its code fields (the half's words rebuilt from zero when it is the half's
// first token), scales and zeros in the block record of unit `unit`, and the layer's scale
// maxima.  One warp.
template <int BK, int BV, int KM, int D>
__device__ __forceinline__ void append_token_store(const DecodeParams &p, long long unit, int blk, int u,
                                                   const uint8_t *scratch, int lane, const unsigned smax_new[2]) {
    constexpr int NJ = D / 32;
    constexpr int KC = 4 * D * BK, KSZ = 4 * D, VC = 4 * D * BV;
    constexpr int REC = KC + KSZ + VC + 4 * D;
    const int e = u & 15, eta = u >> 4;
    uint8_t *rec = p.rec_w + rec_index(p.btab, static_cast<int>(unit / p.Hkv), p.Hkv, static_cast<int>(unit % p.Hkv),
                                       p.cap_blk, blk) * static_cast<long long>(REC);
    const uint8_t *codes = scratch;
    const uint16_t *szs = reinterpret_cast<const uint16_t *>(scratch + 2 * D + 16);
    if (lane < (KM == 1 ? 2 : 1) * NJ) {   // lane = role-major (values, then keys) group
        const int role = lane < NJ ? 1 : 0, j = lane % NJ;
        uint8_t *sz = rec + (role ? KC + KSZ + VC : KC);
        const int so = quant::tok_sz_off(u, j, NJ);
        *reinterpret_cast<uint16_t *>(sz + so) = szs[(role * NJ + j) * 2];
        *reinterpret_cast<uint16_t *>(sz + so + 4 * NJ) = szs[(role * NJ + j) * 2 + 1];
    }
    uint32_t *vwords = reinterpret_cast<uint32_t *>(rec + KC + KSZ + eta * 2 * D * BV);
    uint32_t *kwords = reinterpret_cast<uint32_t *>(rec + eta * 2 * D * BK);
    if (e == 0) {   // the half's first token: its words are rebuilt from zero
        zero_half<BV>(vwords, lane, 32, D);
        if constexpr (KM == 1) zero_half<BK>(kwords, lane, 32, D);
        __syncwarp();
    }
    or_token_words<BV>(vwords, 1, e, codes, lane, D);
    if constexpr (KM == 1) or_token_words<BK>(kwords, 0, e, codes + D, lane, D);
    if (lane == 0) {
        if (smax_new[0]) atomicMax(p.smax_out, smax_new[0]);
        if (smax_new[1]) atomicMax(p.smax_out + 1, smax_new[1]);
    }
}

// Upper bound of the fp16 value scales of a new row: a 32-channel group's scale is at
// most 2 max|v| / (2^BV - 1), and rounding it to fp16 (or to a subnormal step) raises it
// by less than the margin.  Warp-wide (every lane gets it).
template <int BV, int D>
__device__ __forceinline__ float new_value_scale_bound(const uint16_t *vn, int lane) {
    // max |v| from the bf16 magnitude bits (ordered like the values they encode)
    unsigned mb = 0u;
#pragma unroll
    for (int d = lane; d < D; d += 32) mb = max(mb, static_cast<unsigned>(vn[d]) & 0x7FFFu);
    mb = __reduce_max_sync(0xffffffffu, mb);
    const float m = quant::bf16_to_f32(static_cast<uint16_t>(mb));
    return m * (2.0f / static_cast<float>((1 << BV) - 1)) * (1.0f + 0x1p-9f) + 0x1p-24f;
}

// The warp that processes the appended token's block writes the token into its staged
// copy of the block (taken before or while the new bytes reached HBM), so the copy equals
// the block after the append: the code fields of the token (the half's words rebuilt when
// it is the half's first token, as in HBM) and its scales and zeros.  One warp; the
// stage's bulk copy has completed.
template <int BK, int BV, int KM, int D>
__device__ __forceinline__ void patch_stage(uint8_t *stage, int u, const uint8_t *scratch, int lane) {
    constexpr int NJ = D / 32;
    constexpr int KC = 4 * D * BK, KSZ = 4 * D, VC = 4 * D * BV;
    const int e = u & 15, eta = u >> 4;
    const uint16_t *szs = reinterpret_cast<const uint16_t *>(scratch + 2 * D + 16);
    uint32_t *vwords = reinterpret_cast<uint32_t *>(stage + KC + KSZ + eta * 2 * D * BV);
    uint32_t *kwords = reinterpret_cast<uint32_t *>(stage + eta * 2 * D * BK);
    if (e == 0) {
        zero_half<BV>(vwords, lane, 32, D);
        if constexpr (KM == 1) zero_half<BK>(kwords, lane, 32, D);
        __syncwarp();
    }
    or_token_words<BV>(vwords, 1, e, scratch, lane, D);
    if constexpr (KM == 1) or_token_words<BK>(kwords, 0, e, scratch + D, lane, D);
    if (lane < NJ) {
        uint8_t *sz = stage + KC + KSZ + VC + quant::tok_sz_off(u, lane, NJ);
        *reinterpret_cast<uint16_t *>(sz) = szs[(NJ + lane) * 2];
        *reinterpret_cast<uint16_t *>(sz + 4 * NJ) = szs[(NJ + lane) * 2 + 1];
        if constexpr (KM == 1) {
            uint8_t *kz = stage + KC + quant::tok_sz_off(u, lane, NJ);
            *reinterpret_cast<uint16_t *>(kz) = szs[lane * 2];
            *reinterpret_cast<uint16_t *>(kz + 4 * NJ) = szs[lane * 2 + 1];
        }
    }
    __syncwarp();
}

// ------------------------------------------------------------------ per-layer kernel
// FUSED: the instance for kvq_append_decode launches (p.k_new set); decode-only launches
// take the instance without the append code.
template <int BK, int BV, int KM, int D, int NT, bool FUSED>
__global__ void __launch_bounds__(NW * 32, NT == 1 ? 4 : 3) decode_split_kernel(const DecodeParams p) {
    const bool early = p.early != 0;   // CTA-uniform
    if (!early) pdl_enter();
    constexpr int REC = unit_bytes(D, BK, BV, KM, 2);
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.z, h = blockIdx.y, sp = blockIdx.x;
    const int G = p.G, L = p.ragged ? (p.lens_dev ? p.lens_dev[b] : p.lens[b]) : p.L;   // this request's length

    // nstage stages per warp, one more for warps 0 .. nextra - 1 (those with the most blocks)
    const int NS = p.nstage + (warp < p.nextra ? 1 : 0);
    const int sbase = warp * p.nstage + min(warp, p.nextra);
    const int nblk = (L + 31) >> 5;
    const int blk0 = sp * p.bps, blk1 = min(nblk, blk0 + p.bps);
    const int rem = L & 31;
    const int tail_blk = rem ? (L >> 5) : -1;

    const SmemParts sm = carve(smem, NW * p.nstage + p.nextra, REC, D, NT);
    WarpPipe P{sm.stages + static_cast<size_t>(sbase) * REC, sm.bars + sbase, NS, REC, lane, 0, 0, 0u, 0};
    pipe_init(P);
    const int nb = (blk1 - blk0 > warp) ? (blk1 - blk0 - warp + NW - 1) / NW : 0;
    const uint8_t *unit_rec = p.rec + (static_cast<long long>(b) * p.Hkv + h) * p.cap_blk * REC;   // slab plans
    // per-channel keys of the last, incomplete group come from the residual: fetch only
    // the value part of that block's record
    constexpr unsigned VSKIP = KM == 0 ? 2 * 2 * D * BK + 4 * D : 0;
    auto issue_block = [&](int k) {
        const int blk = blk0 + warp + NW * k;
        const uint8_t *src = p.btab ? p.rec + rec_index(p.btab, b, p.Hkv, h, p.cap_blk, blk) * REC
                                    : unit_rec + static_cast<long long>(blk) * REC;
        if (blk == tail_blk) pipe_issue(P, src + VSKIP, REC - VSKIP, VSKIP);
        else pipe_issue(P, src, REC);
    };
    const long long unit = static_cast<long long>(b) * p.Hkv + h;
    // the first stages' block copies and (per-channel keys) the bf16 residual rows of the
    // tail block into L2 (read after the tail's copy)
    auto issue_first = [&]() {
        if constexpr (KM == 0) {
            if (p.res && tail_blk >= blk0 && tail_blk < blk1 && ((tail_blk - blk0) % NW) == warp) {
                const char *r = reinterpret_cast<const char *>(p.res + unit * 32 * D);
                for (int i = lane; i < rem * D * 2 / 128; i += 32) prefetch_l2(r + i * 128);
            }
        }
        for (int k = 0; k < NS && k < nb; ++k) issue_block(k);
    };
    if (early) {
        issue_first();
        pdl_enter();
    }
    // the layer's scale maxima: loaded first (converted at first use), their latency
    // overlaps the set-up
    const unsigned smax_bits_k = p.smax[0], smax_bits_v = p.smax[1];
    // a fused launch appends token L - 1 (the last of block new_blk) in the CTA that holds
    // that block; the block's warp patches its staged copy with the token
    const bool fused = FUSED && p.k_new != nullptr;
    const int new_blk = (L - 1) >> 5;
    const bool append_here = fused && new_blk >= blk0 && new_blk < blk1;   // CTA-uniform
    uint8_t *append_scratch = reinterpret_cast<uint8_t *>(sm.scal_s + 32);
    // the prologue copies (the q rows of the kv head's G query heads and, in the CTA that
    // appends, the token's K and V rows; all 16-byte aligned: rows of 2D bytes) go out
    // before the block copies (unless those went out early), which fill the memory queues
    // for microseconds
    uint16_t *q_s = reinterpret_cast<uint16_t *>(append_scratch + append_scratch_bytes(D));
    uint16_t *kn_s = q_s + 8 * D, *vn_s = kn_s + D;
    uint64_t *pro_bar = reinterpret_cast<uint64_t *>(vn_s + D);
    if (threadIdx.x == 0) {
        mbar_init(pro_bar, 1);
        fence_mbar_init();
        const unsigned qbytes = static_cast<unsigned>(G * D * 2);
        mbar_expect_tx(pro_bar, qbytes + (append_here ? 4 * D : 0));
        bulk_g2s(q_s, p.q + unit * G * D, qbytes, pro_bar);
        if (append_here) {
            bulk_g2s(kn_s, p.k_new + unit * D, 2 * D, pro_bar);
            bulk_g2s(vn_s, p.v_new + unit * D, 2 * D, pro_bar);
        }
    }
    __syncwarp();   // warp 0's other lanes wait on pro_bar after lane 0 initialised it; the
                    // other warps wait on it only after a CTA barrier
    if (!early) issue_first();


    const float smax_k = __half2float(__ushort_as_half(static_cast<unsigned short>(smax_bits_k)));
    const float smax_v = __half2float(__ushort_as_half(static_cast<unsigned short>(smax_bits_v)));
    if (fused && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
        atomicMax(p.smax_out, smax_bits_k);   // carry the old length's maxima forward
        atomicMax(p.smax_out + 1, smax_bits_v);
    }
    BodyCtx c = make_ctx<KM, D, NT>(lane, G, smax_v, sm.aq_s);
    c.res = p.res ? p.res + (static_cast<long long>(b) * p.Hkv + h) * 32 * D : nullptr;
    const int hh = c.g % G;
    // the key prescale needs no new scale (a token that completes a per-channel key group
    // is never fused; per-token keys are scaled in fp32)
    if (warp == 0 && !mbar_wait(pro_bar, 0) && lane == 0) atomicOr(p.status, kStatusWaitExpired);
    setup_query<KM, D, NT>(q_s + hh * D, smax_k, sm.aq_s, sm.scal_s, c, warp);
    __syncthreads();
    load_query_scalars(c, sm.scal_s);
    // the value prescale must cover the new token's scales: every warp bounds them from
    // the new row (the same CTA-uniform result; the row has arrived: warp 0 waited for it)
    if (append_here) {
        if (!mbar_wait(pro_bar, 0) && lane == 0) atomicOr(p.status, kStatusWaitExpired);
        c.pbias = value_bias(fmaxf(smax_v, new_value_scale_bound<BV, D>(vn_s, lane)));
    }
    // the append runs in the warp with the fewest blocks (the block's own warp when none
    // has fewer), before its blocks; the block's warp waits for it (named barrier 1) only
    // before patching its staged copy, its last block
    int owner = 0, helper = 0;
    if (append_here) {
        auto blocks_of = [&](int w) { return (blk1 - blk0 > w) ? (blk1 - blk0 - w + NW - 1) / NW : 0; };
        owner = (new_blk - blk0) % NW;
        helper = owner;
        for (int w = NW - 1; w >= 0; --w)
            if (blocks_of(w) < blocks_of(helper)) helper = w;
        if (warp == helper) {
            // the token's rows (kn, vn) arrive by bulk copy with the q rows
            if (!mbar_wait(pro_bar, 0) && lane == 0) atomicOr(p.status, kStatusWaitExpired);
            unsigned smax_new[2];
            append_token_quantize<BK, BV, KM, D>(append_scratch, kn_s, vn_s, lane, smax_new);
            // the tail reads the new residual row from HBM after the hand-over; the record's
            // words, scales and the maxima are only for later launches: written after it,
            // so the barrier's release does not wait for them
            if constexpr (KM == 0) append_residual_row<D>(p, unit, (L - 1) & 31, kn_s, lane);
            if (helper != owner) asm volatile("bar.arrive 1, %0;" ::"n"(64) : "memory");
            append_token_store<BK, BV, KM, D>(p, unit, new_blk, (L - 1) & 31, append_scratch, lane, smax_new);
        }
    }

    WarpAcc<D, NT> A;
    acc_init(A);
    const bool has_tail = tail_blk >= blk0 && tail_blk < blk1 && ((tail_blk - blk0) % NW) == warp;
    const int nb_main = nb - (has_tail ? 1 : 0);
    // the appended token is in the unit's last block, the last block of its warp: the
    // tail block, or (per-token keys, L % 32 == 0) the last full block, which is then
    // taken out of the main loop
    const bool patch_full = KM == 1 && append_here && !has_tail && nb > 0 && blk0 + warp + NW * (nb - 1) == new_blk;
    const int nb_loop = nb_main - (patch_full ? 1 : 0);
    bool failed = false;
    int i = 0;
    for (; i < nb_loop; ++i) {
        if (!pipe_wait(P)) {
            failed = true;
            break;
        }
        process_unit<BK, BV, KM, D, NT, 2, false>(A, pipe_front(P), 32, c);
        pipe_pop(P);
        if (P.issued < nb) issue_block(P.issued);
    }
    // the helper's codes, scales and zeros are in shared memory and the new residual row
    // in HBM (every path of the owner passes here once; the helper arrives after its
    // quantize, whose wait is bounded)
    if (append_here && warp == owner && helper != owner) asm volatile("bar.sync 1, %0;" ::"n"(64) : "memory");
    if constexpr (KM == 1) {
        if (!failed && patch_full) {
            if (!pipe_wait(P)) {
                failed = true;
            } else {
                patch_stage<BK, BV, KM, D>(const_cast<uint8_t *>(pipe_front(P)), (L - 1) & 31, append_scratch, lane);
                process_unit<BK, BV, KM, D, NT, 2, false>(A, pipe_front(P), 32, c);
                pipe_pop(P);
                ++i;
            }
        }
    }
    if (!failed && has_tail) {
        if (!pipe_wait(P)) {
            failed = true;
        } else {
            const bool patch = append_here && tail_blk == new_blk;
            if (patch)
                patch_stage<BK, BV, KM, D>(const_cast<uint8_t *>(pipe_front(P)), (L - 1) & 31, append_scratch, lane);
            if (rem <= 16) process_unit<BK, BV, KM, D, NT, 2, true, false, 1>(A, pipe_front(P), rem, c);
            else process_unit<BK, BV, KM, D, NT, 2, true>(A, pipe_front(P), rem, c);
            ++i;
        }
    }
    if (failed) {
        pipe_drain(P, i);
        if (lane == 0) atomicOr(p.status, kStatusWaitExpired);
    }
    combine_store<D, NT>(A, c, nb > 0 && !failed, smem, warp, static_cast<long long>(b) * p.Hkv * G + h * G, sp,
                         p.S, p.out_fp32, p.out, p.part_acc, p.part_ml, p.sstride, p.arrive ? p.arrive + unit : nullptr);
}

// ------------------------------------------------------------------ paged kernel
// Splits [0, S2) cover the request's INT2 records (32-token groups, 2-bit keys per
// channel, 2-bit values per token); splits [S2, S2 + S4) its INT4 pages (16 tokens,
// 4-bit keys and values per token): main pages, then the pending pages of INT2 tokens
// whose group is still open.  Every split is bitwidth-homogeneous.  INT4 work items are
// pairs of full pages, staged side by side and processed as one 32-token unit (the
// attention is a sum over tokens: their order does not matter), then the odd full page
// and the partly filled pages one by one.
template <bool INT2>
__device__ __forceinline__ void paged_body(const PagedDecodeParams &p, uint8_t *smem, int warp, int lane, int b,
                                           int h, int sp) {
    constexpr int D = 128, NT = 1;
    constexpr int REC2 = unit_bytes(D, 2, 2, 0, 2), PAGE4 = unit_bytes(D, 4, 4, 1, 1);
    constexpr int STAGE = REC2 > 2 * PAGE4 ? REC2 : 2 * PAGE4;
    const int G = p.G, NS = p.nstage;
    const int n2g = p.cnt[b].n2g, n4 = p.cnt[b].n4, np = p.cnt[b].np;
    // INT4 pages: f4 full main pages (then a partial one of pm tokens), fp full pending
    // pages (0 or 1, then a partial one of pp tokens)
    const int f4 = n4 >> 4, pm = n4 & 15, fp = np >> 4, pp = np & 15;
    const int F = f4 + fp, npair = F >> 1;
    const int nitems = INT2 ? n2g : npair + (F & 1) + (pm ? 1 : 0) + (pp ? 1 : 0);
    const int nsplit = INT2 ? p.S2 : p.S4, si = INT2 ? sp : sp - p.S2;
    const int per = (nitems + nsplit - 1) / nsplit;
    const int u0 = min(nitems, si * per), u1 = min(nitems, u0 + per);
    const SmemParts sm = carve(smem, NW * NS, STAGE, D, NT);
    WarpPipe P{sm.stages + static_cast<size_t>(warp) * NS * STAGE, sm.bars + warp * NS, NS, STAGE, lane, 0, 0, 0u, 0};
    pipe_init(P);
    const int *tab = p.table + static_cast<long long>(b) * p.P_cap;
    const uint8_t *pool2 = p.pool2 + static_cast<long long>(h) * p.n2_cap * REC2;
    const uint8_t *pool4 = p.pool4 + static_cast<long long>(h) * p.n4_cap * PAGE4;
    // table of request b: INT2 groups from the front (entry = the group's first 16-token
    // page, groups occupy page pairs), INT4 main pages from the back
    auto full_page = [&](int f) -> const uint8_t * {   // f-th full INT4 page
        const int page = f < f4 ? tab[p.P_cap - 1 - f] : p.pend_base + 2 * b;
        return pool4 + static_cast<long long>(page) * PAGE4;
    };
    // item u after the pairs: 0 = odd full page, 1 = partial main page, 2 = partial pending page
    auto single_kind = [&](int u) -> int {
        int k = u - npair;
        if (!(F & 1)) ++k;
        if (k >= 1 && !pm) ++k;
        return k;
    };
    auto issue_item = [&](int u) {
        if (INT2) {
            pipe_issue(P, pool2 + static_cast<long long>(tab[u] >> 1) * REC2, REC2);
        } else if (u < npair) {
            const uint8_t *a = full_page(2 * u), *bb = full_page(2 * u + 1);
            const int st = P.ist;
            if (lane == 0) {
                fence_proxy_async();
                mbar_expect_tx(&P.bars[st], 2 * PAGE4);
                uint8_t *dst = P.stages + static_cast<size_t>(st) * P.stage_bytes;
                bulk_g2s(dst, a, PAGE4, &P.bars[st]);
                bulk_g2s(dst + PAGE4, bb, PAGE4, &P.bars[st]);
            }
            ++P.issued;
            if (++P.ist == P.NS) P.ist = 0;
        } else {
            const int k = single_kind(u);
            const int page = k == 0 ? (F - 1 < f4 ? tab[p.P_cap - 1 - (F - 1)] : p.pend_base + 2 * b)
                           : k == 1 ? tab[p.P_cap - 1 - f4] : p.pend_base + 2 * b + fp;
            pipe_issue(P, pool4 + static_cast<long long>(page) * PAGE4, PAGE4);
        }
    };
    const int nb = (u1 - u0 > warp) ? (u1 - u0 - warp + NW - 1) / NW : 0;
    for (int k = 0; k < NS && k < nb; ++k) issue_item(u0 + warp + NW * k);

    const float smax_k = __half2float(__ushort_as_half(static_cast<unsigned short>(p.smax[0])));
    const float smax_v = __half2float(__ushort_as_half(static_cast<unsigned short>(p.smax[1])));
    WarpAcc<D, NT> A;
    acc_init(A);
    const long long qoff = (static_cast<long long>(b) * p.Hkv * G + h * G + (lane >> 2) % G) * D;
    BodyCtx c = make_ctx<INT2 ? 0 : 1, D, NT>(lane, G, smax_v, sm.aq_s);
    c.res = nullptr;
    setup_query<INT2 ? 0 : 1, D, NT>(p.q + qoff, smax_k, sm.aq_s, sm.scal_s, c, warp);
    __syncthreads();
    load_query_scalars(c, sm.scal_s);

    bool failed = false;
    int i = 0;
    for (; i < nb; ++i) {
        if (!pipe_wait(P)) {
            failed = true;
            break;
        }
        const int u = u0 + warp + NW * i;
        if (INT2) {
            process_unit<2, 2, 0, D, NT, 2, false>(A, pipe_front(P), 32, c);
        } else if (u < npair) {
            process_unit<4, 4, 1, D, NT, 2, false, true>(A, pipe_front(P), 32, c);
        } else {
            const int k = single_kind(u);
            const int v = k == 0 ? 16 : (k == 1 ? pm : pp);
            if (v == 16) process_unit<4, 4, 1, D, NT, 1, false>(A, pipe_front(P), 16, c);
            else process_unit<4, 4, 1, D, NT, 1, true>(A, pipe_front(P), v, c);
        }
        pipe_pop(P);
        if (P.issued < nb) issue_item(u0 + warp + NW * P.issued);
    }
    if (failed) {
        pipe_drain(P, i);
        if (lane == 0) atomicOr(p.status, kStatusWaitExpired);
    }
    combine_store<D, NT>(A, c, nb > 0 && !failed, smem, warp, static_cast<long long>(b) * p.Hkv * G + h * G, sp,
                         p.S2 + p.S4, p.out_fp32, p.out, p.part_acc, p.part_ml, p.sstride,
                         p.arrive ? p.arrive + static_cast<long long>(b) * p.Hkv + h : nullptr);
}

__global__ void __launch_bounds__(NW * 32, 4) decode_paged_kernel(const PagedDecodeParams p) {
    pdl_enter();
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.z, h = blockIdx.y, sp = blockIdx.x;
    if (sp < p.S2) paged_body<true>(p, smem, warp, lane, b, h, sp);
    else paged_body<false>(p, smem, warp, lane, b, h, sp);
}

// Log-sum-exp merge of the split partials ("merged by online log-sum-exp"), for split
// counts below kInLaunchMergeSplits.
__global__ void merge_kernel(const MergeParams p) {
    // trigger first: the next kernel (usually the next layer's decode) may launch while the
    // decode this merge follows is still running (the host counts both as launches the
    // next one may overlap)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const long long row = blockIdx.x;   // b * Hq + hq
    const float *ml = p.part_ml + row * p.sstride * 2;
    float M = -INFINITY;
    for (int s = 0; s < p.S; ++s) M = fmaxf(M, ml[2 * s]);
    for (int d = threadIdx.x; d < p.D; d += blockDim.x) {
        float val = 0.f, den = 0.f;
        for (int s = 0; s < p.S; ++s) {
            const float ms = ml[2 * s];
            if (ms == -INFINITY) continue;
            const float wt = fast_exp2(ms - M);
            val = fmaf(wt, p.part_acc[(row * p.sstride + s) * p.D + d], val);
            den = fmaf(wt, ml[2 * s + 1], den);
        }
        const float o = val * __frcp_rn(den);
        if (p.out_fp32) reinterpret_cast<float *>(p.out)[row * p.D + d] = o;
        else reinterpret_cast<__nv_bfloat16 *>(p.out)[row * p.D + d] = __float2bfloat16_rn(o);
    }
}

using KernelFn = void (*)(const DecodeParams);

template <int D, int NT, int KM, bool FUSED>
KernelFn pick_bits(int bk, int bv) {
#define KVQ_CASE(BKv, BVv) \
    if (bk == BKv && bv == BVv) return decode_split_kernel<BKv, BVv, KM, D, NT, FUSED>;
    KVQ_CASE(2, 2) KVQ_CASE(2, 4) KVQ_CASE(2, 8)
    KVQ_CASE(4, 2) KVQ_CASE(4, 4) KVQ_CASE(4, 8)
    KVQ_CASE(8, 2) KVQ_CASE(8, 4) KVQ_CASE(8, 8)
#undef KVQ_CASE
    return nullptr;
}

// Column tiles of the value MMA and layout of the residual query parts: one tile (hi and
// lo columns side by side, the three residual parts in one MMA) when G divides 4, two
// tiles otherwise.
static int nt_for(int G) { return (G == 1 || G == 2 || G == 4) ? 1 : 2; }

template <bool FUSED>
KernelFn pick_kernel_t(int D, int bk, int bv, int kmode, int G) {
    const int NT = nt_for(G);
    if (G < 1 || G > 8) return nullptr;
    if (kmode == 1) {
        // rows (group, head) must fit one 16-row tile and heads must divide 8
        if (!(G == 1 || G == 2 || G == 4) || G * (D / 32) > 16) return nullptr;
        if (D == 64) return pick_bits<64, 1, 1, FUSED>(bk, bv);
        if (D == 128) return pick_bits<128, 1, 1, FUSED>(bk, bv);
        return nullptr;
    }
    if (D == 64) return NT == 1 ? pick_bits<64, 1, 0, FUSED>(bk, bv) : pick_bits<64, 2, 0, FUSED>(bk, bv);
    if (D == 128) return NT == 1 ? pick_bits<128, 1, 0, FUSED>(bk, bv) : pick_bits<128, 2, 0, FUSED>(bk, bv);
    return nullptr;
}

KernelFn pick_kernel(int D, int bk, int bv, int kmode, int G, bool fused) {
    return fused ? pick_kernel_t<true>(D, bk, bv, kmode, G) : pick_kernel_t<false>(D, bk, bv, kmode, G);
}

}  // namespace

// Stages per warp: as many as fit when the CTAs that registers allow per SM (4 for
// G <= 4, else 3) share the SM's 228 KB of shared memory; at least 2 (fewer CTAs then
// fit), at most 6.
int decode_stages(long long rec_bytes, int D, int G) {
    // per-CTA reserve, q fragments, barriers, prologue
    const long long fixed = 1024 + 3 * (D / 16) * 32 * 16 + 64 + prologue_bytes(D);
    for (int ctas = (nt_for(G) == 1 ? 4 : 3); ctas >= 1; --ctas) {
        const long long ns = (228LL * 1024 / ctas - fixed) / (NW * rec_bytes);
        if (ns >= 2) return static_cast<int>(ns > 6 ? 6 : ns);
    }
    return 2;
}

size_t decode_smem_bytes(long long rec_bytes, int nstage, int nextra, int D, int G) {
    const int NT = nt_for(G);
    return smem_total(NW * nstage + nextra, static_cast<int>(rec_bytes), D, NT);
}

// Per-kernel cache of the dynamic shared-memory attribute and occupancy, so launches
// (including launches recorded into CUDA graphs) issue no attribute calls.
struct KernelState {
    const void *fn = nullptr;
    size_t smem_set = 0;
    size_t occ_smem[8] = {};   // occupancy per dynamic shared-memory size (stage counts)
    int occ[8] = {};
};
static std::mutex g_state_mu;
static KernelState g_state[160];   // every decode instance (2 x 54), the paged and merge kernels

static cudaError_t prepare_kernel(const void *fn, size_t smem, int *occ_out) {
    std::lock_guard<std::mutex> lk(g_state_mu);
    KernelState *ks = nullptr;
    for (auto &e : g_state) {
        if (e.fn == fn || e.fn == nullptr) {
            ks = &e;
            break;
        }
    }
    if (!ks) return cudaErrorInvalidValue;
    ks->fn = fn;
    if (smem > ks->smem_set) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        ks->smem_set = smem;
    }
    if (occ_out) {
        int slot = -1;
        for (int i = 0; i < 8; ++i)
            if (ks->occ_smem[i] == smem || ks->occ_smem[i] == 0) {
                slot = i;
                break;
            }
        if (slot < 0) slot = static_cast<int>(smem % 8);   // full: replace an entry
        if (ks->occ_smem[slot] != smem) {
            cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ks->occ[slot], fn, NW * 32, smem);
            if (e != cudaSuccess) return e;
            ks->occ_smem[slot] = smem;
        }
        *occ_out = ks->occ[slot];
    }
    return cudaSuccess;
}

cudaError_t decode_occupancy(int D, int bk, int bv, int kmode, int G, long long rec_bytes, int nstage,
                             int nextra, int *ctas_per_sm) {
    KernelFn fn = pick_kernel(D, bk, bv, kmode, G, false);   // the fused instance has the same occupancy
    if (!fn) return cudaErrorInvalidValue;
    return prepare_kernel(reinterpret_cast<const void *>(fn), decode_smem_bytes(rec_bytes, nstage, nextra, D, G),
                          ctas_per_sm);
}

cudaError_t launch_decode(const DecodeParams &p, int D, int bk, int bv, int kmode, cudaStream_t st,
                          int *ctas_per_sm_out) {
    KernelFn fn = pick_kernel(D, bk, bv, kmode, p.G, p.k_new != nullptr);
    if (!fn) return cudaErrorInvalidValue;
    const size_t smem = decode_smem_bytes(p.rec_bytes, p.nstage, p.nextra, D, p.G);
    cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(fn), smem, ctas_per_sm_out);
    if (e != cudaSuccess) return e;
    dim3 grid(p.S, p.Hkv, p.B);
    e = launch_pdl(fn, grid, dim3(NW * 32), smem, st, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

int paged_rec2_bytes(int D) { return unit_bytes(D, 2, 2, 0, 2); }
int paged_page4_bytes(int D) { return unit_bytes(D, 4, 4, 1, 1); }

// A paged stage holds an INT2 record or two INT4 pages.
static int paged_stage_bytes() {
    return paged_rec2_bytes(128) > 2 * paged_page4_bytes(128) ? paged_rec2_bytes(128) : 2 * paged_page4_bytes(128);
}

int decode_paged_stages() { return decode_stages(paged_stage_bytes(), 128, 4); }

size_t decode_paged_smem_bytes(int nstage) { return smem_total(NW * nstage, paged_stage_bytes(), 128, 1); }

cudaError_t decode_paged_occupancy(int nstage, int *ctas_per_sm) {
    return prepare_kernel(reinterpret_cast<const void *>(decode_paged_kernel), decode_paged_smem_bytes(nstage), ctas_per_sm);
}

cudaError_t launch_merge(const MergeParams &p, cudaStream_t st) {
    cudaError_t e = launch_pdl(merge_kernel, dim3(p.B * p.Hq), dim3(p.D), 0, st, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decode_paged(const PagedDecodeParams &p, cudaStream_t st) {
    const size_t smem = decode_paged_smem_bytes(p.nstage);
    cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(decode_paged_kernel), smem, nullptr);
    if (e != cudaSuccess) return e;
    dim3 grid(p.S2 + p.S4, p.Hkv, p.B);
    e = launch_pdl(decode_paged_kernel, grid, dim3(NW * 32), smem, st, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}


}  // namespace kvq
