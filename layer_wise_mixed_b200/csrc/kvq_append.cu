// Quantize-and-pack of new K/V tokens into the layer cache (sm_100a).
//
// Asymmetric groupwise quantization with groups of 32 ("TriAxialKV per-role
// mixed-precision KV quantization", Facts: quantizer; KVTuner summary, Approach):
// values per token (32 consecutive channels), keys per channel (32 consecutive
// tokens, KIVI style; "Mixed-precision KV-cache quantization per-layer sensitivity",
// Facts) or per token.  Per-channel keys that do not yet fill a group stay in a bf16
// residual until the group's 32nd token arrives.
//
// Each quantizer step is one correctly rounded binary32 operation (__fsub_rn,
// __fdiv_rn, __float2int_rn, __float2half_rn); nothing here is contracted into FMA.
//
// One launch per kvq_append.  CTA roles:
//   [0, nV)         one 16-token half-block of values of one (b, h): quantize the new
//                   tokens (one warp per token, one lane per channel), then rebuild
//                   the half's packed words (one thread per word; tokens already in
//                   the half keep their bits, tokens not yet written read as zero).
//   [nV, nV + nK)   keys.  Per-token mode: as for values.  Per-channel mode: one
//                   completed 32-token group of one (b, h) (the first CTA of each
//                   (b, h) also moves the new tail tokens into the residual, after it
//                   has read the residual tokens of its group).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxD = 256;

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Scale/zero of a group from its min and max (stored fp16 values and their floats).
__device__ __forceinline__ void group_params(float mn, float mx, int bits, float &s, float &z,
                                             uint16_t &s16, uint16_t &z16) {
    const float qmax = static_cast<float>((1 << bits) - 1);
    const float s32 = __fdiv_rn(__fsub_rn(mx, mn), qmax);
    const __half sh = __float2half_rn(s32);
    const __half zh = __float2half_rn(mn);
    s = __half2float(sh);
    z = __half2float(zh);
    s16 = __half_as_ushort(sh);
    z16 = __half_as_ushort(zh);
}

__device__ __forceinline__ int group_code(float x, float s, float z, int bits) {
    if (s == 0.0f) return 0;
    const int c = __float2int_rn(__fdiv_rn(__fsub_rn(x, z), s));
    return max(0, min(c, (1 << bits) - 1));
}

// Owner (token in half e, channel d) of field f of lane word w, for the key operand
// role (role 0) or the value operand role (role 1) of the v1 format.
__device__ __forceinline__ void field_owner(int role, int lane, int w, int f, int bits, int &e,
                                            int &d) {
    const int P = 16 / bits;
    const int slot = w * P + (f % P), hb = f / P;
    const int g = lane >> 2, t = lane & 3;
    if (role == 0) {   // slot = (2k + i)*2 + r ; lane = 4*(u%8) + t ; channel = 16k + 8r + 2t + hb
        const int r = slot & 1, i = (slot >> 1) & 1, k = slot >> 2;
        e = 8 * i + g;
        d = 16 * k + 8 * r + 2 * t + hb;
    } else {           // slot = 4m + 2ch + rh ; lane = 4*g + t ; token = 8ch + 2t + hb
        const int rh = slot & 1, ch = (slot >> 1) & 1, m = slot >> 2;
        e = 8 * ch + 2 * t + hb;
        d = 16 * m + g + 8 * rh;
    }
}

// Byte offsets of a scale/zero pair in the s/z areas of the v1 format.
__device__ __forceinline__ int chan_sz_off(int d) {   // per-channel keys: scale; zero at +4
    const int k = d >> 4, e = d & 15;
    return 16 * (4 * k + ((e & 7) >> 1)) + 8 * (e >> 3) + 2 * (e & 1);
}
__device__ __forceinline__ int tok_sz_off(int u, int j, int nj) {   // per token: scale; zero at +4*nj
    return 8 * nj * (u >> 1) + 4 * j + 2 * (u & 1);
}

// Memory word index inside a half's code area -> (lane, lane word).
__device__ __forceinline__ void word_lane(int widx, int Wh, int &lane, int &w) {
    const int c = Wh < 4 ? Wh : 4;
    const int chunk = widx / (32 * c), rem = widx % (32 * c);
    lane = rem / c;
    w = chunk * c + rem % c;
}

// Per-token quantization of the new tokens of one 16-token half-block and repacking
// of its words.  role 0 = keys (per-token mode), 1 = values.
__device__ void per_token_half(const AppendParams &p, int role, int unit, int hbi,
                               uint8_t (*codes)[kMaxD], unsigned *cta_smax) {
    const int D = p.D, nj = D / 32;
    const int bits = role ? p.bv : p.bk;
    const uint16_t *src = (role ? p.V : p.K) + static_cast<long long>(unit) * p.n * D;
    const int L_new = p.L_old + p.n;
    const int u0 = 16 * hbi;
    const int es = max(p.L_old, u0) - u0, ee = min(L_new, u0 + 16) - u0;
    const int blk = hbi >> 1, eta = hbi & 1;
    uint8_t *rec = p.rec + (static_cast<long long>(unit) * p.cap_blk + blk) * p.rec_bytes;
    uint8_t *sz = rec + (role ? p.kc + p.ks + p.vc : p.kc);
    uint32_t *area = reinterpret_cast<uint32_t *>(rec + (role ? p.kc + p.ks : 0) +
                                                  static_cast<long long>(eta) * 2 * D * bits);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int e = es + warp; e < ee; e += kWarps) {
        const int tok = u0 + e;
        const uint16_t *row = src + static_cast<long long>(tok - p.L_old) * D;
        const int u = 16 * eta + e;
        for (int j = 0; j < nj; ++j) {
            const float x = bf16_to_f32(row[32 * j + lane]);
            float mn = x, mx = x;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            float s, z;
            uint16_t s16, z16;
            group_params(mn, mx, bits, s, z, s16, z16);
            codes[e][32 * j + lane] = static_cast<uint8_t>(group_code(x, s, z, bits));
            if (lane == 0) {
                const int so = tok_sz_off(u, j, nj);
                *reinterpret_cast<uint16_t *>(sz + so) = s16;
                *reinterpret_cast<uint16_t *>(sz + so + 4 * nj) = z16;
                atomicMax(cta_smax, static_cast<unsigned>(s16));
            }
        }
    }
    __syncthreads();

    const int Wh = D * bits / 64, F = 32 / bits, nw = D * bits / 2;
    const uint32_t mask = (1u << bits) - 1u;
    for (int widx = threadIdx.x; widx < nw; widx += kThreads) {
        int ln, w;
        word_lane(widx, Wh, ln, w);
        const uint32_t old = es > 0 ? area[widx] : 0u;
        uint32_t out = 0;
        for (int f = 0; f < F; ++f) {
            int e, d;
            field_owner(role, ln, w, f, bits, e, d);
            uint32_t c;
            if (e >= es && e < ee) c = codes[e][d];
            else if (e < es) c = (old >> (f * bits)) & mask;
            else c = 0;
            out |= c << (f * bits);
        }
        area[widx] = out;
    }
}

// Per-channel quantization of one completed 32-token key group; the CTA with
// first == true also writes the new residual tokens of its (b, h) afterwards.
__device__ void per_channel_group(const AppendParams &p, int unit, int q, bool do_group, bool first,
                                  float (*xs)[kMaxD], uint8_t (*codes)[kMaxD], unsigned *cta_smax) {
    const int D = p.D;
    const uint16_t *src = p.K + static_cast<long long>(unit) * p.n * D;
    uint16_t *res = p.res + static_cast<long long>(unit) * 32 * D;
    const int L_new = p.L_old + p.n;
    if (do_group) {
        const int t0 = 32 * q;
        for (int idx = threadIdx.x; idx < 32 * D; idx += kThreads) {
            const int u = idx / D, d = idx % D, tok = t0 + u;
            const uint16_t v = tok < p.L_old ? res[u * D + d]
                                             : src[static_cast<long long>(tok - p.L_old) * D + d];
            xs[u][d] = bf16_to_f32(v);
        }
        __syncthreads();
        uint8_t *rec = p.rec + (static_cast<long long>(unit) * p.cap_blk + q) * p.rec_bytes;
        for (int d = threadIdx.x; d < D; d += kThreads) {
            float mn = xs[0][d], mx = xs[0][d];
            for (int u = 1; u < 32; ++u) {
                mn = fminf(mn, xs[u][d]);
                mx = fmaxf(mx, xs[u][d]);
            }
            float s, z;
            uint16_t s16, z16;
            group_params(mn, mx, p.bk, s, z, s16, z16);
            for (int u = 0; u < 32; ++u) codes[u][d] = static_cast<uint8_t>(group_code(xs[u][d], s, z, p.bk));
            const int so = chan_sz_off(d);
            *reinterpret_cast<uint16_t *>(rec + p.kc + so) = s16;
            *reinterpret_cast<uint16_t *>(rec + p.kc + so + 4) = z16;
            atomicMax(cta_smax, static_cast<unsigned>(s16));
        }
        __syncthreads();
        const int bits = p.bk, Wh = D * bits / 64, F = 32 / bits, nwh = D * bits / 2;
        uint32_t *area = reinterpret_cast<uint32_t *>(rec);
        for (int widx = threadIdx.x; widx < 2 * nwh; widx += kThreads) {
            const int eta = widx / nwh;
            int ln, w;
            word_lane(widx % nwh, Wh, ln, w);
            uint32_t out = 0;
            for (int f = 0; f < F; ++f) {
                int e, d;
                field_owner(0, ln, w, f, bits, e, d);
                out |= static_cast<uint32_t>(codes[16 * eta + e][d]) << (f * bits);
            }
            area[widx] = out;
        }
        __syncthreads();   // the residual reads above complete before the rewrite below
    }
    if (first) {
        const int res_start = max(p.L_old, 32 * (L_new / 32));
        const int cnt = L_new - res_start;
        for (int idx = threadIdx.x; idx < cnt * D; idx += kThreads) {
            const int tok = res_start + idx / D, d = idx % D;
            res[(tok % 32) * D + d] = src[static_cast<long long>(tok - p.L_old) * D + d];
        }
    }
}

// Scales are non-negative, so their fp16 bit patterns order like their values: the
// largest scale of the layer is kept with integer atomicMax (one per CTA), for the
// decoder's choice of fp16 operand prescales.
__global__ void __launch_bounds__(kThreads) append_kernel(AppendParams p) {
    __shared__ __align__(16) float xs[32][kMaxD];
    __shared__ __align__(16) uint8_t codes[32][kMaxD];
    __shared__ unsigned cta_smax;
    if (threadIdx.x == 0) cta_smax = 0;
    __syncthreads();
    const int cta = blockIdx.x;
    int role;
    if (cta < p.nV) {
        role = 1;
        const int unit = cta / p.nhb, hbi = p.hb0 + cta % p.nhb;
        per_token_half(p, 1, unit, hbi, codes, &cta_smax);
    } else {
        role = 0;
        const int k = cta - p.nV;
        if (p.kmode == 1) {
            const int unit = k / p.nhb, hbi = p.hb0 + k % p.nhb;
            per_token_half(p, 0, unit, hbi, codes, &cta_smax);
        } else {
            const int per_unit = p.ng > 0 ? p.ng : 1;
            const int unit = k / per_unit, qi = k % per_unit;
            per_channel_group(p, unit, p.g0 + qi, p.ng > 0, qi == 0, xs, codes, &cta_smax);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && cta_smax) atomicMax(p.smax + role, cta_smax);
}

}  // namespace

cudaError_t launch_append(const AppendParams &p, cudaStream_t st) {
    if (p.D > kMaxD) return cudaErrorInvalidValue;
    const int grid = p.nV + p.nK;
    if (grid <= 0) return cudaSuccess;
    append_kernel<<<grid, kThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace kvq
