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
#include "kvq_quant.cuh"

namespace kvq {
namespace {

using namespace quant;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxD = 256;

// Per-token quantization of the new tokens of one 16-token half-block and repacking
// of its words.  role 0 = keys (per-token mode), 1 = values.
__device__ void per_token_half(const AppendParams &p, int role, int unit, int hbi, int L_old, int n,
                               uint8_t (*codes)[kMaxD], unsigned *cta_smax) {
    const int D = p.D, nj = D / 32;
    const int bits = role ? p.bv : p.bk;
    const uint16_t *src = (role ? p.V : p.K) + static_cast<long long>(unit) * p.n * D;
    const int L_new = L_old + n;
    const int u0 = 16 * hbi;
    const int es = max(L_old, u0) - u0, ee = min(L_new, u0 + 16) - u0;
    const int blk = hbi >> 1, eta = hbi & 1;
    uint8_t *rec = p.rec + rec_index(p.btab, unit / p.Hkv, p.Hkv, unit % p.Hkv, p.cap_blk, blk) * p.rec_bytes;
    uint8_t *sz = rec + (role ? p.kc + p.ks + p.vc : p.kc);
    uint32_t *area = reinterpret_cast<uint32_t *>(rec + (role ? p.kc + p.ks : 0) +
                                                  static_cast<long long>(eta) * 2 * D * bits);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Wh = D * bits / 64, F = 32 / bits, nw = D * bits / 2;

    // the half's words this thread rewrites, loaded up front (fields of tokens already in
    // the half are kept); a half that starts with these tokens is rebuilt from zero
    uint32_t old[kMaxD * 8 / 2 / kThreads];
#pragma unroll
    for (int r = 0; r < kMaxD * 8 / 2 / kThreads; ++r) {
        const int widx = threadIdx.x + r * kThreads;
        old[r] = (es > 0 && widx < nw) ? area[widx] : 0u;
    }

    // one warp per (new token, 32-channel group)
    for (int it = warp; it < (ee - es) * nj; it += kWarps) {
        const int e = es + it / nj, j = it % nj;
        const int tok = u0 + e;
        const uint16_t *row = src + static_cast<long long>(tok - L_old) * D;
        const int u = 16 * eta + e;
        {
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

    const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
    for (int r = 0; r < kMaxD * 8 / 2 / kThreads; ++r) {
        const int widx = threadIdx.x + r * kThreads;
        if (widx >= nw) break;
        int ln, w;
        word_lane(widx, Wh, ln, w);
        uint32_t out = 0;
        for (int f = 0; f < F; ++f) {
            int e, d;
            field_owner(role, ln, w, f, bits, e, d);
            uint32_t c;
            if (e >= es && e < ee) c = codes[e][d];
            else if (e < es) c = (old[r] >> (f * bits)) & mask;
            else c = 0;
            out |= c << (f * bits);
        }
        area[widx] = out;
    }
}

// Per-channel quantization of one completed 32-token key group; the CTA with
// first == true also writes the new residual tokens of its (b, h) afterwards.
__device__ void per_channel_group(const AppendParams &p, int unit, int q, bool do_group, bool first, int L_old,
                                  int n, float (*xs)[kMaxD], uint8_t (*codes)[kMaxD], unsigned *cta_smax) {
    const int D = p.D;
    const uint16_t *src = p.K + static_cast<long long>(unit) * p.n * D;
    uint16_t *res = p.res + static_cast<long long>(unit) * 32 * D;
    const int L_new = L_old + n;
    if (do_group) {
        const int t0 = 32 * q;
        for (int idx = threadIdx.x; idx < 32 * D; idx += kThreads) {
            const int u = idx / D, d = idx % D, tok = t0 + u;
            const uint16_t v = tok < L_old ? res[u * D + d] : src[static_cast<long long>(tok - L_old) * D + d];
            xs[u][d] = bf16_to_f32(v);
        }
        __syncthreads();
        uint8_t *rec = p.rec + rec_index(p.btab, unit / p.Hkv, p.Hkv, unit % p.Hkv, p.cap_blk, q) * p.rec_bytes;
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
        const int res_start = max(L_old, 32 * (L_new / 32));
        const int cnt = L_new - res_start;
        for (int idx = threadIdx.x; idx < cnt * D; idx += kThreads) {
            const int tok = res_start + idx / D, d = idx % D;
            res[(tok % 32) * D + d] = src[static_cast<long long>(tok - L_old) * D + d];
        }
    }
}

// Scales are non-negative, so their fp16 bit patterns order like their values: the
// largest scale of the layer is kept with integer atomicMax (one per CTA), for the
// decoder's choice of fp16 operand prescales.
__global__ void __launch_bounds__(kThreads) append_kernel(AppendParams p) {
    pdl_enter();
    __shared__ __align__(16) float xs[32][kMaxD];
    __shared__ __align__(16) uint8_t codes[32][kMaxD];
    __shared__ unsigned cta_smax;
    if (threadIdx.x == 0) cta_smax = 0;
    __syncthreads();
    const int cta = blockIdx.x;
    // this CTA's request range: the launch's own, or (ragged) its request's
    auto range = [&](int unit, int &L_old, int &n, int &hb0, int &nhb, int &g0, int &ng) {
        if (!p.ragged) {
            L_old = p.L_old, n = p.n, hb0 = p.hb0, nhb = p.nhb, g0 = p.g0, ng = p.ng;
            return;
        }
        const int b = unit / p.Hkv;
        if (p.ragged_dev) {
            L_old = p.ragged_dev[b];
            n = p.ragged_dev[p.B + b];
        } else {
            L_old = p.L_old_r[b];
            n = p.n_r[b];
        }
        const int L_new = L_old + n;
        hb0 = L_old / 16;
        nhb = n > 0 ? (L_new - 1) / 16 - hb0 + 1 : 0;
        g0 = L_old / 32;
        ng = L_new / 32 - g0;
    };
    int role, L_old, n, hb0, nhb, g0, ng;
    if (cta < p.nV) {
        role = 1;
        const int unit = cta / p.nhb, hi = cta % p.nhb;
        range(unit, L_old, n, hb0, nhb, g0, ng);
        if (hi < nhb) per_token_half(p, 1, unit, hb0 + hi, L_old, n, codes, &cta_smax);
    } else {
        role = 0;
        const int k = cta - p.nV;
        if (p.kmode == 1) {
            const int unit = k / p.nhb, hi = k % p.nhb;
            range(unit, L_old, n, hb0, nhb, g0, ng);
            if (hi < nhb) per_token_half(p, 0, unit, hb0 + hi, L_old, n, codes, &cta_smax);
        } else {
            const int per_unit = p.ng > 0 ? p.ng : 1;
            const int unit = k / per_unit, qi = k % per_unit;
            range(unit, L_old, n, hb0, nhb, g0, ng);
            if (qi < ng || qi == 0)
                per_channel_group(p, unit, g0 + qi, qi < ng, qi == 0, L_old, n, xs, codes, &cta_smax);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && cta_smax) atomicMax(p.smax + role, cta_smax);
    // carry the maxima of the old length into the new length's slot
    if (cta == 0 && threadIdx.x == 0 && p.smax_prev != p.smax) {
        atomicMax(p.smax, p.smax_prev[0]);
        atomicMax(p.smax + 1, p.smax_prev[1]);
    }
}

struct TableChunk {
    int *dst;
    int n;
    int v[1000];   // keeps the parameter block under 4 KB
};

__global__ void set_table_kernel(const TableChunk c) {
    pdl_enter();
    for (int i = threadIdx.x; i < c.n; i += blockDim.x) c.dst[i] = c.v[i];
}

struct ScatterChunk {
    int *dst;
    int n;
    int idx[500], v[500];   // keeps the parameter block under 4 KB
};

__global__ void scatter_table_kernel(const ScatterChunk c) {
    pdl_enter();
    for (int i = threadIdx.x; i < c.n; i += blockDim.x) c.dst[c.idx[i]] = c.v[i];
}

}  // namespace

cudaError_t launch_set_table(int *dst, const int *vals, int n, cudaStream_t st) {
    for (int i0 = 0; i0 < n; i0 += 1000) {
        TableChunk c;
        c.dst = dst + i0;
        c.n = n - i0 < 1000 ? n - i0 : 1000;
        for (int i = 0; i < c.n; ++i) c.v[i] = vals[i0 + i];
        cudaError_t e = launch_pdl(set_table_kernel, dim3(1), dim3(256), 0, st, c);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t launch_scatter_table(int *dst, const int *idx, const int *vals, int n, cudaStream_t st) {
    for (int i0 = 0; i0 < n; i0 += 500) {
        ScatterChunk c;
        c.dst = dst;
        c.n = n - i0 < 500 ? n - i0 : 500;
        for (int i = 0; i < c.n; ++i) {
            c.idx[i] = idx[i0 + i];
            c.v[i] = vals[i0 + i];
        }
        cudaError_t e = launch_pdl(scatter_table_kernel, dim3(1), dim3(256), 0, st, c);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams &p, cudaStream_t st) {


    if (p.D > kMaxD) return cudaErrorInvalidValue;
    const int grid = p.nV + p.nK;
    if (grid <= 0) return cudaSuccess;
    cudaError_t e = launch_pdl(append_kernel, dim3(grid), dim3(kThreads), 0, st, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace kvq
