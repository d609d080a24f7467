// Append path of the INT2/INT4 token-mixed paged cache (sm_100a).
//
// "TriAxialKV per-role mixed-precision KV quantization" (Facts: quantizer, leftovers,
// page pools, decode path): every token carries a tag, INT2 or INT4.  INT2-tagged
// tokens are taken in arrival order; each run of 32 becomes one INT2 group, keys
// quantized per channel with 2 bits (over the group's 32 tokens) and values per token
// with 2 bits.  INT4-tagged tokens are quantized per token, keys and values with 4
// bits, into 16-token INT4 pages.  INT2 tokens whose group is not complete yet are
// routed through the same INT4 per-token path into two pending pages per request; their
// bf16 originals are kept (not attended) so the group can be quantized when its 32nd
// token arrives.
//
// Storage per layer and kv head: an INT2 pool of 32-token records (a group occupies two
// adjacent 16-token pages) followed by an INT4 pool of 16-token pages (the pending pages
// last); a per-request page table lists the INT2 groups from its front and the INT4 main
// pages from its back.  Page allocation is planned on the host (bump allocation in
// request order); the kernels write the new table entries.
//
// One launch per append (plus a tag scan when a call appends more than one token).
// CTA roles, per kv head:
//   INT4 page CTA   one INT4 main page touched by the call: quantize its new tokens,
//                   repack the page's key and value words.
//   INT2 CTA 0      the first group completed by the call (if any), then the open
//                   group's new tokens: bf16 originals into the staging slots and INT4
//                   codes into the pending pages (after the group has read the old
//                   staging slots).
//   INT2 CTA i > 0  group i completed by the call (its members all come from the input).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"
#include "kvq_quant.cuh"

namespace kvq {
namespace {

using namespace quant;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kD = 128;   // head_dim of paged plans
constexpr int kNJ = kD / 32;

// Position of the r-th new INT2 / INT4 token of request b in the call's input.
__device__ __forceinline__ int input_index(const PagedAppendParams &p, const int *inv, int b, int r) {
    return p.n == 1 ? 0 : inv[static_cast<long long>(b) * p.inv_stride + r];
}

// Quantize one token row per token (groups of 32 channels, `bits`), by one warp: the
// codes go to codes_row[D], the scale/zero pairs to the per-token s/z area of a unit at
// token u.  Tracks the largest scale in *smax_cta.
__device__ __forceinline__ void quant_token_row(const uint16_t *row, int bits, uint8_t *codes_row, uint8_t *sz,
                                                int u, unsigned *smax_cta) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < kNJ; ++j) {
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
        codes_row[32 * j + lane] = static_cast<uint8_t>(group_code(x, s, z, bits));
        if (lane == 0) {
            const int so = tok_sz_off(u, j, kNJ);
            *reinterpret_cast<uint16_t *>(sz + so) = s16;
            *reinterpret_cast<uint16_t *>(sz + so + 4 * kNJ) = z16;
            atomicMax(smax_cta, static_cast<unsigned>(s16));
        }
    }
}

// Rebuild the words of one 16-token half (role 0 keys, 1 values) from codes[e][d] for
// tokens e in [es, ee); tokens below es keep their bits, tokens from ee on read zero.
__device__ __forceinline__ void repack_half(uint32_t *area, int role, int bits, int es, int ee,
                                            uint8_t (*codes)[kD]) {
    const int Wh = kD * bits / 64, F = 32 / bits, nw = kD * bits / 2;
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

// Byte offsets inside a 16-token INT4 page: [K codes][K s/z][V codes][V s/z].
constexpr int kP4KC = 2 * kD * 4, kP4KS = 2 * kD, kP4VC = 2 * kD * 4;

// Write tokens of a 16-token INT4 page: slots [es, ee) get the input rows listed by
// `src_row(e)` (a bf16 pointer for K and for V).
template <class SrcFn>
__device__ void write_int4_page(uint8_t *page, int es, int ee, SrcFn src_row, uint8_t (*kc)[kD],
                                uint8_t (*vc)[kD], unsigned *smax_k, unsigned *smax_v) {
    const int warp = threadIdx.x >> 5;
    for (int e = es + warp; e < ee; e += kWarps) {
        const uint16_t *krow, *vrow;
        src_row(e, krow, vrow);
        quant_token_row(krow, 4, kc[e], page + kP4KC, e, smax_k);
        quant_token_row(vrow, 4, vc[e], page + kP4KC + kP4KS + kP4VC, e, smax_v);
    }
    __syncthreads();
    repack_half(reinterpret_cast<uint32_t *>(page), 0, 4, es, ee, kc);
    repack_half(reinterpret_cast<uint32_t *>(page + kP4KC + kP4KS), 1, 4, es, ee, vc);
    __syncthreads();
}

// Quantize one complete INT2 group from its 32 member rows into a 32-token record:
// keys per channel (2 bits), values per token (2 bits).
template <class SrcFn>
__device__ void write_int2_group(uint8_t *rec, SrcFn src_row, float (*xs)[kD], uint8_t (*kc)[kD],
                                 uint8_t (*vc)[kD], unsigned *smax_k, unsigned *smax_v) {
    constexpr int KC = 4 * kD * 2, KS = 4 * kD, VC = 4 * kD * 2;
    for (int idx = threadIdx.x; idx < 32 * kD; idx += kThreads) {
        const int u = idx / kD, d = idx % kD;
        const uint16_t *krow, *vrow;
        src_row(u, krow, vrow);
        xs[u][d] = bf16_to_f32(krow[d]);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < kD; d += kThreads) {
        float mn = xs[0][d], mx = xs[0][d];
        for (int u = 1; u < 32; ++u) {
            mn = fminf(mn, xs[u][d]);
            mx = fmaxf(mx, xs[u][d]);
        }
        float s, z;
        uint16_t s16, z16;
        group_params(mn, mx, 2, s, z, s16, z16);
        for (int u = 0; u < 32; ++u) kc[u][d] = static_cast<uint8_t>(group_code(xs[u][d], s, z, 2));
        const int so = chan_sz_off(d);
        *reinterpret_cast<uint16_t *>(rec + KC + so) = s16;
        *reinterpret_cast<uint16_t *>(rec + KC + so + 4) = z16;
        atomicMax(smax_k, static_cast<unsigned>(s16));
    }
    const int warp = threadIdx.x >> 5;
    for (int u = warp; u < 32; u += kWarps) {
        const uint16_t *krow, *vrow;
        src_row(u, krow, vrow);
        quant_token_row(vrow, 2, vc[u], rec + KC + KS + VC, u, smax_v);
    }
    __syncthreads();
    for (int hf = 0; hf < 2; ++hf) {
        repack_half(reinterpret_cast<uint32_t *>(rec + hf * 2 * kD * 2), 0, 2, 0, 16, kc + 16 * hf);
        repack_half(reinterpret_cast<uint32_t *>(rec + KC + KS + hf * 2 * kD * 2), 1, 2, 0, 16, vc + 16 * hf);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kThreads) paged_append_kernel(const PagedAppendParams p) {
    pdl_enter();
    __shared__ __align__(16) float xs[32][kD];
    __shared__ __align__(16) uint8_t kc[32][kD];
    __shared__ __align__(16) uint8_t vc[32][kD];
    __shared__ unsigned smax_k, smax_v;
    if (threadIdx.x == 0) smax_k = smax_v = 0;
    __syncthreads();

    const int h = blockIdx.x % p.Hkv;
    const int r = blockIdx.x / p.Hkv;
    const int tot4 = p.cta4_off[p.B];
    const bool role4 = r < tot4;
    const int rr = role4 ? r : r - tot4;
    const int *off = role4 ? p.cta4_off : p.cta2_off;
    int b = 0;
    while (b + 1 < p.B && off[b + 1] <= rr) ++b;
    const int idx = rr - off[b];
    const PagedReq &q = p.req[b];
    const long long unit = static_cast<long long>(b) * p.Hkv + h;
    const uint16_t *Kin = p.K + unit * p.n * kD, *Vin = p.V + unit * p.n * kD;
    constexpr int REC2 = 4 * kD * 2 + 4 * kD + 4 * kD * 2 + 4 * kD;
    constexpr int PAGE4 = kP4KC + kP4KS + kP4VC + 2 * kD;
    int *tab = p.table + static_cast<long long>(b) * p.P_cap;

    if (role4) {
        // main INT4 page: positions [16P, 16P + 16) of the request's INT4 stream
        const int first = q.n4_old / 16;
        const int P = first + idx;
        const int es = max(q.n4_old, 16 * P) - 16 * P;
        const int ee = min(q.n4_old + q.k4, 16 * P + 16) - 16 * P;
        const int n4p_old = (q.n4_old + 15) / 16;
        const int page = P < n4p_old ? q.last4 : q.base4 + (P - n4p_old);
        if (h == 0 && threadIdx.x == 0) tab[p.P_cap - 1 - P] = page;
        uint8_t *dst = p.pool4 + (static_cast<long long>(h) * p.n4_cap + page) * PAGE4;
        write_int4_page(dst, es, ee,
                        [&](int e, const uint16_t *&kr, const uint16_t *&vr) {
                            const int j = input_index(p, p.inv4, b, 16 * P + e - q.n4_old);
                            kr = Kin + static_cast<long long>(j) * kD;
                            vr = Vin + static_cast<long long>(j) * kD;
                        },
                        kc, vc, &smax_k, &smax_v);
    } else {
        uint16_t *stK = p.staging + (unit * 2) * 32 * kD;
        uint16_t *stV = stK + 32 * kD;
        const int c0 = 32 * q.n2g_old + q.np_old;   // INT2 stream positions before this call
        if (idx < q.ng) {
            // complete group idx: stream positions [32 (n2g_old + idx), +32)
            const int gbase = 32 * (q.n2g_old + idx);
            const int rec = q.base2 + idx;
            if (h == 0 && threadIdx.x == 0) tab[q.n2g_old + idx] = 2 * rec;
            uint8_t *dst = p.pool2 + (static_cast<long long>(h) * p.n2_cap + rec) * REC2;
            write_int2_group(dst,
                             [&](int u, const uint16_t *&kr, const uint16_t *&vr) {
                                 const int c = gbase + u;
                                 if (c < c0) {
                                     kr = stK + (c - 32 * q.n2g_old) * kD;
                                     vr = stV + (c - 32 * q.n2g_old) * kD;
                                 } else {
                                     const int j = input_index(p, p.inv2, b, c - c0);
                                     kr = Kin + static_cast<long long>(j) * kD;
                                     vr = Vin + static_cast<long long>(j) * kD;
                                 }
                             },
                             xs, kc, vc, &smax_k, &smax_v);
        }
        if (idx == 0) {
            // the open group: stream positions [32 (n2g_old + ng), c0 + k2) -> slots
            const int obase = 32 * (q.n2g_old + q.ng);
            const int first = max(c0, obase) - obase, last = c0 + q.k2 - obase;   // new slots [first, last)
            for (int i = threadIdx.x; i < (last - first) * kD; i += kThreads) {
                const int u = first + i / kD, d = i % kD;
                const int j = input_index(p, p.inv2, b, obase + u - c0);
                stK[u * kD + d] = Kin[static_cast<long long>(j) * kD + d];
                stV[u * kD + d] = Vin[static_cast<long long>(j) * kD + d];
            }
            __syncthreads();
            for (int pg = first / 16; pg * 16 < last; ++pg) {
                const int es = max(first, 16 * pg) - 16 * pg, ee = min(last, 16 * pg + 16) - 16 * pg;
                uint8_t *dst = p.pool4 + (static_cast<long long>(h) * p.n4_cap + p.pend_base + 2 * b + pg) * PAGE4;
                write_int4_page(dst, es, ee,
                                [&](int e, const uint16_t *&kr, const uint16_t *&vr) {
                                    kr = stK + (16 * pg + e) * kD;
                                    vr = stV + (16 * pg + e) * kD;
                                },
                                kc, vc, &smax_k, &smax_v);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (smax_k) atomicMax(p.smax, smax_k);
        if (smax_v) atomicMax(p.smax + 1, smax_v);
    }
}

// Per request: input index of the r-th INT2-tagged and r-th INT4-tagged new token.
__global__ void __launch_bounds__(1024) paged_scan_kernel(const uint8_t *tags, int n, int *inv2, int *inv4,
                                                          int stride) {
    pdl_enter();
    __shared__ int part2[1024];
    const int b = blockIdx.x;
    const uint8_t *tg = tags + static_cast<long long>(b) * n;
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int lo = min(n, static_cast<int>(threadIdx.x) * per), hi = min(n, lo + per);
    int c2 = 0;
    for (int i = lo; i < hi; ++i) c2 += tg[i] == 2;
    part2[threadIdx.x] = c2;
    __syncthreads();
    if (threadIdx.x == 0) {   // exclusive prefix over the chunks (1024 entries)
        int run = 0;
        for (int i = 0; i < static_cast<int>(blockDim.x); ++i) {
            const int v = part2[i];
            part2[i] = run;
            run += v;
        }
    }
    __syncthreads();
    int r2 = part2[threadIdx.x], r4 = lo - r2;
    int *o2 = inv2 + static_cast<long long>(b) * stride, *o4 = inv4 + static_cast<long long>(b) * stride;
    for (int i = lo; i < hi; ++i) {
        if (tg[i] == 2) o2[r2++] = i;
        else o4[r4++] = i;
    }
}

}  // namespace

cudaError_t launch_paged_scan(const uint8_t *tags, int B, int n, int *inv2, int *inv4, int inv_stride,
                              cudaStream_t st) {
    cudaError_t e = launch_pdl(paged_scan_kernel, dim3(B), dim3(1024), 0, st, tags, n, inv2, inv4, inv_stride);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_paged_append(const PagedAppendParams &p, int grid, cudaStream_t st) {
    if (grid <= 0) return cudaSuccess;
    cudaError_t e = launch_pdl(paged_append_kernel, dim3(grid), dim3(kThreads), 0, st, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace kvq
