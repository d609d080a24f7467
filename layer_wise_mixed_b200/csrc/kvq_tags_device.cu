// Per-tag distortion D_k(b) on the GPU ("TriAxialKV per-role mixed-precision KV
// quantization for agentic prefills", Facts: per-tag distortion, quantizer, leftover
// routing).  The definition is the host entry point's (kvq_tag_distortion): tag k's tokens
// at b bits and every other token exact, causal attention over the calibration prefill,
// output MSE per query head; max over heads, mean over requests, sum over layers.  All
// attention arithmetic is fp64 on the CUDA cores, so the results equal the host's up to
// the order of the sums.
//
// Per layer:
//  1. calib_token_kernel: every token's 4-bit per-token K and V (groups of 32 channels),
//     and the 2-bit path's per-token values; a tag's last (count mod 32) tokens take the
//     4-bit K and V on the 2-bit path too.  Dequantized to fp64 (code * s + z is exact).
//  2. calib_keygroup_kernel: the 2-bit path's keys, per channel over consecutive 32-token
//     groups of one tag's tokens of a request, in token order.
//  3. calib_attn_kernel: one CTA per (32 queries, query head, request).  The exact
//     attention of each query row once (row max m_i in a first pass, then l_i and the
//     numerator N_i with weights exp(s - m_i)); then, per (tag, b), only the terms of the
//     tag's tokens change: O'_i = (N_i + dN_i) / (l_i + dl_i), dN and dl summed over
//     those tokens with the same m_i.  The CTA writes its sum of squared differences.
//     Its 16-token tiles of fp64 rows (exact and quantized) come by cp.async into two
//     buffers, the next tile of the CTA's whole sequence of passes in flight while the
//     current one is used.
// Then calib_reduce_kernel takes the per-head means, the max over heads, the mean over
// requests and the sum over layers, in a fixed order.
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

#include "kvq.h"
#include "kvq_internal.h"
#include "kvq_quant.cuh"

namespace {

using kvq::quant::bf16_to_f32;

constexpr int kQB = 32;        // query rows per attention CTA
constexpr int kKT = 16;        // key rows per staged tile
constexpr int kThreads = 256;  // attention CTA: thread = (query row t / 8, lane group t % 8)

struct CalibDims {
    int NL, R, Hq, Hkv, D, T, ntags, nqb, maxg;
};

// Workspace regions (byte offsets, 256-byte aligned).
struct CalibLayout {
    size_t list, off, tags, rank, gstart, ngroups, kx, vx, kq2, vq2, kq4, vq4, part, res, total;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

CalibLayout calib_layout(const CalibDims &d) {
    CalibLayout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align256(o + bytes);
        return at;
    };
    const size_t RT = static_cast<size_t>(d.R) * d.T;
    L.list = take(RT * 4);                                           // tokens by (tag, position)
    L.off = take(static_cast<size_t>(d.R) * (d.ntags + 1) * 4);      // list offset of each tag
    L.tags = take(RT * 4);
    L.rank = take(RT * 4);                                           // position in its tag's list
    L.gstart = take(static_cast<size_t>(d.R) * d.maxg * 4);          // list index of each 2-bit key group
    L.ngroups = take(static_cast<size_t>(d.R) * 4);
    const size_t arr = static_cast<size_t>(d.R) * d.Hkv * d.T * d.D * sizeof(double);   // one layer
    L.kx = take(arr);   // exact keys and values in fp64
    L.vx = take(arr);
    L.kq2 = take(arr);
    L.vq2 = take(arr);
    L.kq4 = take(arr);
    L.vq4 = take(arr);
    L.part = take(static_cast<size_t>(d.NL) * d.R * d.Hq * d.nqb * d.ntags * 2 * sizeof(double));
    L.res = take(static_cast<size_t>(d.ntags) * 2 * sizeof(double));
    L.total = o;
    return L;
}

// One group of 32 values quantized at `bits` with the cache's binary32 steps, returned
// dequantized in fp64 (the code times the fp16 scale is exact in fp64, so the fma rounds
// once, like code * s + z).
template <int BITS>
__device__ __forceinline__ void dequant32(const float (&x)[32], double (&out)[32]) {
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int i = 1; i < 32; ++i) {
        mn = fminf(mn, x[i]);
        mx = fmaxf(mx, x[i]);
    }
    float s, z;
    uint16_t s16, z16;
    kvq::quant::group_params(mn, mx, BITS, s, z, s16, z16);
#pragma unroll
    for (int i = 0; i < 32; ++i)
        out[i] = fma(static_cast<double>(kvq::quant::group_code(x[i], s, z, BITS)), static_cast<double>(s),
                     static_cast<double>(z));
}

__device__ __forceinline__ void load32(const uint16_t *src, float (&x)[32]) {
    const uint4 *w = reinterpret_cast<const uint4 *>(src);   // 64 bytes, 16-byte aligned
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 u = w[i];
        const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[8 * i + 2 * j] = __uint_as_float(ws[j] << 16);
            x[8 * i + 2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
        }
    }
}

// Thread = (token t, 32-channel group g) of one (request, kv head) of layer `lay`; it also
// writes the exact keys and values in fp64, the form the attention kernel stages.
__global__ void calib_token_kernel(const uint16_t *__restrict__ K, const uint16_t *__restrict__ V, int lay,
                                   CalibDims d, const int *__restrict__ tags, const int *__restrict__ rank,
                                   const int *__restrict__ off, double *kx, double *vx, double *kq2, double *vq2,
                                   double *kq4, double *vq4) {
    const int nj = d.D / 32;
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(d.T) * nj) return;
    const int t = static_cast<int>(idx / nj), g = static_cast<int>(idx % nj);
    const int rh = blockIdx.y;   // request * Hkv + kv head
    const int r = rh / d.Hkv;
    const long long src = ((static_cast<long long>(lay) * d.R * d.Hkv + rh) * d.T + t) * d.D + 32 * g;
    const long long dst = (static_cast<long long>(rh) * d.T + t) * d.D + 32 * g;
    float xk[32], xv[32];
    double o[32];
    load32(K + src, xk);
    load32(V + src, xv);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        kx[dst + i] = static_cast<double>(xk[i]);
        vx[dst + i] = static_cast<double>(xv[i]);
    }
    const int k = tags[static_cast<long long>(r) * d.T + t];
    const int n = off[r * (d.ntags + 1) + k + 1] - off[r * (d.ntags + 1) + k];
    const bool leftover = rank[static_cast<long long>(r) * d.T + t] >= n / 32 * 32;
    dequant32<4>(xk, o);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        kq4[dst + i] = o[i];
        if (leftover) kq2[dst + i] = o[i];   // else: calib_keygroup_kernel
    }
    dequant32<4>(xv, o);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        vq4[dst + i] = o[i];
        if (leftover) vq2[dst + i] = o[i];
    }
    if (!leftover) {
        dequant32<2>(xv, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) vq2[dst + i] = o[i];
    }
}

// CTA = (2-bit key group gi, request * Hkv + kv head); thread = channel (blockDim.x = D).
__global__ void calib_keygroup_kernel(const uint16_t *__restrict__ K, int lay, CalibDims d,
                                      const int *__restrict__ list, const int *__restrict__ gstart,
                                      const int *__restrict__ ngroups, double *kq2) {
    const int rh = blockIdx.y, r = rh / d.Hkv, gi = blockIdx.x, c = threadIdx.x;
    if (gi >= ngroups[r] || c >= d.D) return;
    const int *tok = list + static_cast<long long>(r) * d.T + gstart[r * d.maxg + gi];
    const uint16_t *base = K + (static_cast<long long>(lay) * d.R * d.Hkv + rh) * d.T * d.D + c;
    float x[32];
    double o[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = bf16_to_f32(base[static_cast<long long>(tok[i]) * d.D]);
    dequant32<2>(x, o);
    double *dst = kq2 + static_cast<long long>(rh) * d.T * d.D + c;
#pragma unroll
    for (int i = 0; i < 32; ++i) dst[static_cast<long long>(tok[i]) * d.D] = o[i];
}

template <int D>
struct CalibSmem {
    double q[kQB][D + 2];                  // rows padded: 16-byte aligned, bank-spread
    double t[2][4][kKT][D + 2];            // two tile buffers: exact k, exact v, quantized k, quantized v
    double pe[kQB][kKT + 2], pq[kQB][kKT + 2];   // exact / quantized weights exp(s - m_i)
    double red[kThreads / 32];
    int tok[2][kKT];                       // token of each tile row (-1: none)
};

__device__ __forceinline__ void cp16(void *smem, const void *gmem) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait_prev() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Dot products of query row qi with tile rows kp and kp + 8: the even and the odd
// channels in two chains each (channel order within a chain), then added.
template <int D>
__device__ __forceinline__ void dot2(const double (*q)[D + 2], const double (*k)[D + 2], int qi, int kp, double &s0,
                                     double &s1) {
    double e0 = 0.0, o0 = 0.0, e1 = 0.0, o1 = 0.0;
#pragma unroll 8
    for (int c = 0; c < D; c += 2) {
        const double2 a = *reinterpret_cast<const double2 *>(&q[qi][c]);
        const double2 b0 = *reinterpret_cast<const double2 *>(&k[kp][c]);
        const double2 b1 = *reinterpret_cast<const double2 *>(&k[kp + 8][c]);
        e0 = fma(a.x, b0.x, e0);
        o0 = fma(a.y, b0.y, o0);
        e1 = fma(a.x, b1.x, e1);
        o1 = fma(a.y, b1.y, o1);
    }
    s0 = e0 + o0;
    s1 = e1 + o1;
}

// dot2 against the exact rows k and the quantized rows kh at once (one query load per
// channel pair); each product is summed exactly as dot2 sums it.
template <int D>
__device__ __forceinline__ void dot4(const double (*q)[D + 2], const double (*k)[D + 2], const double (*kh)[D + 2],
                                     int qi, int kp, double &se0, double &se1, double &sq0, double &sq1) {
    double e0 = 0.0, o0 = 0.0, e1 = 0.0, o1 = 0.0, f0 = 0.0, p0 = 0.0, f1 = 0.0, p1 = 0.0;
#pragma unroll 4
    for (int c = 0; c < D; c += 2) {
        const double2 a = *reinterpret_cast<const double2 *>(&q[qi][c]);
        const double2 b0 = *reinterpret_cast<const double2 *>(&k[kp][c]);
        const double2 b1 = *reinterpret_cast<const double2 *>(&k[kp + 8][c]);
        const double2 h0 = *reinterpret_cast<const double2 *>(&kh[kp][c]);
        const double2 h1 = *reinterpret_cast<const double2 *>(&kh[kp + 8][c]);
        e0 = fma(a.x, b0.x, e0);
        o0 = fma(a.y, b0.y, o0);
        e1 = fma(a.x, b1.x, e1);
        o1 = fma(a.y, b1.y, o1);
        f0 = fma(a.x, h0.x, f0);
        p0 = fma(a.y, h0.y, p0);
        f1 = fma(a.x, h1.x, f1);
        p1 = fma(a.y, h1.y, p1);
    }
    se0 = e0 + o0;
    se1 = e1 + o1;
    sq0 = f0 + p0;
    sq1 = f1 + p1;
}

__device__ __forceinline__ double sum8(double x) {   // over the 8 lanes of a query row
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    return x;
}

__device__ __forceinline__ double max8(double x) {
    x = fmax(x, __shfl_xor_sync(0xffffffffu, x, 1));
    x = fmax(x, __shfl_xor_sync(0xffffffffu, x, 2));
    x = fmax(x, __shfl_xor_sync(0xffffffffu, x, 4));
    return x;
}

// Where a CTA is in its sequence of 16-token tiles: pass 0 (row max over tokens 0..i_max),
// pass 1 (l and N over the same tiles), then pass 2 for every (tag with a token <= i_max,
// b): the tag's tokens in list order.
struct TilePos {
    int ph, k, bi, ti, nt;   // pass, tag, bit index (0: 2 bits, 1: 4 bits), tile, tiles in the pass
};

// CTA = (query block qb, query head hq, request r) of layer `lay`.  Thread t: query row
// qi = t / 8 of the block; as a scorer it takes tile rows sub and sub + 8 (sub = t % 8),
// as an accumulator the channels 16m + 2 sub + {0, 1}.  Tiles are fp64 rows copied by
// cp.async into two buffers: the next tile (of any pass) is in flight while the current
// one is used.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    calib_attn_kernel(const uint16_t *__restrict__ Q, int lay, CalibDims d, double rs, const int *__restrict__ list,
                      const int *__restrict__ off, const double *kx, const double *vx, const double *kq2,
                      const double *vq2, const double *kq4, const double *vq4, double *part) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    CalibSmem<D> &sm = *reinterpret_cast<CalibSmem<D> *>(smem_raw);
    constexpr int NM = D / 16;   // channel pairs per accumulating thread
    const int tid = threadIdx.x, qi = tid >> 3, sub = tid & 7;
    const int qb = d.nqb - 1 - static_cast<int>(blockIdx.x);   // longest rows first
    const int hq = blockIdx.y, r = blockIdx.z, h = hq / (d.Hq / d.Hkv);
    const int i0 = qb * kQB, i = i0 + qi;
    const int i_max = min(i0 + kQB, d.T) - 1;
    const bool valid_q = i < d.T;
    const uint16_t *qbase = Q + ((static_cast<long long>(lay) * d.R + r) * d.Hq + hq) * d.T * D;
    const long long uo = (static_cast<long long>(r) * d.Hkv + h) * d.T * D;   // (request, kv head) in one layer
    const double *kxp = kx + uo, *vxp = vx + uo;
    const int *offr = off + r * (d.ntags + 1);
    const int *listr = list + static_cast<long long>(r) * d.T;
    const int nt_exact = i_max / kKT + 1;

    // tiles of tag k: its list entries <= i_max (the list is in token order)
    auto tag_tiles = [&](int k) {
        const int a = offr[k];
        int lo = 0, hi = offr[k + 1] - a;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (listr[a + mid] <= i_max)
                lo = mid + 1;
            else
                hi = mid;
        }
        return (lo + kKT - 1) / kKT;
    };
    auto advance = [&](TilePos &p) {   // false past the last tile
        if (++p.ti < p.nt) return true;
        p.ti = 0;
        if (p.ph == 0) {
            p.ph = 1;
            return true;
        }
        if (p.ph == 1) {
            p.ph = 2;
            p.k = 0;
            p.bi = 0;
        } else if (p.bi == 0) {
            p.bi = 1;
            return true;
        } else {
            ++p.k;
            p.bi = 0;
        }
        while (p.k < d.ntags && (p.nt = tag_tiles(p.k)) == 0) ++p.k;
        return p.k < d.ntags;
    };
    // copies of the tile at p into buffer buf (rows without a token are zeroed), one group
    auto issue = [&](int buf, const TilePos &p) {
        const int narr = p.ph == 0 ? 1 : (p.ph == 1 ? 2 : 4);
        const int a = p.ph == 2 ? offr[p.k] : 0;
        const int n = p.ph == 2 ? offr[p.k + 1] - a : 0;
        const int first = p.ti * kKT;
        const double *kqp = (p.bi ? kq4 : kq2) + uo, *vqp = (p.bi ? vq4 : vq2) + uo;
        for (int e = tid; e < kKT * (D / 2); e += kThreads) {
            const int row = e / (D / 2), ch = e % (D / 2);
            const int tok = p.ph == 2 ? (first + row < n ? listr[a + first + row] : -1)
                                      : (first + row <= i_max ? first + row : -1);
            if (ch == 0) sm.tok[buf][row] = tok;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                if (x >= narr) break;
                const double *src = x == 0 ? kxp : x == 1 ? vxp : x == 2 ? kqp : vqp;
                double *dst = &sm.t[buf][x][row][2 * ch];
                if (tok >= 0)
                    cp16(dst, src + static_cast<long long>(tok) * D + 2 * ch);
                else
                    *reinterpret_cast<double2 *>(dst) = make_double2(0.0, 0.0);
            }
        }
        cp_commit();
    };

    TilePos cur{0, 0, 0, 0, nt_exact};
    issue(0, cur);
    for (int e = tid; e < kQB * D / 8; e += kThreads) {   // query rows as fp64 (bf16 is exact)
        const int row = e / (D / 8), chunk = e % (D / 8);
        double2 *o = reinterpret_cast<double2 *>(&sm.q[row][8 * chunk]);
        if (i0 + row < d.T) {
            const uint4 u = *reinterpret_cast<const uint4 *>(qbase + static_cast<long long>(i0 + row) * D + 8 * chunk);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                o[j] = make_double2(static_cast<double>(__uint_as_float(w[j] << 16)),
                                    static_cast<double>(__uint_as_float(w[j] & 0xffff0000u)));
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = make_double2(0.0, 0.0);
        }
    }

    double m = -INFINITY, l = 0.0, dl = 0.0;
    double2 N[NM], A[NM], B[NM];   // exact numerator; sum pq vh and sum pe v of the current (tag, b)
#pragma unroll
    for (int mm = 0; mm < NM; ++mm) N[mm] = make_double2(0.0, 0.0);
    for (int buf = 0;; buf ^= 1) {
        TilePos nxt = cur;
        const bool more = advance(nxt);
        if (more)
            issue(buf ^ 1, nxt);
        else
            cp_commit();   // an empty group keeps the wait below uniform
        cp_wait_prev();     // this tile's copies (the group before the newest) have landed
        __syncthreads();
        const double(*tk)[D + 2] = sm.t[buf][0];
        if (cur.ph == 0) {   // row max of s_ij = (q_i . k_j) rs over j <= i
            const int j0 = cur.ti * kKT;
            double s0, s1;
            dot2<D>(sm.q, tk, qi, sub, s0, s1);
            if (valid_q && j0 + sub <= i) m = fmax(m, s0 * rs);
            if (valid_q && j0 + sub + 8 <= i) m = fmax(m, s1 * rs);
            if (cur.ti == cur.nt - 1) m = max8(m);
        } else if (cur.ph == 1) {   // l_i and N_i with the exact weights exp(s_ij - m_i)
            const int j0 = cur.ti * kKT;
            double s0, s1;
            dot2<D>(sm.q, tk, qi, sub, s0, s1);
            const double p0 = valid_q && j0 + sub <= i ? exp(s0 * rs - m) : 0.0;
            const double p1 = valid_q && j0 + sub + 8 <= i ? exp(s1 * rs - m) : 0.0;
            sm.pe[qi][sub] = p0;
            sm.pe[qi][sub + 8] = p1;
            l += p0;
            l += p1;
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < kKT; ++kk) {
                const double p = sm.pe[qi][kk];
#pragma unroll
                for (int mm = 0; mm < NM; ++mm) {
                    const double2 vv = *reinterpret_cast<const double2 *>(&sm.t[buf][1][kk][16 * mm + 2 * sub]);
                    N[mm].x = fma(p, vv.x, N[mm].x);
                    N[mm].y = fma(p, vv.y, N[mm].y);
                }
            }
            if (cur.ti == cur.nt - 1) l = sum8(l);
        } else {   // the tag's tokens j <= i at b bits; A and B apart, so exact levels give 0 exactly
            if (cur.ti == 0) {
#pragma unroll
                for (int mm = 0; mm < NM; ++mm) {
                    A[mm] = make_double2(0.0, 0.0);
                    B[mm] = make_double2(0.0, 0.0);
                }
                dl = 0.0;
            }
            double se0, se1, sq0, sq1;
            dot4<D>(sm.q, tk, sm.t[buf][2], qi, sub, se0, se1, sq0, sq1);
            const int t0 = sm.tok[buf][sub], t1 = sm.tok[buf][sub + 8];
            const bool v0 = valid_q && t0 >= 0 && t0 <= i, v1 = valid_q && t1 >= 0 && t1 <= i;
            const double pe0 = v0 ? exp(se0 * rs - m) : 0.0, pq0 = v0 ? exp(sq0 * rs - m) : 0.0;
            const double pe1 = v1 ? exp(se1 * rs - m) : 0.0, pq1 = v1 ? exp(sq1 * rs - m) : 0.0;
            sm.pe[qi][sub] = pe0;
            sm.pq[qi][sub] = pq0;
            sm.pe[qi][sub + 8] = pe1;
            sm.pq[qi][sub + 8] = pq1;
            dl += pq0 - pe0;
            dl += pq1 - pe1;
            __syncthreads();
#pragma unroll 2
            for (int kk = 0; kk < kKT; ++kk) {
                const double pe = sm.pe[qi][kk], pq = sm.pq[qi][kk];
#pragma unroll
                for (int mm = 0; mm < NM; ++mm) {
                    const double2 vx2 = *reinterpret_cast<const double2 *>(&sm.t[buf][1][kk][16 * mm + 2 * sub]);
                    const double2 vh = *reinterpret_cast<const double2 *>(&sm.t[buf][3][kk][16 * mm + 2 * sub]);
                    A[mm].x = fma(pq, vh.x, A[mm].x);
                    A[mm].y = fma(pq, vh.y, A[mm].y);
                    B[mm].x = fma(pe, vx2.x, B[mm].x);
                    B[mm].y = fma(pe, vx2.y, B[mm].y);
                }
            }
            if (cur.ti == cur.nt - 1) {   // the pass's squared output differences, summed over the CTA
                const double dls = sum8(dl);
                double err = 0.0;
                if (valid_q) {
                    const double lq = l + dls;
#pragma unroll
                    for (int mm = 0; mm < NM; ++mm) {
                        const double ex = (N[mm].x + (A[mm].x - B[mm].x)) / lq - N[mm].x / l;
                        const double ey = (N[mm].y + (A[mm].y - B[mm].y)) / lq - N[mm].y / l;
                        err += ex * ex;
                        err += ey * ey;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) err += __shfl_xor_sync(0xffffffffu, err, o);
                if ((tid & 31) == 0) sm.red[tid >> 5] = err;
                __syncthreads();
                if (tid == 0) {
                    double s = 0.0;
                    for (int w = 0; w < kThreads / 32; ++w) s += sm.red[w];
                    part[((((static_cast<long long>(lay) * d.R + r) * d.Hq + hq) * d.nqb + qb) * d.ntags + cur.k) * 2 +
                         cur.bi] = s;
                }
            }
        }
        __syncthreads();   // this buffer (and sm.pe, sm.red) is free again
        if (!more) break;
        cur = nxt;
    }
}

// res[k][b]: sum over layers of the mean over requests of the max over query heads of
// the output MSE (the CTA sums over query blocks, divided by T x D).
__global__ void calib_reduce_kernel(const double *__restrict__ part, CalibDims d, double *res) {
    for (int kb = threadIdx.x; kb < 2 * d.ntags; kb += blockDim.x) {
        const int k = kb >> 1, bi = kb & 1;
        const double td = static_cast<double>(static_cast<long long>(d.T) * d.D);
        double s = 0.0;
        for (int lay = 0; lay < d.NL; ++lay) {
            double msum = 0.0;
            for (int r = 0; r < d.R; ++r) {
                double w = 0.0;
                for (int hq = 0; hq < d.Hq; ++hq) {
                    double e = 0.0;
                    for (int qb = 0; qb < d.nqb; ++qb)
                        e += part[((((static_cast<long long>(lay) * d.R + r) * d.Hq + hq) * d.nqb + qb) * d.ntags + k) *
                                      2 +
                                  bi];
                    w = fmax(w, e / td);
                }
                msum += w;
            }
            s += msum / d.R;
        }
        res[kb] = s;
    }
}

int check_dims(int NL, int R, int Hq, int Hkv, int D, int T, int ntags, CalibDims &d) {
    if (NL < 1 || R < 1 || Hq < 1 || Hkv < 1 || T < 1 || ntags < 1)
        return kvq::host_fail(KVQ_EINVAL, "layers, requests, heads, T and num_tags must be positive");
    if (Hq % Hkv) return kvq::host_fail(KVQ_EINVAL, "n_q_heads must be a multiple of n_kv_heads");
    if (D != 64 && D != 128) return kvq::host_fail(KVQ_EUNSUPPORTED, "head_dim must be 64 or 128 on the device path");
    if (Hq > 65535 || R > 65535 || static_cast<long long>(R) * Hkv > 65535)
        return kvq::host_fail(KVQ_EUNSUPPORTED, "too many heads or requests for one launch");
    d = CalibDims{NL, R, Hq, Hkv, D, T, ntags, (T + kQB - 1) / kQB, T / 32 + 1};
    return KVQ_OK;
}

template <int D>
cudaError_t launch_attn(const uint16_t *Q, int lay, const CalibDims &d, double rs, const int *list, const int *off,
                        const double *kx, const double *vx, const double *kq2, const double *vq2, const double *kq4,
                        const double *vq4, double *part, cudaStream_t st) {
    const size_t smem = sizeof(CalibSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(calib_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    calib_attn_kernel<D><<<dim3(d.nqb, d.Hq, d.R), kThreads, smem, st>>>(Q, lay, d, rs, list, off, kx, vx, kq2, vq2,
                                                                         kq4, vq4, part);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

int kvq_tag_distortion_workspace_bytes(int num_layers, int num_requests, int n_q_heads, int n_kv_heads,
                                       int head_dim, int T, int num_tags, size_t *bytes) {
    if (!bytes) return kvq::host_fail(KVQ_EINVAL, "null argument");
    CalibDims d{};
    const int rc = check_dims(num_layers, num_requests, n_q_heads, n_kv_heads, head_dim, T, num_tags, d);
    if (rc != KVQ_OK) return rc;
    *bytes = calib_layout(d).total;
    return kvq::host_ok();
}

int kvq_tag_distortion_device(int num_layers, int num_requests, int n_q_heads, int n_kv_heads, int head_dim, int T,
                              const void *Q, const void *K, const void *V, const int32_t *tags, int num_tags,
                              void *workspace, size_t workspace_bytes, double *D2, double *D4, int64_t *counts,
                              void *stream) {
    CalibDims d{};
    const int rc = check_dims(num_layers, num_requests, n_q_heads, n_kv_heads, head_dim, T, num_tags, d);
    if (rc != KVQ_OK) return rc;
    if (!Q || !K || !V || !tags || !D2 || !D4 || !counts) return kvq::host_fail(KVQ_EINVAL, "null argument");
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) & 15)
        return kvq::host_fail(KVQ_EALIGN, "Q, K and V must be 16-byte aligned");
    const CalibLayout L = calib_layout(d);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) || workspace_bytes < L.total)
        return kvq::host_fail(KVQ_EUNBOUND, "workspace missing, not 256-byte aligned or smaller than "
                                            "kvq_tag_distortion_workspace_bytes");
    const int R = d.R, NT = d.ntags;
    for (long long x = 0; x < static_cast<long long>(R) * T; ++x)
        if (tags[x] < 0 || tags[x] >= NT) return kvq::host_fail(KVQ_EINVAL, "tag out of range");

    // host bookkeeping: per request the tokens ordered by (tag, position), the offsets of
    // each tag, every token's position in its tag's list and the 2-bit key groups
    std::vector<int> list(static_cast<size_t>(R) * T), off(static_cast<size_t>(R) * (NT + 1), 0),
        rank(static_cast<size_t>(R) * T), gstart(static_cast<size_t>(R) * d.maxg, 0), ngroups(R, 0);
    for (int k = 0; k < NT; ++k) counts[k] = 0;
    int maxg_used = 0;
    for (int r = 0; r < R; ++r) {
        const int32_t *tr = tags + static_cast<long long>(r) * T;
        int *o = off.data() + static_cast<size_t>(r) * (NT + 1);
        for (int t = 0; t < T; ++t) ++o[tr[t] + 1];
        for (int k = 0; k < NT; ++k) {
            counts[k] += o[k + 1];
            o[k + 1] += o[k];
        }
        std::vector<int> fill(o, o + NT);
        for (int t = 0; t < T; ++t) {
            const int k = tr[t];
            rank[static_cast<size_t>(r) * T + t] = fill[k] - o[k];
            list[static_cast<size_t>(r) * T + fill[k]++] = t;
        }
        int g = 0;
        for (int k = 0; k < NT; ++k)
            for (int s = 0; s + 32 <= o[k + 1] - o[k]; s += 32) gstart[static_cast<size_t>(r) * d.maxg + g++] = o[k] + s;
        ngroups[r] = g;
        maxg_used = std::max(maxg_used, g);
    }

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    int *d_list = reinterpret_cast<int *>(ws + L.list), *d_off = reinterpret_cast<int *>(ws + L.off);
    int *d_tags = reinterpret_cast<int *>(ws + L.tags), *d_rank = reinterpret_cast<int *>(ws + L.rank);
    int *d_gstart = reinterpret_cast<int *>(ws + L.gstart), *d_ng = reinterpret_cast<int *>(ws + L.ngroups);
    double *kx = reinterpret_cast<double *>(ws + L.kx), *vx = reinterpret_cast<double *>(ws + L.vx);
    double *kq2 = reinterpret_cast<double *>(ws + L.kq2), *vq2 = reinterpret_cast<double *>(ws + L.vq2);
    double *kq4 = reinterpret_cast<double *>(ws + L.kq4), *vq4 = reinterpret_cast<double *>(ws + L.vq4);
    double *part = reinterpret_cast<double *>(ws + L.part), *res = reinterpret_cast<double *>(ws + L.res);
    auto fail_cuda = [](cudaError_t e) {
        return kvq::host_fail(KVQ_ECUDA, cudaGetErrorString(e));
    };
    cudaError_t e = cudaSuccess;
    const std::pair<void *, const std::vector<int> *> up[] = {
        {d_list, &list}, {d_off, &off}, {d_rank, &rank}, {d_gstart, &gstart}, {d_ng, &ngroups}};
    for (const auto &u : up)
        if ((e = cudaMemcpyAsync(u.first, u.second->data(), u.second->size() * sizeof(int), cudaMemcpyHostToDevice,
                                 st)) != cudaSuccess)
            return fail_cuda(e);
    if ((e = cudaMemcpyAsync(d_tags, tags, static_cast<size_t>(R) * T * sizeof(int), cudaMemcpyHostToDevice, st)) !=
        cudaSuccess)
        return fail_cuda(e);

    const uint16_t *q16 = static_cast<const uint16_t *>(Q), *k16 = static_cast<const uint16_t *>(K),
                   *v16 = static_cast<const uint16_t *>(V);
    // a CTA writes only the (tag, b) sums of tags with a token at or before its last query
    if ((e = cudaMemsetAsync(part, 0, L.res - L.part, st)) != cudaSuccess) return fail_cuda(e);
    const double rs = 1.0 / std::sqrt(static_cast<double>(d.D));
    const long long tok_threads = static_cast<long long>(T) * (d.D / 32);
    for (int lay = 0; lay < d.NL; ++lay) {
        calib_token_kernel<<<dim3(static_cast<unsigned>((tok_threads + 255) / 256), R * d.Hkv), 256, 0, st>>>(
            k16, v16, lay, d, d_tags, d_rank, d_off, kx, vx, kq2, vq2, kq4, vq4);
        if ((e = cudaGetLastError()) != cudaSuccess) return fail_cuda(e);
        if (maxg_used > 0) {
            calib_keygroup_kernel<<<dim3(maxg_used, R * d.Hkv), d.D, 0, st>>>(k16, lay, d, d_list, d_gstart, d_ng,
                                                                               kq2);
            if ((e = cudaGetLastError()) != cudaSuccess) return fail_cuda(e);
        }
        e = d.D == 128 ? launch_attn<128>(q16, lay, d, rs, d_list, d_off, kx, vx, kq2, vq2, kq4, vq4, part, st)
                       : launch_attn<64>(q16, lay, d, rs, d_list, d_off, kx, vx, kq2, vq2, kq4, vq4, part, st);
        if (e != cudaSuccess) return fail_cuda(e);
    }
    calib_reduce_kernel<<<1, 128, 0, st>>>(part, d, res);
    if ((e = cudaGetLastError()) != cudaSuccess) return fail_cuda(e);
    std::vector<double> out(static_cast<size_t>(NT) * 2);
    if ((e = cudaMemcpyAsync(out.data(), res, out.size() * sizeof(double), cudaMemcpyDeviceToHost, st)) !=
        cudaSuccess)
        return fail_cuda(e);
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return fail_cuda(e);
    for (int k = 0; k < NT; ++k) {
        D2[k] = out[2 * k];
        D4[k] = out[2 * k + 1];
    }
    return kvq::host_ok();
}

}  // extern "C"
