// Per-tag distortion D_k(b) on the GPU ("TriAxialKV per-role mixed-precision KV
// quantization for agentic prefills", Facts: per-tag distortion, quantizer, leftover
// routing).  The definition is the host entry point's (kvq_tag_distortion): tag k's tokens
// at b bits and every other token exact, causal attention over the calibration prefill,
// output MSE per query head; max over heads, mean over requests, sum over layers.  All
// attention arithmetic is fp64 (the products on the fp64 tensor cores), so the results
// equal the host's up to the order of the sums.
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
//     Both products run on the fp64 tensor cores (mma m8n8k4).  Its 16-token tiles of
//     fp64 rows (exact and quantized) come by cp.async into two buffers, the next tile of
//     the CTA's whole sequence of passes in flight while the current one is used.
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
    double q[kQB][D + 4];                  // rows padded: 16-byte aligned, fragment loads conflict-free
    double t[2][4][kKT][D + 4];            // two tile buffers: exact k, exact v, quantized k, quantized v
    double pe[kQB][kKT + 4], pq[kQB][kKT + 4];   // exact / quantized weights exp(s - m_i)
    double mx[2][kQB], ls[2][kQB], dl[2][kQB];   // per key half: row max, sum of weights, sum of pq - pe
    double red[kThreads / 32];
    int tok[2][kKT];                       // token of each tile row (-1: none)
};

__device__ __forceinline__ void cp16(void *smem, const void *gmem) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait_prev() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// d += a b on the fp64 tensor cores: an 8 x 8 x 4 product per warp.  Lane l holds
// a = A[l/4][l%4], b = B[l%4][l/4] and d = D[l/4][2(l%4)], D[l/4][2(l%4) + 1].
__device__ __forceinline__ void dmma(double &d0, double &d1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

// Scores of query tile mt (rows 8mt..8mt+7) against key tile nt of rows k and of rows kh
// (the exact and the quantized keys, one query fragment for both), channel order in
// steps of 4: lane l gets the keys 8nt + 2(l%4) + {0, 1} of query 8mt + l/4.
template <int D, bool TWO>
__device__ __forceinline__ void score_tile(const double (*q)[D + 4], const double (*k)[D + 4],
                                           const double (*kh)[D + 4], int mt, int nt, int lane, double (&se)[2],
                                           double (&sq)[2]) {
    se[0] = se[1] = sq[0] = sq[1] = 0.0;
    const double *qa = &q[8 * mt + (lane >> 2)][lane & 3];
    const double *kb = &k[8 * nt + (lane >> 2)][lane & 3];
    const double *hb = &kh[8 * nt + (lane >> 2)][lane & 3];
#pragma unroll 8
    for (int c = 0; c < D; c += 4) {
        const double a = qa[c];
        dmma(se[0], se[1], a, kb[c]);
        if (TWO) dmma(sq[0], sq[1], a, hb[c]);
    }
}

// Where a CTA is in its sequence of 16-token tiles: pass 0 (row max over tokens 0..i_max),
// pass 1 (l and N over the same tiles), then pass 2 for every (tag with a token <= i_max,
// b): the tag's tokens in list order.
struct TilePos {
    int ph, k, bi, ti, nt;   // pass, tag, bit index (0: 2 bits, 1: 4 bits), tile, tiles in the pass
};

// CTA = (query block qb, query head hq, request r) of layer `lay`: 8 warps, both products
// on the fp64 tensor cores (mma m8n8k4).  Scores: warp w takes query tile mt = w % 4
// (8 queries) and key tile w / 4 (8 of the tile's 16 keys).  Weighted values: warp w takes
// output channels [8 NTW w, 8 NTW (w + 1)) of all 32 queries.  Tiles are fp64 rows copied
// by cp.async into two buffers: the next tile (of any pass) is in flight while the
// current one is used.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    calib_attn_kernel(const uint16_t *__restrict__ Q, int lay, CalibDims d, double rs, const int *__restrict__ list,
                      const int *__restrict__ off, const double *kx, const double *vx, const double *kq2,
                      const double *vq2, const double *kq4, const double *vq4, double *part) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    CalibSmem<D> &sm = *reinterpret_cast<CalibSmem<D> *>(smem_raw);
    constexpr int NTW = D / 64;   // 8-channel output tiles per warp
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int mt = w & 3, nt = w >> 2;            // score tile of this warp
    const int sq_row = 8 * mt + (lane >> 2);     // its query row in the block
    const int key0 = 8 * nt + 2 * (lane & 3);    // its first key in the tile
    const int qb = d.nqb - 1 - static_cast<int>(blockIdx.x);   // longest rows first
    const int hq = blockIdx.y, r = blockIdx.z, h = hq / (d.Hq / d.Hkv);
    const int i0 = qb * kQB, i = i0 + sq_row;
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
            const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                o[j] = make_double2(static_cast<double>(__uint_as_float(wd[j] << 16)),
                                    static_cast<double>(__uint_as_float(wd[j] & 0xffff0000u)));
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = make_double2(0.0, 0.0);
        }
    }

    // score side (query sq_row, keys key0, key0 + 1): row max, weight sums; value side
    // (queries 8 m + lane / 4, channels 8 (NTW w + j) + 2 (lane % 4) + {0, 1}): N, A, B
    double m = -INFINITY, lp = 0.0, dlp = 0.0;
    double N[4][NTW][2], A[4][NTW][2], B[4][NTW][2];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int j = 0; j < NTW; ++j) N[a][j][0] = N[a][j][1] = 0.0;

    // weighted values of the tile: acc (+)= P V over its 16 keys, 4 per step
    auto pv = [&](const double (*P)[kKT + 4], const double (*V)[D + 4], double (&acc)[4][NTW][2]) {
#pragma unroll
        for (int k4 = 0; k4 < kKT; k4 += 4) {
            double a[4], b[NTW];
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) a[mm] = P[8 * mm + (lane >> 2)][k4 + (lane & 3)];
#pragma unroll
            for (int j = 0; j < NTW; ++j) b[j] = V[k4 + (lane & 3)][8 * (NTW * w + j) + (lane >> 2)];
#pragma unroll
            for (int mm = 0; mm < 4; ++mm)
#pragma unroll
                for (int j = 0; j < NTW; ++j) dmma(acc[mm][j][0], acc[mm][j][1], a[mm], b[j]);
        }
    };

    for (int buf = 0;; buf ^= 1) {
        TilePos nxt = cur;
        const bool more = advance(nxt);
        if (more)
            issue(buf ^ 1, nxt);
        else
            cp_commit();   // an empty group keeps the wait below uniform
        cp_wait_prev();     // this tile's copies (the group before the newest) have landed
        __syncthreads();
        const double(*tk)[D + 4] = sm.t[buf][0];
        if (cur.ph == 0) {   // row max of s_ij = (q_i . k_j) rs over j <= i
            const int j0 = cur.ti * kKT;
            double se[2], sq[2];
            score_tile<D, false>(sm.q, tk, tk, mt, nt, lane, se, sq);
#pragma unroll
            for (int v = 0; v < 2; ++v)
                if (valid_q && j0 + key0 + v <= i) m = fmax(m, se[v] * rs);
            if (cur.ti == cur.nt - 1) {
                m = fmax(m, __shfl_xor_sync(0xffffffffu, m, 1));
                m = fmax(m, __shfl_xor_sync(0xffffffffu, m, 2));
                if ((lane & 3) == 0) sm.mx[nt][sq_row] = m;
            }
        } else if (cur.ph == 1) {   // l_i and N_i with the exact weights exp(s_ij - m_i)
            if (cur.ti == 0) m = fmax(sm.mx[0][sq_row], sm.mx[1][sq_row]);
            const int j0 = cur.ti * kKT;
            double se[2], sq[2];
            score_tile<D, false>(sm.q, tk, tk, mt, nt, lane, se, sq);
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                const double p = valid_q && j0 + key0 + v <= i ? exp(se[v] * rs - m) : 0.0;
                sm.pe[sq_row][key0 + v] = p;
                lp += p;
            }
            __syncthreads();
            pv(sm.pe, sm.t[buf][1], N);
            if (cur.ti == cur.nt - 1) {
                lp += __shfl_xor_sync(0xffffffffu, lp, 1);
                lp += __shfl_xor_sync(0xffffffffu, lp, 2);
                if ((lane & 3) == 0) sm.ls[nt][sq_row] = lp;
            }
        } else {   // the tag's tokens j <= i at b bits; A and B apart, so exact levels give 0 exactly
            if (cur.ti == 0) {
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int j = 0; j < NTW; ++j) A[a][j][0] = A[a][j][1] = B[a][j][0] = B[a][j][1] = 0.0;
                dlp = 0.0;
            }
            double se[2], sq[2];
            score_tile<D, true>(sm.q, tk, sm.t[buf][2], mt, nt, lane, se, sq);
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                const int tt = sm.tok[buf][key0 + v];
                const bool ok = valid_q && tt >= 0 && tt <= i;
                const double pe = ok ? exp(se[v] * rs - m) : 0.0, pq = ok ? exp(sq[v] * rs - m) : 0.0;
                sm.pe[sq_row][key0 + v] = pe;
                sm.pq[sq_row][key0 + v] = pq;
                dlp += pq - pe;
            }
            __syncthreads();
            pv(sm.pq, sm.t[buf][3], A);
            pv(sm.pe, sm.t[buf][1], B);
            if (cur.ti == cur.nt - 1) {   // the pass's squared output differences, summed over the CTA
                dlp += __shfl_xor_sync(0xffffffffu, dlp, 1);
                dlp += __shfl_xor_sync(0xffffffffu, dlp, 2);
                if ((lane & 3) == 0) sm.dl[nt][sq_row] = dlp;
                __syncthreads();
                double err = 0.0;
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) {
                    const int row = 8 * mm + (lane >> 2);
                    if (i0 + row >= d.T) continue;
                    const double l = sm.ls[0][row] + sm.ls[1][row];
                    const double lq = l + (sm.dl[0][row] + sm.dl[1][row]);
#pragma unroll
                    for (int j = 0; j < NTW; ++j)
#pragma unroll
                        for (int v = 0; v < 2; ++v) {
                            const double e = (N[mm][j][v] + (A[mm][j][v] - B[mm][j][v])) / lq - N[mm][j][v] / l;
                            err += e * e;
                        }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) err += __shfl_xor_sync(0xffffffffu, err, o);
                if (lane == 0) sm.red[w] = err;
                __syncthreads();
                if (tid == 0) {
                    double s = 0.0;
                    for (int x = 0; x < kThreads / 32; ++x) s += sm.red[x];
                    part[((((static_cast<long long>(lay) * d.R + r) * d.Hq + hq) * d.nqb + qb) * d.ntags + cur.k) * 2 +
                         cur.bi] = s;
                }
            }
        }
        __syncthreads();   // this buffer (and sm.pe, sm.pq, sm.red) is free again
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
    if (T > (1 << 30)) return kvq::host_fail(KVQ_EUNSUPPORTED, "T above 2^30 tokens");
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
