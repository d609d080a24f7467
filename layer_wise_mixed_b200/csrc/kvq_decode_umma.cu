// Split-KV decode attention over the packed per-layer cache on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory): a variant of decode_split_kernel
// for head_dim 128, up to 8 query heads per kv head and either key mode.
//
// The same attention as the mma.sync kernel (flash-decoding splits merged by log-sum-exp:
// "TriAxialKV per-role mixed-precision KV quantization", Facts: decode path; one static
// precision pair per layer: KVTuner summary, Approach), with both contractions issued as
// tcgen05.mma (kind::f16, fp32 accumulate) by one thread, operands staged in shared memory
// in the no-swizzle K-major layout (8-row x 16-byte core matrices):
//
//   scores, per 32-token block:  D_K [row][token] = sum_c A_K [row][c] B_K [token][c]
//     A_K rows = (part, head): q~_c s_c as an exact fp16 hi + lo pair.  Up to 4 heads: 8
//       rows read with stride-byte-offset 0, so all 128 accumulator lanes hold copies of
//       the 8 rows and each warp reads its own block's scores from its lane quarter; 5 to 8
//       heads: 16 rows (the tile's other rows read past them and are not used), whose
//       scores warp 0 reads and passes on through shared memory;
//     B_K = the block's key codes as exact fp16 integers; the zero term sum_c q~_c z_c is
//       added on the CUDA cores.
//     Per-token keys: A_K rows = (32-channel group j, head) with q~ masked to group j, one
//       tile for every block; score = sum_j (s_tj D_K [(j, head)][t] + z_tj sum_{c in j} q~_c).
//   values, per 4-block chunk:  D_V [c][n] = sum_t A_V [c][t] B_V [n][t]
//     A_V = value codes (channel x token), B_V columns n = (group j, head, part): p_t s_tj
//       as an fp16 hi/lo pair; channel c reads the 8 columns of its group j = c / 32; the
//       zero term sum_t p_t z_tj on the CUDA cores.
//   the open per-channel key group (bf16 residual rows) is scored on the CUDA cores in fp32.
//
// CTA = 4 warps for one (batch, kv head, split); the split's blocks go in chunks of 4 (one
// per warp while unpacking), the chunk's records in one shared-memory stage filled by
// cp.async.bulk (the next chunk's copies overlap the value MMAs).  Thread t of the CTA owns
// channel t of the output (the value accumulator lanes), so the running O, l, m live in
// registers; the online softmax is CTA-wide per chunk.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_quant.cuh"

namespace kvq {
namespace {

constexpr int UD = 128;              // head_dim
constexpr int UCHUNK = 4;            // blocks per chunk (one per warp)
constexpr int UTMEM_COLS = 128;      // 4 blocks x 32 score columns; the value MMA reuses columns 0-31
constexpr float kLog2eU = 1.4426950408889634f;

// byte offset of element (row, k) of a K-major fp16 tile with R rows (R a multiple of 8):
// core matrices of 8 rows x 8 elements (128 bytes), row groups 128 bytes apart, K chunks
// R * 16 bytes apart
__host__ __device__ constexpr int kmaj(int row, int k, int R) {
    return ((k >> 3) * (R >> 3) + (row >> 3)) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

// shared-memory matrix descriptor: no swizzle, version 1 (sm_100)
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46);
}

// instruction descriptor of kind::f16: fp16 A and B (K-major), fp32 accumulator, M x N
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 32 columns (this warp's lane quarter), one 32-bit column per register
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 8 columns
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// CTA-wide maxima of N values per thread (one barrier pair); red holds [4 warps][N]
template <int N>
__device__ __forceinline__ void block_maxn(const float *v, float *out, float *red, int warp, int lane) {
    float m[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        m[i] = v[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], o));
    }
    __syncthreads();
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 4) *reinterpret_cast<float4 *>(red + N * warp + i) = make_float4(m[i], m[i + 1], m[i + 2], m[i + 3]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = fmaxf(fmaxf(red[i], red[N + i]), fmaxf(red[2 * N + i], red[3 * N + i]));
}

__device__ __forceinline__ float block_sum128(float v, float *red, int warp, int lane) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    return (red[0] + red[1]) + (red[2] + red[3]);
}

// 32 lanes x 16 columns
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared memory of one CTA (dynamic, 1024-byte aligned base) for up to GM query heads per
// kv head (GM = 4 or 8) and key mode KM.
template <int GM, int KM>
struct UmmaSmem {
    // A_K rows: per-channel keys, hi and lo per head (one tile per block); per-token keys,
    // (32-channel group, head) with q masked to the group (one tile for every block)
    static constexpr int RK = KM == 0 ? 2 * GM : (UD / 32) * GM;
    static constexpr int NAK = KM == 0 ? UCHUNK : 1;
    static constexpr int NV = 8 * GM;                    // B_V columns: (group, head, part)
    static constexpr int TILE = UD * 128 * 2;            // B_K (128 tokens x 128 channels) / A_V (128 x 128)
    static constexpr int AK = RK * UD * 2;               // one A_K tile
    static constexpr int BV = NV * 128 * 2;              // B_V: NV columns x 128 tokens
    static constexpr int QS_ROW = UD + 4;                // q~ row stride (floats): heads on different banks
    static constexpr int PB_ROW = 36;                    // p row stride (floats)
    static constexpr int SC_ROW = 36;                    // score row stride (floats): conflict-free 16-byte stores
    static constexpr int off_tile = 0;
    static constexpr int off_ak = off_tile + TILE;
    static constexpr int off_bv = off_ak + NAK * AK;
    static constexpr int off_qs = off_bv + BV;                        // q~ [GM][QS_ROW] fp32
    static constexpr int off_sc = off_qs + GM * QS_ROW * 4;           // per block: scores [RK][SC_ROW] fp32
    static constexpr int off_pb = off_sc + UCHUNK * RK * SC_ROW * 4;  // per warp: p [GM][PB_ROW]
    static constexpr int off_zk = off_pb + UCHUNK * GM * PB_ROW * 4;  // per warp: key zero terms [GM] (KM = 0);
                                                                      // q~ sums [group][GM] (KM = 1)
    static constexpr int off_zv = off_zk + UCHUNK * GM * 4;           // per warp: value zero terms [4 j][GM]
    static constexpr int off_red = off_zv + UCHUNK * 4 * GM * 4;      // reductions [4 warps][GM]
    static constexpr int off_bar = off_red + 4 * GM * 4;              // copy, mma, q barriers + tmem slot
    static constexpr int off_q = off_bar + 64;                        // bf16 q rows [G][128]
    static constexpr int off_stage = ((off_q + GM * UD * 2 + 127) / 128) * 128;
    static constexpr int bytes(int rec) { return off_stage + UCHUNK * rec; }
};

template <int BK, int BV, int GM, int KM>
__global__ void __launch_bounds__(128, 1) decode_umma_kernel(const DecodeParams p) {
    pdl_enter();
    using SM = UmmaSmem<GM, KM>;
    constexpr int D = UD, NJ = D / 32, KS = D / 16;
    constexpr int RK = SM::RK, NV = SM::NV;
    constexpr int REC = unit_bytes(D, BK, BV, KM, 2);
    constexpr int KC = 4 * D * BK, KSZ = 4 * D, VC = 4 * D * BV;
    constexpr int PK = 16 / BK, PV = 16 / BV;
    constexpr int WHK = D * BK / 64, WHV = D * BV / 64;
    // GM = 4: the 8 A_K rows are read with stride-byte-offset 0, so every lane quarter
    // holds them and each warp reads its own block's scores; GM = 8: 16 rows, lanes 0-15
    // (warp 0's quarter) hold them and warp 0 passes every block's scores on
    constexpr bool ALIAS = KM == 0 && GM == 4;   // per-token keys: RK = 4 GM rows, never aliased
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int b = blockIdx.z, h = blockIdx.y, sp = blockIdx.x;
    const int G = p.G;
    const int L = p.ragged ? (p.lens_dev ? p.lens_dev[b] : p.lens[b]) : p.L;
    const int nblk = (L + 31) >> 5, rem = L & 31;
    const int tail_blk = rem ? (L >> 5) : -1;
    const int blk0 = sp * p.bps, blk1 = min(nblk, blk0 + p.bps);
    const long long unit = static_cast<long long>(b) * p.Hkv + h;

    uint8_t *tile = smem + SM::off_tile;
    uint8_t *ak = smem + SM::off_ak;
    uint8_t *bv = smem + SM::off_bv;
    float *qs = reinterpret_cast<float *>(smem + SM::off_qs);
    float *sc = reinterpret_cast<float *>(smem + SM::off_sc);
    float *pb = reinterpret_cast<float *>(smem + SM::off_pb);
    float *zk = reinterpret_cast<float *>(smem + SM::off_zk);
    float *zv = reinterpret_cast<float *>(smem + SM::off_zv);
    float *red = reinterpret_cast<float *>(smem + SM::off_red);
    uint64_t *copy_bar = reinterpret_cast<uint64_t *>(smem + SM::off_bar);
    uint64_t *mma_bar = copy_bar + 1;
    uint64_t *q_bar = copy_bar + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(copy_bar + 3);
    uint16_t *q_s = reinterpret_cast<uint16_t *>(smem + SM::off_q);
    uint8_t *stage = smem + SM::off_stage;

    auto rec_src = [&](int blk) {
        return p.rec + rec_index(p.btab, b, p.Hkv, h, p.cap_blk, blk) * static_cast<long long>(REC);
    };
    // one chunk's record copies (thread 0): blocks c0 .. c0 + 3 that exist
    auto issue_chunk = [&](int c0) {
        const int n = min(UCHUNK, blk1 - c0);
        mbar_expect_tx(copy_bar, static_cast<unsigned>(n * REC));
        for (int i = 0; i < n; ++i) bulk_g2s(stage + i * REC, rec_src(c0 + i), REC, copy_bar);
    };
    const bool has_data = blk1 > blk0;
    if (tid == 0) {
        mbar_init(copy_bar, 1);
        mbar_init(mma_bar, 1);
        mbar_init(q_bar, 1);
        fence_mbar_init();
        mbar_expect_tx(q_bar, static_cast<unsigned>(G * D * 2));
        bulk_g2s(q_s, p.q + unit * G * D, static_cast<unsigned>(G * D * 2), q_bar);
        if (has_data) issue_chunk(blk0);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(UTMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool failed = false;

    // ---- q~ per head (thread = channel), kq as in the mma.sync kernel.  Per-channel keys:
    // q~ = q log2(e)/sqrt(D) 2^kq with q~ < 2^15 and q~ s_k < 2^14 for the layer's largest
    // key scale; per-token keys: q~ = q 2^kq < 2^15 (exact in fp16), the score scale applied
    // with unscale
    if (!mbar_wait(q_bar, 0)) failed = true;
    const float smax_k = __half2float(__ushort_as_half(static_cast<unsigned short>(p.smax[0])));
    const float smax_v = __half2float(__ushort_as_half(static_cast<unsigned short>(p.smax[1])));
    const float qscale = kLog2eU * rsqrtf(static_cast<float>(D));
    float unscale[GM];
    {
        float qv[GM], aq[GM], amax[GM];
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) {
            qv[hh] = hh < G ? quant::bf16_to_f32(q_s[hh * D + tid]) * (KM == 0 ? qscale : 1.f) : 0.f;
            aq[hh] = fabsf(qv[hh]);
        }
        block_maxn<GM>(aq, amax, red, warp, lane);
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) {
            int kq = 0;
            if (amax[hh] > 0.f) {
                kq = 14 - floor_log2(amax[hh]);
                if (KM == 0 && smax_k > 0.f) kq = min(kq, 12 - floor_log2(amax[hh]) - floor_log2(smax_k));
                kq = max(-120, min(100, kq));
            }
            qv[hh] *= pow2f(kq);
            qs[hh * SM::QS_ROW + tid] = qv[hh];
            unscale[hh] = KM == 0 ? pow2f(-kq) : qscale * pow2f(-kq);
        }
        if constexpr (KM == 1) {
            // A_K rows (group j, head hh): q~ of channel tid in row (tid / 32) GM + hh, zeros
            // in the other groups' rows (fp16, exact: a bf16 value times a power of two below
            // 2^15); the groups' q~ sums for the zero terms (warp = group)
            const int j = tid >> 5;
#pragma unroll
            for (int r = 0; r < RK; ++r) {
                const int hh = r % GM;
                const float v = (r / GM == j && hh < G) ? qv[hh] : 0.f;
                *reinterpret_cast<__half *>(ak + kmaj(r, tid, RK)) = __float2half_rn(v);
            }
#pragma unroll
            for (int hh = 0; hh < GM; ++hh) {
                float sum = qv[hh];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) zk[j * GM + hh] = sum;   // qsum [group][head]
            }
        }
    }
    const int kp = smax_v > 0.f ? max(-24, min(14, 13 - floor_log2(smax_v))) : 14;
    const float pbias = static_cast<float>(kp);
    __syncthreads();

    float m_run[GM], l_acc[GM], o_acc[GM];
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) {
        m_run[hh] = -INFINITY;
        l_acc[hh] = 0.f;
        o_acc[hh] = 0.f;
    }
    constexpr uint32_t IDESC_K = umma_idesc(128, 32);
    constexpr uint32_t IDESC_V = umma_idesc(128, NV);
    unsigned copy_phase = 0, mma_phase = 0;

    for (int c0 = blk0; c0 < blk1; c0 += UCHUNK) {
        const int nb = min(UCHUNK, blk1 - c0);
        const int blk = c0 + warp;                       // this warp's block of the chunk
        const bool mine = warp < nb;
        const bool is_tail = mine && blk == tail_blk;
        const int valid = !mine ? 0 : (is_tail ? rem : 32);
        const uint8_t *R = stage + warp * REC;
        if (!mbar_wait(copy_bar, copy_phase)) failed = true;
        copy_phase ^= 1u;

        // ---- (1) key tiles of this warp's block: B_K codes; per-channel keys also A_K = q~ s
        // hi/lo and the zero term (their open group's keys are the residual rows instead)
        const bool has_codes = mine && (KM == 1 || !is_tail);
        if (has_codes) {
            uint32_t kw[2][WHK];   // this lane's code words of both halves
            load_lane_words<WHK>(R, lane, kw[0]);
            load_lane_words<WHK>(R + 2 * D * BK, lane, kw[1]);
#pragma unroll
            for (int k = 0; k < KS; ++k)
#pragma unroll
                for (int n = 0; n < 4; ++n) {   // 8-token tiles: half n >> 1, rows 8 (n & 1) + g
                    const int s0 = (2 * k + (n & 1)) * 2;
                    const uint32_t word = kw[n >> 1][s0 / PK];
                    const int tok = 32 * warp + 8 * n + g;
                    *reinterpret_cast<uint32_t *>(tile + kmaj(tok, 16 * k + 2 * t, 128)) = unpack<BK>(word, s0 % PK);
                    *reinterpret_cast<uint32_t *>(tile + kmaj(tok, 16 * k + 8 + 2 * t, 128)) =
                        unpack<BK>(word, s0 % PK + 1);
                }
        }
        if (KM == 0 && has_codes) {
            // A_K: lane = (row r = lane % RK, 8-channel chunks lane / RK + (32 / RK) i); row r:
            // head r % GM, the hi (r < GM) or lo part of q~_c s_c; one 16-byte store per chunk
            // (8 lanes fill a 128-byte core matrix).  The hi-row lanes also sum q~_c z_c.
            uint8_t *a = ak + warp * SM::AK;
            const int r = lane % RK, hh = r % GM;
            const bool hi_row = r < GM, live = hh < G;
            float zs = 0.f;
#pragma unroll
            for (int it = 0; it < 16 * RK / 32; ++it) {
                const int c8 = lane / RK + (32 / RK) * it, d0 = 8 * c8;
                // scales/zeros of channels d0 .. d0 + 7: half2 pairs 16 bytes apart
                const uint8_t *szp = R + KC + quant::chan_sz_off(d0);
                float sv[8], zv8[8], qv[8];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const __half2 s2 = *reinterpret_cast<const __half2 *>(szp + 8 * e);
                    const __half2 z2 = *reinterpret_cast<const __half2 *>(szp + 8 * e + 4);
                    sv[e] = __low2float(s2);
                    sv[e + 1] = __high2float(s2);
                    zv8[e] = __low2float(z2);
                    zv8[e + 1] = __high2float(z2);
                }
                const float4 q0 = *reinterpret_cast<const float4 *>(qs + hh * SM::QS_ROW + d0);
                const float4 q1 = *reinterpret_cast<const float4 *>(qs + hh * SM::QS_ROW + d0 + 4);
                qv[0] = q0.x; qv[1] = q0.y; qv[2] = q0.z; qv[3] = q0.w;
                qv[4] = q1.x; qv[5] = q1.y; qv[6] = q1.z; qv[7] = q1.w;
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float v0 = live ? qv[e] * sv[e] : 0.f, v1 = live ? qv[e + 1] * sv[e + 1] : 0.f;
                    const float h0 = trunc11(v0), h1 = trunc11(v1);
                    w4[e >> 1] = hi_row ? pack_h2(h0, h1) : pack_h2(v0 - h0, v1 - h1);
                    zs = fmaf(qv[e], zv8[e], fmaf(qv[e + 1], zv8[e + 1], zs));
                }
                *reinterpret_cast<uint4 *>(a + kmaj(r, d0, RK)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
#pragma unroll
            for (int o = RK; o < 32; o <<= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
            if (lane < GM) zk[warp * GM + lane] = live ? zs : 0.f;
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- (2) score MMAs: block i of the chunk into accumulator columns 32 i .. 32 i + 31
        bool any_k = false;
        for (int i = 0; i < nb; ++i) any_k |= (KM == 1 || c0 + i != tail_blk);
        if (tid == 0 && any_k) {
            for (int i = 0; i < nb; ++i) {
                if (KM == 0 && c0 + i == tail_blk) continue;
#pragma unroll
                for (int s = 0; s < KS; ++s) {
                    const uint8_t *a_tile = ak + (KM == 0 ? i * SM::AK : 0);
                    const uint64_t ad = umma_desc(smem_u32(a_tile) + s * 2 * RK * 16, RK * 16, ALIAS ? 0 : 128);
                    const uint64_t bd = umma_desc(smem_u32(tile) + 512 * i + s * 4096, 2048, 128);
                    umma_f16(tmem + 32 * i, ad, bd, IDESC_K, s > 0 ? 1u : 0u);
                }
            }
            umma_commit(mma_bar);
        }
        if (any_k) {
            if (!mbar_wait(mma_bar, mma_phase)) failed = true;
            mma_phase ^= 1u;
        }
        tc_fence_after();
        // ---- (3) scores: lane = token of this warp's block, GM heads (log2 units)
        float s4[GM];
        if constexpr (ALIAS) {
            if (mine && !is_tail) {
                float v[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * warp, v);
                if (lane < RK) {
                    float *row = sc + (warp * RK + lane) * SM::SC_ROW;
#pragma unroll
                    for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4 *>(row + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                }
                __syncwarp();
            }
        } else {
            // rows 0 .. RK - 1 sit in lanes 0 .. RK - 1: warp 0 reads every block's columns
            if (warp == 0) {
                for (int i = 0; i < nb; ++i) {
                    if (KM == 0 && c0 + i == tail_blk) continue;
                    float v[32];
                    tmem_ld32(tmem + 32 * i, v);
                    if (lane < RK) {
                        float *row = sc + (i * RK + lane) * SM::SC_ROW;
#pragma unroll
                        for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4 *>(row + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                    }
                }
            }
            __syncthreads();
        }
        if (KM == 1 && mine) {
            // per-token keys: sum over the groups of s_uj * rows (j, head) + z_uj * qsum (j, head)
            float acc[GM];
#pragma unroll
            for (int hh = 0; hh < GM; ++hh) acc[hh] = 0.f;
            if (lane < valid) {
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const uint8_t *szp = R + KC + quant::tok_sz_off(lane, j, NJ);
                    const float sk = __half2float(*reinterpret_cast<const __half *>(szp));
                    const float zk_ = __half2float(*reinterpret_cast<const __half *>(szp + 4 * NJ));
#pragma unroll
                    for (int hh = 0; hh < GM; ++hh)
                        acc[hh] = fmaf(sk, sc[(warp * RK + j * GM + hh) * SM::SC_ROW + lane],
                                       fmaf(zk_, zk[j * GM + hh], acc[hh]));
                }
            }
#pragma unroll
            for (int hh = 0; hh < GM; ++hh) s4[hh] = acc[hh] * unscale[hh];
        } else if (KM == 0 && mine && !is_tail) {
#pragma unroll
            for (int hh = 0; hh < GM; ++hh)
                s4[hh] = (sc[(warp * RK + hh) * SM::SC_ROW + lane] + sc[(warp * RK + GM + hh) * SM::SC_ROW + lane] +
                          zk[warp * GM + hh]) * unscale[hh];
        } else if (KM == 0 && is_tail) {
            // the open group's keys: bf16 residual rows, fp32 dot products
            float acc[GM];
#pragma unroll
            for (int hh = 0; hh < GM; ++hh) acc[hh] = 0.f;
            if (lane < rem) {
                const uint16_t *row = p.res + (unit * 32 + lane) * D;
                for (int c = 0; c < D; c += 2) {
                    const uint32_t w2 = *reinterpret_cast<const uint32_t *>(row + c);
                    const float k0 = __uint_as_float(w2 << 16), k1 = __uint_as_float(w2 & 0xFFFF0000u);
#pragma unroll
                    for (int hh = 0; hh < GM; ++hh)
                        acc[hh] = fmaf(qs[hh * SM::QS_ROW + c], k0, fmaf(qs[hh * SM::QS_ROW + c + 1], k1, acc[hh]));
                }
            }
#pragma unroll
            for (int hh = 0; hh < GM; ++hh) s4[hh] = acc[hh] * unscale[hh];
        }
        const bool tok_ok = lane < valid;
#pragma unroll
        for (int hh = 0; hh < GM; ++hh)
            if (!tok_ok || hh >= G) s4[hh] = -INFINITY;
        // ---- (4) online softmax over the chunk (CTA-wide per head)
        float alpha[GM], m_new[GM], cm[GM];
        block_maxn<GM>(s4, cm, red, warp, lane);
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) {
            m_new[hh] = fmaxf(m_run[hh], cm[hh]);
            alpha[hh] = (m_new[hh] == -INFINITY) ? 1.f : fast_exp2(m_run[hh] - m_new[hh]);
            m_run[hh] = m_new[hh];
        }
        float p4[GM];
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) {
            p4[hh] = tok_ok && hh < G ? fast_exp2(s4[hh] - m_new[hh] + pbias) : 0.f;
            l_acc[hh] = fmaf(l_acc[hh], alpha[hh], p4[hh]);
        }
        // ---- (5) B_V = p s_V hi/lo per (group, head): lane = column n = (group j, head, part)
        // (GM = 8: two columns per lane), the warp's 4 token octets, one 16-byte store each
        // (8 lanes fill a core matrix); the hi lanes also sum the value zero term p_t z_tj
#pragma unroll
        for (int hh = 0; hh < GM; ++hh) pb[(warp * GM + hh) * SM::PB_ROW + lane] = p4[hh];
        __syncwarp();
#pragma unroll
        for (int nn = 0; nn < NV / 32; ++nn) {
            const int n = lane + 32 * nn, j = n / (2 * GM), hh = (n >> 1) % GM, part = n & 1;
            float zsum = 0.f;
#pragma unroll
            for (int o = 0; o < 4; ++o) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const int u = 8 * o + e;   // token pair (u, u + 1) of the block
                    float v0 = 0.f, v1 = 0.f;
                    if (u < valid) {
                        const uint8_t *szp = R + KC + KSZ + VC + quant::tok_sz_off(u, j, NJ);
                        const __half2 s2 = *reinterpret_cast<const __half2 *>(szp);
                        const __half2 z2 = *reinterpret_cast<const __half2 *>(szp + 4 * NJ);
                        const float p0 = pb[(warp * GM + hh) * SM::PB_ROW + u];
                        const float p1 = u + 1 < valid ? pb[(warp * GM + hh) * SM::PB_ROW + u + 1] : 0.f;
                        v0 = p0 * __low2float(s2);
                        v1 = u + 1 < valid ? p1 * __high2float(s2) : 0.f;
                        zsum = fmaf(p0, __low2float(z2), zsum);
                        if (u + 1 < valid) zsum = fmaf(p1, __high2float(z2), zsum);
                    }
                    const float h0 = trunc11(v0), h1 = trunc11(v1);
                    w4[e >> 1] = part == 0 ? pack_h2(h0, h1) : pack_h2(v0 - h0, v1 - h1);
                }
                *reinterpret_cast<uint4 *>(bv + kmaj(n, 32 * warp + 8 * o, NV)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            if (part == 0) zv[warp * 4 * GM + j * GM + hh] = zsum;
        }
        // ---- (6) A_V = value codes (channel x token) of this warp's block (zeros for none)
        if (mine) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                uint32_t vw[WHV];
                load_lane_words<WHV>(R + KC + KSZ + kk * 2 * D * BV, lane, vw);
#pragma unroll
                for (int m = 0; m < KS; ++m)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {   // slot 4m + r: channel 16m + g + 8 (r & 1), tokens 8 (r >> 1) + 2t, +1
                        const int s = 4 * m + r;
                        const int c = 16 * m + g + 8 * (r & 1);
                        const int tokc = 32 * warp + 16 * kk + 8 * (r >> 1) + 2 * t;
                        *reinterpret_cast<uint32_t *>(tile + kmaj(c, tokc, 128)) = unpack<BV>(vw[s / PV], s % PV);
                    }
            }
        } else {
            for (int i = lane; i < 128 * 32 / 2; i += 32) {   // the warp's 32 token columns of every channel
                const int c = i / 16, tk = 2 * (i % 16);
                *reinterpret_cast<uint32_t *>(tile + kmaj(c, 32 * warp + tk, 128)) = 0u;
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();   // the stage, the score columns and the tiles are free / complete
        tc_fence_after();
        if (tid == 0) {
            if (c0 + UCHUNK < blk1) issue_chunk(c0 + UCHUNK);
#pragma unroll
            for (int s = 0; s < 8; ++s) {   // K = 128 tokens
                const uint64_t ad = umma_desc(smem_u32(tile) + s * 4096, 2048, 128);
                const uint64_t bd = umma_desc(smem_u32(bv) + s * 2 * NV * 16, NV * 16, 128);
                umma_f16(tmem, ad, bd, IDESC_V, s > 0 ? 1u : 0u);
            }
            umma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mma_phase)) failed = true;
        mma_phase ^= 1u;
        tc_fence_after();
        // ---- (7) channel tid = 32 warp + lane of group j = warp: its 2 GM columns
        {
            float v[2 * GM];
            if constexpr (GM == 4) tmem_ld8(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 2 * GM * warp, v);
            else tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 2 * GM * warp, v);
#pragma unroll
            for (int hh = 0; hh < GM; ++hh) {
                const float z = (zv[0 * 4 * GM + warp * GM + hh] + zv[1 * 4 * GM + warp * GM + hh]) +
                                (zv[2 * 4 * GM + warp * GM + hh] + zv[3 * 4 * GM + warp * GM + hh]);
                o_acc[hh] = fmaf(o_acc[hh], alpha[hh], v[2 * hh] + v[2 * hh + 1] + z);
            }
        }
        tc_fence_before();
        __syncthreads();   // score columns and zero terms read before the next chunk reuses them
        tc_fence_after();
    }

    // ---- epilogue: l over the CTA, output or split partials (thread = channel)
    float l_tot[GM];
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) l_tot[hh] = block_sum128(l_acc[hh], red, warp, lane);
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) {
        if (hh >= G) continue;
        const long long row = unit * G + hh;
        if (p.S == 1) {
            const float o = o_acc[hh] / l_tot[hh];
            if (p.out_fp32) reinterpret_cast<float *>(p.out)[row * D + tid] = o;
            else reinterpret_cast<__nv_bfloat16 *>(p.out)[row * D + tid] = __float2bfloat16_rn(o);
        } else {
            p.part_acc[(row * p.sstride + sp) * D + tid] = o_acc[hh];
            if (tid == 0) {
                p.part_ml[(row * p.sstride + sp) * 2] = has_data ? m_run[hh] - pbias : -INFINITY;
                p.part_ml[(row * p.sstride + sp) * 2 + 1] = l_tot[hh];
            }
        }
    }
    if (failed && lane == 0) atomicOr(p.status, kStatusWaitExpired);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(UTMEM_COLS));
}

using UmmaFn = void (*)(const DecodeParams);

template <int GM, int KM>
UmmaFn pick_umma_g(int bk, int bv) {
#define KVQ_UCASE(BKv, BVv) \
    if (bk == BKv && bv == BVv) return decode_umma_kernel<BKv, BVv, GM, KM>;
    KVQ_UCASE(2, 2) KVQ_UCASE(2, 4) KVQ_UCASE(2, 8)
    KVQ_UCASE(4, 2) KVQ_UCASE(4, 4) KVQ_UCASE(4, 8)
    KVQ_UCASE(8, 2) KVQ_UCASE(8, 4) KVQ_UCASE(8, 8)
#undef KVQ_UCASE
    return nullptr;
}

UmmaFn pick_umma(int bk, int bv, int G, int kmode) {
    if (G < 1 || G > 8 || (kmode != 0 && kmode != 1)) return nullptr;
    if (kmode == 0) return G <= 4 ? pick_umma_g<4, 0>(bk, bv) : pick_umma_g<8, 0>(bk, bv);
    return G <= 4 ? pick_umma_g<4, 1>(bk, bv) : pick_umma_g<8, 1>(bk, bv);
}

std::mutex g_umma_mu;
const void *g_umma_set[36] = {};
size_t g_umma_smem[36] = {};

}  // namespace

size_t decode_umma_smem_bytes(int bk, int bv, int G, int kmode) {
    const int rec = unit_bytes(UD, bk, bv, kmode, 2);
    if (kmode == 0) return static_cast<size_t>(G <= 4 ? UmmaSmem<4, 0>::bytes(rec) : UmmaSmem<8, 0>::bytes(rec));
    return static_cast<size_t>(G <= 4 ? UmmaSmem<4, 1>::bytes(rec) : UmmaSmem<8, 1>::bytes(rec));
}

cudaError_t decode_umma_occupancy(int bk, int bv, int G, int kmode, int *ctas_per_sm) {
    UmmaFn fn = pick_umma(bk, bv, G, kmode);
    if (!fn) return cudaErrorInvalidValue;
    const size_t smem = decode_umma_smem_bytes(bk, bv, G, kmode);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, fn, 128, smem);
}

cudaError_t launch_decode_umma(const DecodeParams &p, int bk, int bv, int kmode, cudaStream_t st) {
    UmmaFn fn = pick_umma(bk, bv, p.G, kmode);
    if (!fn) return cudaErrorInvalidValue;
    const size_t smem = decode_umma_smem_bytes(bk, bv, p.G, kmode);
    {
        std::lock_guard<std::mutex> lk(g_umma_mu);
        int slot = -1;
        for (int k = 0; k < 36; ++k)
            if (g_umma_set[k] == reinterpret_cast<const void *>(fn) || g_umma_set[k] == nullptr) {
                slot = k;
                break;
            }
        if (slot < 0) return cudaErrorInvalidValue;
        if (g_umma_set[slot] == nullptr || g_umma_smem[slot] < smem) {
            cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
            if (e != cudaSuccess) return e;
            g_umma_set[slot] = reinterpret_cast<const void *>(fn);
            g_umma_smem[slot] = smem;
        }
    }
    dim3 grid(p.S, p.Hkv, p.B);
    cudaError_t e = launch_pdl(fn, grid, dim3(128), smem, st, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace kvq
