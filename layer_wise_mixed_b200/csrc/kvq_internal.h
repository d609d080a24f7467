// Internal declarations shared by the host library and the CUDA kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace kvq {

constexpr int kGroup = 32;          // quantization group (tokens or channels)
constexpr int kMaxSplits = 64;      // partial slots per (batch, query head)
constexpr int kDecodeWarps = 4;     // warps per decode CTA

// Device status word bits (written with atomicOr, read by kvq_device_status).
constexpr unsigned kStatusWaitExpired = 1u;   // a bounded mbarrier wait gave up

// Per-layer geometry and precision, resolved by the host.
struct LayerGeom {
    int bk, bv, kmode;          // bits, key mode (0 per-channel, 1 per-token)
    long long rec_bytes;        // bytes of one 32-token block record
    long long kc, ks, vc, vs;   // sizes of the four record areas
    long long unit_bytes;       // record bytes of one (b, h) unit (capacity blocks)
    long long rec_off;          // workspace offset of the layer's records
    long long res_off;          // workspace offset of the residual (-1 if none)
};

struct AppendParams {
    const uint16_t *K, *V;      // bf16 [B][Hkv][n][D]
    unsigned *smax;             // this layer's {max key scale, max value scale} (fp16 bits)
    uint8_t *rec;               // layer records [B][Hkv][cap][rec_bytes]
    uint16_t *res;              // residual [B][Hkv][32][D] bf16 (per-channel keys)
    int B, Hkv, D, bk, bv, kmode;
    int L_old, n, cap_blk;
    long long rec_bytes, kc, ks, vc;
    int hb0, nhb;               // first touched 16-token half-block, count per unit
    int g0, ng;                 // first completed key group, count per unit
    int nV, nK;                 // CTA counts of the two roles
};

struct DecodeParams {
    const uint8_t *rec;         // layer records
    const uint16_t *res;        // residual (per-channel keys) or null
    const uint16_t *q;          // bf16 [B][Hq][D]
    const unsigned *smax;       // this layer's {max key scale, max value scale} (fp16 bits)
    void *out;                  // [B][Hq][D] bf16 or fp32
    float *part_acc;            // [B][Hq][kMaxSplits][D]
    float *part_ml;             // [B][Hq][kMaxSplits][2]  (m in log2 units, l)
    unsigned *status;
    int B, Hkv, G, L, cap_blk, S, bps, out_fp32, nstage;
    long long rec_bytes;
};

struct MergeParams {
    const float *part_acc;
    const float *part_ml;
    void *out;
    int B, Hq, D, S, out_fp32;
};

cudaError_t launch_append(const AppendParams &p, cudaStream_t st);
// Returns cudaErrorInvalidValue if no kernel exists for the combination.
cudaError_t launch_decode(const DecodeParams &p, int D, int bk, int bv, int kmode,
                          cudaStream_t st, int *ctas_per_sm_out);
cudaError_t decode_occupancy(int D, int bk, int bv, int kmode, int G, long long rec_bytes,
                             int nstage, int *ctas_per_sm);
cudaError_t launch_merge(const MergeParams &p, cudaStream_t st);
int decode_stages(long long rec_bytes, int D, int G);
size_t decode_smem_bytes(long long rec_bytes, int nstage, int D, int G);

}  // namespace kvq
