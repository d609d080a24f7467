// Internal declarations shared by the host library and the CUDA kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace kvq {

// Programmatic dependent launch.  Every kernel of this library is launched with
// launch_pdl: it may be scheduled while the previous kernel of the stream is still
// running.  pdl_enter() first waits until the previous kernel has completed and its
// memory is visible (griddepcontrol.wait), then lets the next kernel's CTAs launch
// (griddepcontrol.launch_dependents).  Every global-memory access comes after it, so
// stream order semantics are unchanged and only launch latency and prologues overlap --
// with one exception: a decode launch whose host-side plan marks it `early` copies its
// first cache blocks before pdl_enter().  That is safe because of the order above: when
// a kernel of this library starts, the kernel before it in the stream has passed its own
// wait, so every kernel two or more launches back has completed.  The merge kernel alone
// lets its dependents launch before it waits; it always follows a decode launch, so a
// kernel may overlap at most the two launches before it, and the host marks a decode
// launch early only if neither of those writes the blocks it reads.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_enter() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

constexpr int kGroup = 32;          // quantization group (tokens or channels)

#ifdef __CUDACC__
// Index of the record of block blk of (request b, kv head h) in a layer's record area:
// the unit's slab of cap_blk records, or (block pools, btab != null) the pool block that
// the table btab [B][cap_blk] assigns to that block of the request, one record per kv head.
__host__ __device__ __forceinline__ long long rec_index(const int *btab, int b, int Hkv, int h, int cap_blk, int blk) {
    return btab ? static_cast<long long>(btab[static_cast<long long>(b) * cap_blk + blk]) * Hkv + h
                : (static_cast<long long>(b) * Hkv + h) * cap_blk + blk;
}
#endif
constexpr int kMaxSplits = 64;      // partial slots per (batch, query head)
constexpr int kMaxRagged = 64;      // requests whose per-request lengths travel in the kernel
                                    // parameters; larger batches use a device table
constexpr int kDecodeWarps = 4;     // warps per decode CTA

// Device status word bits (written with atomicOr, read by kvq_device_status).
constexpr unsigned kStatusWaitExpired = 1u;   // a bounded mbarrier wait gave up
// Wall-time limit of one bounded wait inside a kernel (nanoseconds of the GPU's global
// timer): 100 ms, far above any copy's latency, far below what would hold a GPU.
constexpr unsigned long long kWaitLimitNs = 100ull * 1000 * 1000;

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
    const uint16_t *K, *V;      // bf16 [B][Hkv][n][D] (ragged: n = the largest count, request b
                                // uses its first n_r[b] tokens)
    unsigned *smax;             // {max key scale, max value scale} (fp16 bits) at the new length
    const unsigned *smax_prev;  // the same at the old length (other parity slot), or smax
    uint8_t *rec;               // layer records [B][Hkv][cap][rec_bytes]
    uint16_t *res;              // residual [B][Hkv][32][D] bf16 (per-channel keys)
    int B, Hkv, D, bk, bv, kmode;
    int L_old, n, cap_blk;
    long long rec_bytes, kc, ks, vc;
    int hb0, nhb;               // first touched 16-token half-block, count per unit
    int g0, ng;                 // first completed key group, count per unit
    int nV, nK;                 // CTA counts of the two roles
    // per-request lengths (ragged != 0): request b appends n_r[b] tokens at L_old_r[b];
    // nhb and ng are then the largest counts over the requests (grid sizing) and each CTA
    // derives its request's own range, idling when it has none.  Batches of more than
    // kMaxRagged requests read them from the device table ragged_dev instead: [B] L_old,
    // then [B] n (written on the stream by launch_set_table just before).
    int ragged;
    int L_old_r[kMaxRagged], n_r[kMaxRagged];
    const int *ragged_dev;
    const int *btab;            // block pools: [B][cap_blk] pool block of each block (rec is the pool)
};

struct DecodeParams {
    const uint8_t *rec;         // layer records
    const uint16_t *res;        // residual (per-channel keys) or null
    const uint16_t *q;          // bf16 [B][Hq][D]
    const unsigned *smax;       // this layer's {max key scale, max value scale} (fp16 bits)
    void *out;                  // [B][Hq][D] bf16 or fp32
    float *part_acc;            // [B][Hq][sstride][D]
    float *part_ml;             // [B][Hq][sstride][2]  (m in log2 units, l)
    int sstride;                // partial slots per (batch, query head): kMaxSplits in the
                                // workspace, the launch's split count in the built-in scratch
    unsigned *arrive;           // [B][Hkv] split arrival counters (zero between launches), or null:
                                // split partials merged by merge_kernel
    unsigned *status;
    int B, Hkv, G, L, cap_blk, S, bps, out_fp32;
    int nstage, nextra;         // stages per warp; one more for warps 0 .. nextra - 1
    // per-request lengths (ragged != 0): request b has lens[b] tokens (L above is the
    // largest, which sets the split partition); batches of more than kMaxRagged requests
    // read them from the device table lens_dev [B] (written by launch_set_table)
    int ragged;
    int lens[kMaxRagged];
    const int *lens_dev;
    long long rec_bytes;
    // Fused one-token append (kvq_append_decode), null otherwise: the new token's K and V
    // rows (bf16 [B][Hkv][D]), now token L - 1; writable records and residual; the
    // scale-maximum slot of length L (smax above is the slot of length L - 1).
    const uint16_t *k_new, *v_new;
    uint8_t *rec_w;
    uint16_t *res_w;
    unsigned *smax_out;
    // early != 0: the first stages' block copies (and the L2 prefetch of the residual
    // rows) are issued before pdl_enter(); the host sets it only when the previous launch
    // in the stream writes none of this layer's records or residual (see pdl_enter)
    int early;
    const int *btab;            // block pools: [B][cap_blk] pool block of each block (rec is the pool)
};


// ---------------------------------------------------------------- paged INT2/INT4
constexpr int kMaxPagedBatch = 64;   // requests per paged plan (kernel-parameter tables)

struct PagedCounts {
    int n2g;    // complete INT2 groups (32 tokens each)
    int n4;     // tokens in the INT4 main pages
    int np;     // INT2 tokens of the open group (held as INT4 in the pending pages)
    int pad;
};

struct PagedDecodeParams {
    const uint8_t *pool2;       // [Hkv][n2_cap records] of 32-token INT2 records
    const uint8_t *pool4;       // [Hkv][n4_cap pages] of 16-token INT4 pages (pending pages last)
    long long n2_cap, n4_cap;
    const int *table;           // [B][P_cap]: INT2 first pages from the front, INT4 pages from the back
    int P_cap, pend_base;
    PagedCounts cnt[kMaxPagedBatch];
    const uint16_t *q;
    const unsigned *smax;
    void *out;
    float *part_acc, *part_ml;
    int sstride;                // as in DecodeParams
    unsigned *arrive;           // as in DecodeParams
    unsigned *status;
    int B, Hkv, G, S2, S4, out_fp32, nstage;
};

struct PagedReq {               // one request's append plan
    int n2g_old, n4_old, np_old;
    int k2, k4;                 // new INT2 / INT4 tokens in this call
    int ng;                     // INT2 groups completed by this call
    int base2;                  // first new INT2 record id
    int base4;                  // first new INT4 main page id
    int last4;                  // page id of the partly filled INT4 main page (-1 if none)
    int c4, c2;                 // CTAs of this request: INT4 main pages touched, INT2 work CTAs
};

struct PagedAppendParams {
    const uint16_t *K, *V;      // bf16 [B][Hkv][n][D]
    const uint8_t *tags;        // device [B][n]: 2 or 4
    const int *inv2, *inv4;     // [B][n_max]: input index of the r-th new INT2 / INT4 token (n > 1)
    int inv_stride;
    uint8_t *pool2, *pool4;
    long long n2_cap, n4_cap;
    int *table;
    int P_cap, pend_base;
    uint16_t *staging;          // [B][Hkv][2][32][D] bf16 originals of the open INT2 group (K, V)
    unsigned *smax;
    int B, Hkv, D, n;
    int cta4_off[kMaxPagedBatch + 1];   // prefix offsets of the INT4-page CTAs per request
    int cta2_off[kMaxPagedBatch + 1];   // prefix offsets of the INT2 CTAs per request
    PagedReq req[kMaxPagedBatch];
};

struct MergeParams {
    const float *part_acc;
    const float *part_ml;
    void *out;
    int B, Hq, D, S, out_fp32;
    int sstride;                // partial slots per (batch, query head)
};

// Split counts from which the decode launch merges its own partials (the last CTA of a
// (batch, kv head) to finish); below, merge_kernel follows.  Measured on one B200: two or
// three splits are faster with the separate launch (every CTA's arrival costs a global
// round trip at its exit), nine (the paged 32K-context workload) with the in-launch merge.
constexpr int kInLaunchMergeSplits = 4;

// Set the thread's kvq_last_error message and return code / clear it and return KVQ_OK
// (for entry points outside kvq_host.cu).
int host_fail(int code, const char *msg);
int host_ok();

cudaError_t launch_append(const AppendParams &p, cudaStream_t st);
// Write n host integers into the device table dst on stream st, as kernel launches that
// carry the values in their parameters (1000 per launch): the values are captured by
// value into CUDA graphs, and each launch writes only after the preceding kernel of the
// stream has completed (programmatic dependent launch waits first).
cudaError_t launch_set_table(int *dst, const int *vals, int n, cudaStream_t st);
// The same for n scattered entries: dst[idx[i]] = vals[i] (500 per launch).
cudaError_t launch_scatter_table(int *dst, const int *idx, const int *vals, int n, cudaStream_t st);


// Returns cudaErrorInvalidValue if no kernel exists for the combination.
cudaError_t launch_decode(const DecodeParams &p, int D, int bk, int bv, int kmode,
                          cudaStream_t st, int *ctas_per_sm_out);
cudaError_t decode_occupancy(int D, int bk, int bv, int kmode, int G, long long rec_bytes,
                             int nstage, int nextra, int *ctas_per_sm);
cudaError_t launch_merge(const MergeParams &p, cudaStream_t st);
cudaError_t launch_decode_paged(const PagedDecodeParams &p, cudaStream_t st);
// tcgen05 variant of the per-layer decode (head_dim 128, G <= 8, either key mode,
// decode-only; kvq_decode_umma.cu): the kernel's dynamic shared memory, CTAs per SM, launch
size_t decode_umma_smem_bytes(int bk, int bv, int G, int kmode);
cudaError_t decode_umma_occupancy(int bk, int bv, int G, int kmode, int *ctas_per_sm);
cudaError_t launch_decode_umma(const DecodeParams &p, int bk, int bv, int kmode, cudaStream_t st);
cudaError_t decode_paged_occupancy(int nstage, int *ctas_per_sm);
int decode_paged_stages();
size_t decode_paged_smem_bytes(int nstage);
cudaError_t launch_paged_scan(const uint8_t *tags, int B, int n, int *inv2, int *inv4, int inv_stride,
                              cudaStream_t st);
cudaError_t launch_paged_append(const PagedAppendParams &p, int grid, cudaStream_t st);
int paged_rec2_bytes(int D);
int paged_page4_bytes(int D);
int decode_stages(long long rec_bytes, int D, int G);
size_t decode_smem_bytes(long long rec_bytes, int nstage, int nextra, int D, int G);

}  // namespace kvq
