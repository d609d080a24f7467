/*
 * kvq.h -- C ABI of the layer-wise mixed-precision KV-cache library for B200 (sm_100a).
 *
 * What the library computes (cited by page title and section):
 *  - A static per-layer key/value precision pair {bk, bv} (e.g. K8V4, K4V2), chosen
 *    offline and applied at inference with no online decision
 *    ("KVTuner: Sensitivity-Aware Layer-Wise Mixed-Precision KV Cache Quantization",
 *    atlas.scime.ai summary: Approach; "Mixed-precision KV-cache quantization
 *    per-layer sensitivity", Facts).
 *  - Asymmetric groupwise quantization with group size 32: keys per channel (KIVI
 *    style, groups of 32 consecutive tokens of one channel) or per token, values per
 *    token (groups of 32 consecutive channels) ("TriAxialKV per-role mixed-precision
 *    KV quantization", Facts: quantizer; per-layer sensitivity Facts: per-channel
 *    asymmetric keys).  For a group x_0..x_31 and b bits:
 *        s = fp16_rne(fp32((max - min) / (2^b - 1))), z = fp16_rne(min),
 *        code_i = clamp(rne(fp32((x_i - float(z)) / float(s))), 0, 2^b - 1)  (0 if s = 0)
 *    every step a single correctly rounded binary32 operation (no FMA contraction);
 *    dequant x^ = code * s + z.
 *  - Keys in per-channel mode: the newest L mod 32 tokens that do not fill a group
 *    stay unquantized in a bf16 residual (TriAxialKV Facts mention KIVI's
 *    full-precision residual buffer).
 *  - Single-token decode attention over the packed cache, dequantizing in
 *    registers, split over the sequence into flash-decoding partials merged by
 *    log-sum-exp (TriAxialKV Facts: bitwidth-homogeneous splits merged by online
 *    log-sum-exp).  out[b, hq] = sum_t softmax_t(q . k^_t / sqrt(D)) v^_t over all L
 *    cached tokens; query head hq uses kv head hq / G, G = n_q_heads / n_kv_heads.
 *
 * Storage format v2 (the pages fix none; chosen so that each decoder thread's tensor
 * core operand fragments are contiguous; v1, whose scales and zeros were in plain index
 * order, is not readable as v2).  Per layer, per (batch b, kv head h):
 * capacity ceil(max_ctx/32) block records of 32 tokens, then (per-channel keys) a
 * residual of 32 x D bf16.  Record of block beta, D = head_dim, nj = D/32:
 *     [K codes 4*D*bk B][K s/z 4*D B][V codes 4*D*bv B][V s/z 4*D B]
 *   Scales and zeros are fp16, at byte offsets inside their s/z area:
 *     per-channel K, channel d: k=d/16, e=d%16, t=(e%8)/2, r=e/8, hb=e%2:
 *       scale at 16*(4k+t) + 8r + 2hb, zero at +4;
 *     per-token K and V, token u of the block, group j=d/32:
 *       scale at 8*nj*(u/2) + 4j + 2*(u%2), zero at +4*nj.
 *   Code areas = two 16-token halves of 2*D*b bytes; token u in half u/16; in the half
 *   each code has a lane (0..31) and a slot:
 *     keys:   i=(u%16)/8, gk=u%8, k=d/16, e=d%16, t=(e%8)/2, r=e/8, hb=e%2,
 *             lane=4*gk+t, slot=(2k+i)*2+r
 *     values: e=u%16, t=(e%8)/2, ch=e/8, hb=e%2, m=d/16, rho=d%16, g=rho%8, rh=rho/8,
 *             lane=4*g+t, slot=4m+2ch+rh
 *   A lane has Wh = D*b/64 little-endian 32-bit words per half, F = 32/b fields of b
 *   bits each (LSB first), P = F/2 slots per word: the code sits in lane word
 *   slot/P, field slot%P + hb*P.  Lane words are stored in chunks of c = min(4, Wh):
 *   word index in half = ((w/c)*32 + lane)*c + w%c.
 *
 * Conventions for every entry point:
 *  - Return value: a kvq_status (0 = success).  Arguments are checked on the host
 *    before any launch; on failure nothing is launched and kvq_last_error() returns
 *    a message (thread-local, valid until the next call on that thread).
 *  - Device pointers are plain CUDA global-memory pointers owned by the caller; the
 *    library never allocates device memory.  `stream` is a cudaStream_t (NULL = the
 *    legacy default stream); calls that take one are asynchronous on it.
 *  - K/V/q/out pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *  - Sequences of a plan start at length 0 and stay equal under kvq_append and
 *    kvq_append_decode; kvq_append_ragged gives them their own lengths (per-layer
 *    plans), and the library then tracks one length per (layer, sequence).  A handle
 *    is not thread-safe: serialize calls on one handle.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVQ_OK = 0,
    KVQ_EINVAL = -1,        /* bad argument (null pointer, layer index, sizes)   */
    KVQ_EUNSUPPORTED = -2,  /* valid but not supported by this build (e.g. D)    */
    KVQ_ECAPACITY = -3,     /* append would exceed max_ctx / a page pool         */
    KVQ_EUNBOUND = -4,      /* no workspace bound, or workspace too small        */
    KVQ_EALIGN = -5,        /* pointer alignment                                 */
    KVQ_ECUDA = -6,         /* a CUDA runtime call or launch failed              */
    KVQ_EDEVICE = -7        /* a kernel reported an error through the status word */
} kvq_status;

typedef enum { KVQ_PER_CHANNEL = 0, KVQ_PER_TOKEN = 1 } kvq_mode;

/* One layer's precision pair.  bk, bv in {2, 4, 8}; vmode must be KVQ_PER_TOKEN. */
typedef struct {
    int bk, bv;
    int kmode;   /* kvq_mode for keys   */
    int vmode;   /* kvq_mode for values */
} kvq_layer_cfg;

typedef struct {
    int num_layers;
    int batch;
    int n_kv_heads;
    int n_q_heads;      /* multiple of n_kv_heads; G = n_q_heads / n_kv_heads <= 8 */
    int head_dim;       /* 64 or 128 */
    int group;          /* must be 32 */
    int max_ctx;        /* token capacity per sequence and layer, at most 2^30 */
    const kvq_layer_cfg *layers;   /* num_layers entries, copied by kvq_plan */
    int paged;          /* 0: per-layer maps (this header's format); 1: INT2/INT4 paged */
    int page_tokens;    /* paged: 16 */
    float avg_bits;     /* paged: expected mean bits of the tag mask (sizes the pools) */
    int pool_blocks;    /* per-layer plans: 0 = every sequence reserves max_ctx tokens of every
                         * layer (a slab of ceil(max_ctx/32) records per (sequence, kv head));
                         * > 0 = block pools: each layer's 32-token records come from a pool of
                         * pool_blocks blocks (one record per kv head each), assigned to a
                         * sequence's blocks through a block table as it grows and returned by
                         * kvq_truncate / kvq_reset_sequences, so sequences of very different
                         * lengths share the memory; a sequence still holds at most max_ctx
                         * tokens.  Ignored by paged plans. */
} kvq_plan_desc;


typedef struct kvq_handle kvq_handle;

/* Validate a plan and create a host handle (host memory only). */
KVQ_API int kvq_plan(const kvq_plan_desc *desc, kvq_handle **out);

/* Device workspace size the plan needs: all layers' cache regions (slabs, or block
 * pools and block tables), the per-layer length tables, the split partials, split
 * arrival counters, the scale maxima and a status word. */
KVQ_API int kvq_workspace_bytes(const kvq_handle *h, size_t *bytes);

/* Bind caller-owned device memory (>= kvq_workspace_bytes, 256-byte aligned) and
 * reset every layer to length 0.  No device work is issued. */
KVQ_API int kvq_bind(kvq_handle *h, void *dev_ptr, size_t bytes);

/* Append n_new tokens to every sequence of `layer`: K, V are bf16 [B][Hkv][n_new][D]
 * (device).  Quantizes values per token, keys per channel (completing 32-token groups
 * from residual + new tokens; the rest goes to the residual) or per token.  One kernel
 * launch.  n_new >= 1; returns KVQ_ECAPACITY beyond max_ctx (for any sequence). */
KVQ_API int kvq_append(kvq_handle *h, int layer, const void *K, const void *V, int n_new, void *stream);

/* Append n_new[b] tokens to sequence b of `layer` (0 <= n_new[b] <= n_max; n_new is a
 * host array of batch entries): K, V bf16 [B][Hkv][n_max][D] (device), request b's
 * tokens in its first n_new[b] slots.  Sequences may then differ in length (ragged
 * batches); every other entry point works per request from then on: decode attends
 * over each sequence's own tokens, kvq_append_decode appends one token to each,
 * kvq_export_layer exports each unit at its own length, kvq_truncate cuts every
 * sequence to the same length.  Any batch size: up to 64 requests the per-request
 * lengths travel in the kernels' parameters, above that in a per-layer [2][B] int32
 * table in the workspace, written on `stream` just before the launch that reads it.
 * Errors as kvq_append, plus KVQ_EINVAL for a count outside [0, n_max]. */
KVQ_API int kvq_append_ragged(kvq_handle *h, int layer, const void *K, const void *V, const int32_t *n_new,
                              int n_max, void *stream);

/* Paged plans (desc.paged = 1; head_dim 128, G in {1, 2, 4}, batch <= 64): append n_new
 * tokens per request with their tags, 2 (INT2) or 4 (INT4), given twice: host_tags
 * [B][n_new] for the host-side page planning, dev_tags (same bytes, device) for the
 * kernels; the caller keeps them equal.  INT2-tagged tokens, in arrival order, form
 * groups of 32 (keys per channel 2-bit, values per token 2-bit) in the INT2 pool; INT4
 * tokens go to 16-token INT4 pages (keys and values per token 4-bit); INT2 tokens whose
 * group is still open are held the INT4 way in two pending pages per request (with
 * their bf16 originals) until the group completes ("TriAxialKV per-role
 * mixed-precision KV quantization", Facts: quantizer, leftover routing, page pools).
 * The INT2 and INT4 pools of each (layer, kv head) share one region split at an offset
 * from avg_bits; KVQ_ECAPACITY when a pool or a page table would overflow (checked
 * before any launch).  A multi-token call launches a tag scan first.  The per-layer bit
 * map is not used by paged plans (layers may be NULL). */
KVQ_API int kvq_append_tagged(kvq_handle *h, int layer, const void *K, const void *V, int n_new,
                              const uint8_t *host_tags, const uint8_t *dev_tags, void *stream);

/* Decode attention of one query token per sequence over all L tokens of `layer`:
 * q bf16 [B][Hq][D] (device); out [B][Hq][D] (device) bf16, or fp32 if out_fp32.
 * One kernel launch.  A sequence split in two or three parts adds a log-sum-exp merge
 * launch; from four splits the last CTA of each (batch, kv head) to finish merges the
 * partials inside the decode launch.  Requires L >= 1. */
KVQ_API int kvq_decode_attn(kvq_handle *h, int layer, const void *q, void *out, int out_fp32,
                    void *stream);

/* One decode step in one launch: append one token (K, V bf16 [B][Hkv][1][D], device)
 * to `layer` and then run kvq_decode_attn with q over all L + 1 tokens; same results
 * and errors as kvq_append(..., n_new = 1, ...) followed by kvq_decode_attn.  The CTA
 * that decodes a sequence's last block first quantizes and packs the new token into it
 * (the pages apply quantize-and-pack and decode attention per step; fusing them is this
 * library's choice).  A token that completes a 32-token per-channel key group (of any
 * sequence) takes the two-launch path, since the whole group is quantized then.  On a
 * ragged layer each sequence gets one token at its own length.  Per-layer plans only
 * (paged plans: KVQ_EINVAL). */
KVQ_API int kvq_append_decode(kvq_handle *h, int layer, const void *K, const void *V, const void *q,
                              void *out, int out_fp32, void *stream);

/* Decode path of kvq_decode_attn on per-layer plans (default KVQ_DECODE_MMA_SYNC).
 *
 * KVQ_DECODE_MMA_SYNC: decode_split_kernel, mma.sync tensor-core tiles in registers; every
 *   plan kvq_plan accepts.
 * KVQ_DECODE_TCGEN05: the same attention (the pages' flash-decoding splits merged by
 *   log-sum-exp, "TriAxialKV per-role mixed-precision KV quantization", Facts: decode
 *   path) with both contractions on the 5th-generation tensor cores: tcgen05.mma with
 *   operands staged in shared memory and accumulators in tensor memory.  Layers with
 *   head_dim 128 and at most 8 query heads per kv head, either key mode; head_dim 64
 *   fails with KVQ_EUNSUPPORTED (nothing is launched).  Results meet the same tolerances
 *   as the default path, not bit for bit the same values.
 *
 * kvq_append_decode (the fused step) and paged plans always use their own kernels.
 * Returns KVQ_EINVAL for an unknown path or a null handle; the setting applies to the
 * handle's later kvq_decode_attn calls. */
#define KVQ_DECODE_MMA_SYNC 0
#define KVQ_DECODE_TCGEN05 1
KVQ_API int kvq_set_decode_path(kvq_handle *h, int path);

/* Force the number of sequence splits used by kvq_decode_attn (0 = automatic; the
 * value is capped by the number of 32-token blocks and the partial buffer size). */
KVQ_API int kvq_set_num_splits(kvq_handle *h, int num_splits);

/* The split count kvq_decode_attn would use for `layer` at its current length, on the
 * handle's current decode path (kvq_set_decode_path). */
KVQ_API int kvq_get_num_splits(const kvq_handle *h, int layer, int *num_splits);

/* Copy one layer's cache to host memory in canonical order (parity checks): for each
 * (b, h) the records 0..ceil(L/32)-1 then, for per-channel keys, the residual; bytes
 * that hold no token of 0..L-1 are zero.  Paged plans: for each (b, h) the INT2 records
 * in group order, the INT4 main pages in order, the two pending pages, then the bf16
 * staging keys and values (32 x D each) of the open INT2 group.  Synchronous (device-wide).  If host_buf is
 * NULL or bytes is too small, only *needed is written (KVQ_EINVAL if too small). */
KVQ_API int kvq_export_layer(const kvq_handle *h, int layer, void *host_buf, size_t bytes,
                     size_t *needed);

/* Current length L of `layer` (the largest over its sequences). */
KVQ_API int kvq_seq_len(const kvq_handle *h, int layer, int *L);

/* Current length of every sequence of `layer`: L host int32 [batch].  Per-layer plans
 * only (paged plans: KVQ_EUNSUPPORTED). */
KVQ_API int kvq_seq_lens(const kvq_handle *h, int layer, int32_t *L);

/* Shorten every sequence of `layer` to L tokens (host bookkeeping only).  L <= the
 * shortest sequence and L % 32 == 0 (so no token of a kept block is partially
 * overwritten later). */
KVQ_API int kvq_truncate(kvq_handle *h, int layer, int L);

/* Empty the sequences seqs[0..n) in every layer (host bookkeeping only): their lengths
 * become 0 and, with block pools (desc.pool_blocks > 0), their blocks return to each
 * layer's pool for any sequence to take (continuous batching: a finished request leaves,
 * a new one takes its slot).  An emptied sequence must be appended to before the next
 * decode of a layer (decode needs every sequence non-empty).  Per-layer plans only
 * (paged plans: KVQ_EUNSUPPORTED); KVQ_EINVAL for an index outside [0, batch). */
KVQ_API int kvq_reset_sequences(kvq_handle *h, const int32_t *seqs, int n);


/* Read and clear the device status word (synchronizes `stream`).  KVQ_EDEVICE if a
 * kernel reported a bounded wait that expired; *flags gets the raw bits. */
KVQ_API int kvq_device_status(kvq_handle *h, void *stream, unsigned *flags);

/* Decode attention without any caller-provided scratch: the same computation and
 * arguments as kvq_decode_attn, but the split partials go to a 32 MiB buffer built
 * into the library (one per GPU that loads it, held until the process exits)
 * instead of the workspace.  For callers that cannot allocate or lend device scratch
 * (hosts that plan every device byte up front, code living in another component's
 * memory pool).  The pages describe no such entry point; it has no counterpart
 * there.  The first call on a device, with that device current, looks up the
 * buffer's device address; make that first call before any stream capture.  Returns
 * KVQ_EUNSUPPORTED when the call needs more partial space than the buffer holds:
 * a call split in S > 1 parts needs about B * Hq * S * (head_dim + 2) * 4 bytes
 * (batch 64 with 32 query heads at head_dim 128: up to 31 splits; no space without
 * splits).  All
 * calls share the one buffer: calls that may overlap on the GPU (different streams,
 * no ordering between them) race on it and must not be issued. */
KVQ_API int kvq_decode_attn_noalloc(kvq_handle *h, int layer, const void *q, void *out, int out_fp32,
                                    void *stream);

/* ---- Per-tag bit allocation of paged plans (host memory, no device work) ----------
 * From "TriAxialKV per-role mixed-precision KV quantization for agentic prefills",
 * Facts: the per-tag distortion D_k(b) is the attention-output MSE, taken as the max over
 * heads, the mean over requests and the sum over layers; each tag gets INT2 or INT4 under
 * an average-bit budget, by exhaustive search for 22 or fewer tags and a greedy
 * per-bit-gain rule otherwise.  The tagger (chat-template markers) is not part of this
 * library: tags arrive as integers. */

/* D_k(2) and D_k(4) for every tag k from calibration prefills (host pointers):
 *   Q bf16 [num_layers][num_requests][n_q_heads][T][head_dim],
 *   K, V bf16 [num_layers][num_requests][n_kv_heads][T][head_dim],
 *   tags int32 [num_requests][T] in [0, num_tags), shared by layers and heads.
 * For (tag k, b): the tokens of tag k are quantized at b bits and every other token is
 * kept exact; b = 4 quantizes K and V per token (groups of 32 channels); b = 2 quantizes
 * K per channel over consecutive 32-token groups of the tag's tokens of that request
 * (in token order) and V per token, and the tag's last T_k mod 32 tokens take the 4-bit
 * per-token path for K and V (leftover routing of the pages).  The error measure is the
 * mean squared difference of the causal attention outputs (all T queries, fp64) against
 * the exact keys and values, per query head; D_k(b) = sum over layers of the mean over
 * requests of the max over query heads.  Tags with no token get 0.  counts[k] receives
 * the number of tokens of tag k over all requests.  Cost O(layers x requests x tags x
 * n_q_heads x T^2 x head_dim), spread over the host's cores (as many as keep the
 * workers' T x T fp64 score buffers within about 2 GB): a calibration tool for prefills
 * of up to a few thousand tokens.  Errors: KVQ_EINVAL (counts, shapes: head_dim
 * a multiple of 32, n_q_heads a multiple of n_kv_heads; tags out of range; null). */
KVQ_API int kvq_tag_distortion(int num_layers, int num_requests, int n_q_heads, int n_kv_heads, int head_dim,
                               int T, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                               const int32_t *tags, int num_tags, double *D2, double *D4, int64_t *counts);

/* Device workspace bytes that kvq_tag_distortion_device needs at these sizes: the
 * per-request token lists, one layer's dequantized keys and values at 2 and 4 bits
 * (4 x num_requests x n_kv_heads x T x head_dim fp64) and the per-CTA error sums.
 * Errors as kvq_tag_distortion_device's size checks. */
KVQ_API int kvq_tag_distortion_workspace_bytes(int num_layers, int num_requests, int n_q_heads, int n_kv_heads,
                                               int head_dim, int T, int num_tags, size_t *bytes);

/* kvq_tag_distortion computed on the GPU: the same D_k(2), D_k(4) and counts, by the
 * same definition, with the attention in fp64 on the device (equal to the host entry
 * point's up to the order of the sums).  Q, K, V: device pointers, same layouts,
 * 16-byte aligned; tags, D2, D4, counts: host pointers; workspace: caller-owned device
 * memory of at least kvq_tag_distortion_workspace_bytes, 256-byte aligned.  Work is
 * issued on `stream`; the call returns after the results are on the host (it
 * synchronizes `stream`).  head_dim 64 or 128 (else KVQ_EUNSUPPORTED).  Cost
 * O(layers x requests x n_q_heads x T^2 x head_dim), about 4 passes over each query's
 * keys.  Errors: KVQ_EINVAL (shapes, tags out of range, null), KVQ_EALIGN,
 * KVQ_EUNBOUND (workspace), KVQ_ECUDA. */
KVQ_API int kvq_tag_distortion_device(int num_layers, int num_requests, int n_q_heads, int n_kv_heads,
                                      int head_dim, int T, const void *Q, const void *K, const void *V,
                                      const int32_t *tags, int num_tags, void *workspace, size_t workspace_bytes,
                                      double *D2, double *D4, int64_t *counts, void *stream);

/* bits[k] in {2, 4} for every tag: minimise sum_k D_{b_k}(k) subject to
 * sum_k counts[k] * bits[k] <= avg_bits * sum_k counts[k].  Tags with counts[k] == 0
 * take no part and get 4.  With P <= 22 tags present: exhaustive over all 2^P choices,
 * distortion summed in ascending tag order, the first least-distortion choice in
 * ascending mask order (bit i = the i-th present tag at INT2).  Otherwise greedy: start
 * from all INT4 and move to INT2 the tag of least (D_k(2) - D_k(4)) / (2 counts[k])
 * (ties: lower index) until the budget holds.  *total_distortion (if not NULL) gets the
 * chosen sum.  Errors: KVQ_EINVAL (avg_bits outside [2, 4], negative counts, null). */
KVQ_API int kvq_tag_allocate(int num_tags, const double *D2, const double *D4, const int64_t *counts,
                             double avg_bits, int *bits, double *total_distortion);

/* Free the handle (not the caller's workspace). */
KVQ_API void kvq_destroy(kvq_handle *h);

/* Message for the last failing call on this thread ("" if none). */
KVQ_API const char *kvq_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
