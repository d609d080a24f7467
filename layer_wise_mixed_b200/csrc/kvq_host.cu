// Host side of the C ABI declared in include/kvq.h: plan validation, workspace layout,
// argument checks, launch dispatch, split selection and the canonical export.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "kvq.h"
#include "kvq_internal.h"

using kvq::LayerGeom;

struct kvq_handle {
    kvq_plan_desc desc{};
    std::vector<kvq_layer_cfg> cfg;
    std::vector<LayerGeom> geom;
    std::vector<int> len;
    int cap_blk = 0;
    long long status_off = 0, smax_off = 0, meta_bytes = 0, part_acc_off = 0, part_ml_off = 0, total = 0;
    uint8_t *ws = nullptr;
    size_t ws_bytes = 0;
    int forced_splits = 0;
    int sm_count = 0;
    int device = -1;
    bool status_clear = false;   // status word zeroed on the device since the last bind
};

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok() {
    g_err.clear();
    return KVQ_OK;
}

bool valid_bits(int b) { return b == 2 || b == 4 || b == 8; }
long long align256(long long x) { return (x + 255) & ~255LL; }
bool aligned(const void *p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_layer(const kvq_handle *h, int layer) {
    if (!h) return fail(KVQ_EINVAL, "null handle");
    if (layer < 0 || layer >= h->desc.num_layers)
        return fail(KVQ_EINVAL, "layer %d out of range [0, %d)", layer, h->desc.num_layers);
    return KVQ_OK;
}

int check_bound(const kvq_handle *h) {
    if (!h->ws) return fail(KVQ_EUNBOUND, "no workspace bound (kvq_bind)");
    return KVQ_OK;
}

int cuda_fail(cudaError_t e, const char *what);

// The status word and the per-layer maximum scales live in caller memory of unknown
// content: zero them on the stream of the first launch after a bind.
int prepare_status(kvq_handle *h, cudaStream_t st) {
    if (h->status_clear) return KVQ_OK;
    cudaError_t e = cudaMemsetAsync(h->ws + h->status_off, 0, static_cast<size_t>(h->meta_bytes), st);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    h->status_clear = true;
    return KVQ_OK;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(KVQ_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Sequence splits for decode: minimise (waves) x (blocks per warp + per-CTA overhead).
int choose_splits(const kvq_handle *h, int units, int nblk, int slots) {
    const int smax = std::min(kvq::kMaxSplits, nblk);
    if (h->forced_splits > 0) return std::min(h->forced_splits, smax);
    int best = 1;
    double best_t = 1e300;
    for (int s = 1; s <= smax; ++s) {
        const int bps = (nblk + s - 1) / s;
        const int sreal = (nblk + bps - 1) / bps;
        const double waves = std::ceil(static_cast<double>(units) * sreal / std::max(1, slots));
        const double per_cta = std::ceil(static_cast<double>(bps) / kvq::kDecodeWarps) + 1.0;
        const double tcost = waves * per_cta * (1.0 + 0.002 * sreal);
        if (tcost < best_t - 1e-9) {
            best_t = tcost;
            best = sreal;
        }
    }
    return best;
}

}  // namespace

extern "C" {

const char *kvq_last_error(void) { return g_err.c_str(); }

int kvq_plan(const kvq_plan_desc *d, kvq_handle **out) {
    if (!d || !out) return fail(KVQ_EINVAL, "null argument");
    *out = nullptr;
    if (d->num_layers < 1 || d->batch < 1 || d->n_kv_heads < 1 || d->n_q_heads < 1 || d->max_ctx < 1)
        return fail(KVQ_EINVAL, "num_layers, batch, heads and max_ctx must be positive");
    if (d->n_q_heads % d->n_kv_heads)
        return fail(KVQ_EINVAL, "n_q_heads (%d) must be a multiple of n_kv_heads (%d)", d->n_q_heads, d->n_kv_heads);
    const int G = d->n_q_heads / d->n_kv_heads;
    if (G > 8) return fail(KVQ_EUNSUPPORTED, "GQA group %d > 8 not supported", G);
    if (d->group != kvq::kGroup) return fail(KVQ_EUNSUPPORTED, "group must be 32 (got %d)", d->group);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(KVQ_EUNSUPPORTED, "head_dim %d not supported (64 or 128)", d->head_dim);
    if (d->paged) return fail(KVQ_EUNSUPPORTED, "paged plans are not available in this build");
    if (!d->layers) return fail(KVQ_EINVAL, "null layer map");
    const long long max_units = static_cast<long long>(d->batch) * d->n_kv_heads;
    if (max_units > 65535LL * 65535LL) return fail(KVQ_EUNSUPPORTED, "too many (batch, head) units");
    if (d->batch > 65535 || d->n_kv_heads > 65535) return fail(KVQ_EUNSUPPORTED, "batch/heads exceed grid limits");

    auto *h = new kvq_handle();
    h->desc = *d;
    h->cfg.assign(d->layers, d->layers + d->num_layers);
    h->desc.layers = nullptr;
    h->cap_blk = (d->max_ctx + 31) / 32;
    const int D = d->head_dim;
    h->status_off = 0;
    h->smax_off = 256;                                      // after the status word
    h->meta_bytes = align256(256 + 8LL * d->num_layers);   // {K, V} max scale per layer
    long long off = h->meta_bytes;
    for (int l = 0; l < d->num_layers; ++l) {
        const kvq_layer_cfg &c = h->cfg[l];
        if (!valid_bits(c.bk) || !valid_bits(c.bv)) {
            delete h;
            return fail(KVQ_EINVAL, "layer %d: bits must be 2, 4 or 8 (bk=%d bv=%d)", l, c.bk, c.bv);
        }
        if (c.kmode != KVQ_PER_CHANNEL && c.kmode != KVQ_PER_TOKEN) {
            delete h;
            return fail(KVQ_EINVAL, "layer %d: bad key mode %d", l, c.kmode);
        }
        if (c.vmode != KVQ_PER_TOKEN) {
            delete h;
            return fail(KVQ_EUNSUPPORTED, "layer %d: values are quantized per token only", l);
        }
        if (c.kmode == KVQ_PER_TOKEN && (!(G == 1 || G == 2 || G == 4) || G * (D / 32) > 16)) {
            delete h;
            return fail(KVQ_EUNSUPPORTED, "layer %d: per-token keys need G in {1,2,4} and G*D/32 <= 16", l);
        }
        LayerGeom g{};
        g.bk = c.bk;
        g.bv = c.bv;
        g.kmode = c.kmode;
        g.kc = 4LL * D * c.bk;
        g.ks = 4LL * D;
        g.vc = 4LL * D * c.bv;
        g.vs = 4LL * D;
        g.rec_bytes = g.kc + g.ks + g.vc + g.vs;
        g.unit_bytes = g.rec_bytes * h->cap_blk;
        g.rec_off = off;
        off = align256(off + g.unit_bytes * max_units);
        if (c.kmode == KVQ_PER_CHANNEL) {
            g.res_off = off;
            off = align256(off + 64LL * D * max_units);
        } else {
            g.res_off = -1;
        }
        h->geom.push_back(g);
    }
    const long long rows = static_cast<long long>(d->batch) * d->n_q_heads;
    h->part_acc_off = off;
    off = align256(off + rows * kvq::kMaxSplits * D * 4);
    h->part_ml_off = off;
    off = align256(off + rows * kvq::kMaxSplits * 2 * 4);
    h->total = off;
    h->len.assign(d->num_layers, 0);
    *out = h;
    return ok();
}

int kvq_workspace_bytes(const kvq_handle *h, size_t *bytes) {
    if (!h || !bytes) return fail(KVQ_EINVAL, "null argument");
    *bytes = static_cast<size_t>(h->total);
    return ok();
}

int kvq_bind(kvq_handle *h, void *dev_ptr, size_t bytes) {
    if (!h || !dev_ptr) return fail(KVQ_EINVAL, "null argument");
    if (!aligned(dev_ptr, 256)) return fail(KVQ_EALIGN, "workspace must be 256-byte aligned");
    if (bytes < static_cast<size_t>(h->total))
        return fail(KVQ_EUNBOUND, "workspace too small: %zu < %lld bytes", bytes, h->total);
    h->ws = static_cast<uint8_t *>(dev_ptr);
    h->ws_bytes = bytes;
    h->status_clear = false;
    std::fill(h->len.begin(), h->len.end(), 0);
    return ok();
}

int kvq_append(kvq_handle *h, int layer, const void *K, const void *V, int n_new, void *stream) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if ((rc = check_bound(h))) return rc;
    if (!K || !V) return fail(KVQ_EINVAL, "null K or V");
    if (!aligned(K, 16) || !aligned(V, 16)) return fail(KVQ_EALIGN, "K and V must be 16-byte aligned");
    if (n_new < 1) return fail(KVQ_EINVAL, "n_new must be >= 1 (got %d)", n_new);
    const int L_old = h->len[layer];
    if (static_cast<long long>(L_old) + n_new > h->desc.max_ctx)
        return fail(KVQ_ECAPACITY, "layer %d: %d + %d tokens exceed max_ctx %d", layer, L_old, n_new, h->desc.max_ctx);
    const LayerGeom &g = h->geom[layer];
    const int units = h->desc.batch * h->desc.n_kv_heads;
    const int L_new = L_old + n_new;
    kvq::AppendParams p{};
    p.K = static_cast<const uint16_t *>(K);
    p.V = static_cast<const uint16_t *>(V);
    p.smax = reinterpret_cast<unsigned *>(h->ws + h->smax_off) + 2 * layer;
    p.rec = h->ws + g.rec_off;
    p.res = g.res_off >= 0 ? reinterpret_cast<uint16_t *>(h->ws + g.res_off) : nullptr;
    p.B = h->desc.batch;
    p.Hkv = h->desc.n_kv_heads;
    p.D = h->desc.head_dim;
    p.bk = g.bk;
    p.bv = g.bv;
    p.kmode = g.kmode;
    p.L_old = L_old;
    p.n = n_new;
    p.cap_blk = h->cap_blk;
    p.rec_bytes = g.rec_bytes;
    p.kc = g.kc;
    p.ks = g.ks;
    p.vc = g.vc;
    p.hb0 = L_old / 16;
    p.nhb = (L_new - 1) / 16 - p.hb0 + 1;
    p.g0 = L_old / 32;
    p.ng = L_new / 32 - L_old / 32;
    const long long nV = static_cast<long long>(units) * p.nhb;
    const long long nK = g.kmode == KVQ_PER_TOKEN ? nV : static_cast<long long>(units) * std::max(p.ng, 1);
    if (nV + nK > 0x7FFFFFFFLL) return fail(KVQ_EUNSUPPORTED, "append too large for one launch");
    p.nV = static_cast<int>(nV);
    p.nK = static_cast<int>(nK);
    if ((rc = prepare_status(h, static_cast<cudaStream_t>(stream)))) return rc;
    cudaError_t e = kvq::launch_append(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    h->len[layer] = L_new;
    return ok();
}

static int ensure_device_info(kvq_handle *h) {
    if (h->sm_count > 0) return KVQ_OK;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    e = cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    h->device = dev;
    return KVQ_OK;
}

static int splits_for(kvq_handle *h, int layer, int *S_out, int *nstage_out) {
    const LayerGeom &g = h->geom[layer];
    const int L = h->len[layer];
    const int nblk = (L + 31) / 32;
    const int G = h->desc.n_q_heads / h->desc.n_kv_heads;
    const int nstage = kvq::decode_stages(g.rec_bytes, h->desc.head_dim, G);
    int rc = ensure_device_info(h);
    if (rc) return rc;
    int per_sm = 1;
    cudaError_t e = kvq::decode_occupancy(h->desc.head_dim, g.bk, g.bv, g.kmode, G, g.rec_bytes, nstage, &per_sm);
    if (e != cudaSuccess) return cuda_fail(e, "decode occupancy");
    const int units = h->desc.batch * h->desc.n_kv_heads;
    *S_out = choose_splits(h, units, nblk, std::max(1, per_sm) * h->sm_count);
    *nstage_out = nstage;
    return KVQ_OK;
}

int kvq_decode_attn(kvq_handle *h, int layer, const void *q, void *out, int out_fp32, void *stream) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if ((rc = check_bound(h))) return rc;
    if (!q || !out) return fail(KVQ_EINVAL, "null q or out");
    if (!aligned(q, 16) || !aligned(out, 16)) return fail(KVQ_EALIGN, "q and out must be 16-byte aligned");
    const int L = h->len[layer];
    if (L < 1) return fail(KVQ_EINVAL, "layer %d is empty", layer);
    int S = 1, nstage = 2;
    if ((rc = splits_for(h, layer, &S, &nstage))) return rc;
    const LayerGeom &g = h->geom[layer];
    const int nblk = (L + 31) / 32;
    kvq::DecodeParams p{};
    p.rec = h->ws + g.rec_off;
    p.res = g.res_off >= 0 ? reinterpret_cast<const uint16_t *>(h->ws + g.res_off) : nullptr;
    p.q = static_cast<const uint16_t *>(q);
    p.smax = reinterpret_cast<const unsigned *>(h->ws + h->smax_off) + 2 * layer;
    p.out = out;
    p.part_acc = reinterpret_cast<float *>(h->ws + h->part_acc_off);
    p.part_ml = reinterpret_cast<float *>(h->ws + h->part_ml_off);
    p.status = reinterpret_cast<unsigned *>(h->ws + h->status_off);
    p.B = h->desc.batch;
    p.Hkv = h->desc.n_kv_heads;
    p.G = h->desc.n_q_heads / h->desc.n_kv_heads;
    p.L = L;
    p.cap_blk = h->cap_blk;
    p.bps = (nblk + S - 1) / S;
    p.S = (nblk + p.bps - 1) / p.bps;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.nstage = nstage;
    p.rec_bytes = g.rec_bytes;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = prepare_status(h, st))) return rc;
    cudaError_t e = kvq::launch_decode(p, h->desc.head_dim, g.bk, g.bv, g.kmode, st, nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    if (p.S > 1) {
        kvq::MergeParams m{};
        m.part_acc = p.part_acc;
        m.part_ml = p.part_ml;
        m.out = out;
        m.B = p.B;
        m.Hq = h->desc.n_q_heads;
        m.D = h->desc.head_dim;
        m.S = p.S;
        m.out_fp32 = p.out_fp32;
        e = kvq::launch_merge(m, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge launch");
    }
    return ok();
}

int kvq_set_num_splits(kvq_handle *h, int num_splits) {
    if (!h) return fail(KVQ_EINVAL, "null handle");
    if (num_splits < 0) return fail(KVQ_EINVAL, "num_splits must be >= 0");
    h->forced_splits = num_splits;
    return ok();
}

int kvq_get_num_splits(const kvq_handle *hc, int layer, int *num_splits) {
    int rc = check_layer(hc, layer);
    if (rc) return rc;
    if (!num_splits) return fail(KVQ_EINVAL, "null argument");
    kvq_handle *h = const_cast<kvq_handle *>(hc);
    const int L = h->len[layer];
    if (L < 1) {
        *num_splits = 0;
        return ok();
    }
    int S = 1, nstage = 2;
    if ((rc = splits_for(h, layer, &S, &nstage))) return rc;
    const int nblk = (L + 31) / 32;
    const int bps = (nblk + S - 1) / S;
    *num_splits = (nblk + bps - 1) / bps;
    return ok();
}

int kvq_export_layer(const kvq_handle *h, int layer, void *host_buf, size_t bytes, size_t *needed) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if (!needed) return fail(KVQ_EINVAL, "null argument");
    const LayerGeom &g = h->geom[layer];
    const int L = h->len[layer];
    const int nblk = (L + 31) / 32;
    const int D = h->desc.head_dim;
    const long long res_bytes = g.kmode == KVQ_PER_CHANNEL ? 64LL * D : 0;
    const long long unit_img = nblk * g.rec_bytes + res_bytes;
    const int units = h->desc.batch * h->desc.n_kv_heads;
    *needed = static_cast<size_t>(unit_img * units);
    if (!host_buf) return ok();
    if (bytes < *needed) return fail(KVQ_EINVAL, "export buffer too small: %zu < %zu", bytes, *needed);
    if ((rc = check_bound(h))) return rc;
    if (!h->status_clear) return fail(KVQ_EINVAL, "nothing appended since the workspace was bound");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    uint8_t *dst = static_cast<uint8_t *>(host_buf);
    const int r = L % 32;
    const int nj = D / 32;
    for (int u = 0; u < units; ++u) {
        uint8_t *img = dst + u * unit_img;
        if (nblk > 0) {
            e = cudaMemcpy(img, h->ws + g.rec_off + u * g.unit_bytes, nblk * g.rec_bytes, cudaMemcpyDeviceToHost);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy (records)");
        }
        if (res_bytes) {
            e = cudaMemcpy(img + nblk * g.rec_bytes, h->ws + g.res_off + u * res_bytes, res_bytes,
                           cudaMemcpyDeviceToHost);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy (residual)");
            std::memset(img + nblk * g.rec_bytes + 2LL * D * r, 0, res_bytes - 2LL * D * r);
        }
        if (r) {
            // zero every byte of the last block that holds no token of 0..L-1
            uint8_t *tail = img + (nblk - 1) * g.rec_bytes;
            // per-token scale/zero of token u, group j: 8*nj*(u/2) + 4j + 2(u%2), zero +4*nj
            auto zero_tok_sz = [&](uint8_t *area) {
                for (int u = r; u < 32; ++u)
                    for (int j = 0; j < nj; ++j) {
                        const long long so = 8LL * nj * (u / 2) + 4LL * j + 2LL * (u % 2);
                        std::memset(area + so, 0, 2);
                        std::memset(area + so + 4LL * nj, 0, 2);
                    }
            };
            if (g.kmode == KVQ_PER_CHANNEL) {
                std::memset(tail, 0, g.kc + g.ks);
            } else {
                if (r <= 16) std::memset(tail + 2LL * D * g.bk, 0, 2LL * D * g.bk);
                zero_tok_sz(tail + g.kc);
            }
            if (r <= 16) std::memset(tail + g.kc + g.ks + 2LL * D * g.bv, 0, 2LL * D * g.bv);
            zero_tok_sz(tail + g.kc + g.ks + g.vc);
        }
    }
    return ok();
}

int kvq_seq_len(const kvq_handle *h, int layer, int *L) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if (!L) return fail(KVQ_EINVAL, "null argument");
    *L = h->len[layer];
    return ok();
}

int kvq_truncate(kvq_handle *h, int layer, int L) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if (L < 0 || L > h->len[layer]) return fail(KVQ_EINVAL, "truncate length %d outside [0, %d]", L, h->len[layer]);
    if (L % 32) return fail(KVQ_EINVAL, "truncate length must be a multiple of 32 (got %d)", L);
    h->len[layer] = L;
    return ok();
}

int kvq_device_status(kvq_handle *h, void *stream, unsigned *flags) {
    if (!h) return fail(KVQ_EINVAL, "null handle");
    int rc = check_bound(h);
    if (rc) return rc;
    unsigned v = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&v, h->ws + h->status_off, sizeof v, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(h->ws + h->status_off, 0, sizeof v, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (flags) *flags = v;
    if (v) return fail(KVQ_EDEVICE, "device status 0x%x (a bounded wait expired)", v);
    return ok();
}

void kvq_destroy(kvq_handle *h) { delete h; }

}  // extern "C"

// ---------------------------------------------------------------------------------
// Decode attention for callers that cannot allocate device memory.
//
// kvq_decode_attn keeps its split partials in the caller's workspace.  Some callers
// cannot provide scratch at all: an embedded or real-time host that plans every
// device byte ahead of time, a plugin that runs inside someone else's memory pool,
// or code between the points where allocating would be unsafe.  For them the
// partials live in a fixed buffer compiled into this library.  The buffer exists
// once per GPU that loads the library and stays until the process exits.  Host code
// cannot use the array's name as a device address: the address is looked up once
// per device (the first call on that device, with that device current) and cached.
static constexpr size_t kStaticScratchBytes = size_t(32) << 20;   // 32 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
std::mutex g_scratch_mu;
void *g_scratch_addr[256];   // per device ordinal

int static_scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 256) return fail(KVQ_EUNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress (static scratch)");
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return KVQ_OK;
}
}  // namespace

extern "C" {

int kvq_decode_attn_noalloc(kvq_handle *h, int layer, const void *q, void *out, int out_fp32, void *stream) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if ((rc = check_bound(h))) return rc;
    if (!q || !out) return fail(KVQ_EINVAL, "null q or out");
    if (!aligned(q, 16) || !aligned(out, 16)) return fail(KVQ_EALIGN, "q and out must be 16-byte aligned");
    const int L = h->len[layer];
    if (L < 1) return fail(KVQ_EINVAL, "layer %d is empty", layer);
    int S = 1, nstage = 2;
    if ((rc = splits_for(h, layer, &S, &nstage))) return rc;
    const LayerGeom &g = h->geom[layer];
    const int nblk = (L + 31) / 32;
    const int bps = (nblk + S - 1) / S;
    S = (nblk + bps - 1) / bps;
    const long long rows = static_cast<long long>(h->desc.batch) * h->desc.n_q_heads;
    const long long acc_bytes = rows * kvq::kMaxSplits * h->desc.head_dim * 4;
    const long long need = S > 1 ? acc_bytes + rows * kvq::kMaxSplits * 2 * 4 : 0;
    if (need > static_cast<long long>(kStaticScratchBytes))
        return fail(KVQ_EUNSUPPORTED,
                    "split partials need %lld bytes but the built-in scratch holds %zu; use kvq_decode_attn",
                    need, kStaticScratchBytes);
    void *scratch = nullptr;
    if ((rc = static_scratch_address(&scratch))) return rc;
    kvq::DecodeParams p{};
    p.rec = h->ws + g.rec_off;
    p.res = g.res_off >= 0 ? reinterpret_cast<const uint16_t *>(h->ws + g.res_off) : nullptr;
    p.q = static_cast<const uint16_t *>(q);
    p.smax = reinterpret_cast<const unsigned *>(h->ws + h->smax_off) + 2 * layer;
    p.out = out;
    p.part_acc = static_cast<float *>(scratch);
    p.part_ml = reinterpret_cast<float *>(static_cast<unsigned char *>(scratch) + acc_bytes);
    p.status = reinterpret_cast<unsigned *>(h->ws + h->status_off);
    p.B = h->desc.batch;
    p.Hkv = h->desc.n_kv_heads;
    p.G = h->desc.n_q_heads / h->desc.n_kv_heads;
    p.L = L;
    p.cap_blk = h->cap_blk;
    p.bps = bps;
    p.S = S;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.nstage = nstage;
    p.rec_bytes = g.rec_bytes;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = prepare_status(h, st))) return rc;
    cudaError_t e = kvq::launch_decode(p, h->desc.head_dim, g.bk, g.bv, g.kmode, st, nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    if (p.S > 1) {
        kvq::MergeParams m{};
        m.part_acc = p.part_acc;
        m.part_ml = p.part_ml;
        m.out = out;
        m.B = p.B;
        m.Hq = h->desc.n_q_heads;
        m.D = h->desc.head_dim;
        m.S = p.S;
        m.out_fp32 = p.out_fp32;
        e = kvq::launch_merge(m, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge launch");
    }
    return ok();
}

}  // extern "C"
