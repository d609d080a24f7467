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
#include <unordered_map>
#include <vector>

#include "kvq.h"
#include "kvq_internal.h"

using kvq::LayerGeom;

struct kvq_handle {
    kvq_plan_desc desc{};
    std::vector<kvq_layer_cfg> cfg;
    std::vector<LayerGeom> geom;
    // per stream: the layers whose records or residual the last two launches of this
    // handle wrote (-1: none), for the decode's early block copies (kvq_internal.h,
    // pdl_enter)
    std::unordered_map<const void *, std::pair<int, int>> last_write;
    std::vector<int> len;                    // per layer: the largest request length
    std::vector<std::vector<int>> rlen;      // per-layer plans: per layer, per request
    std::vector<unsigned> ver;               // per layer: appends since bind (scale-maximum slot)
    int cap_blk = 0;
    long long status_off = 0, smax_off = 0, arrive_off = 0, meta_bytes = 0, part_acc_off = 0, part_ml_off = 0,
              total = 0;
    long long lens_off = 0;                  // per-layer plans: per layer [2][B] int32 length tables
    // block pools of per-layer plans (desc.pool_blocks > 0)
    bool pools = false;
    std::vector<long long> btab_off;                   // per layer: device block table [B][cap_blk]
    std::vector<std::vector<int>> free_blocks;         // per layer: free pool blocks (a stack)
    std::vector<std::vector<std::vector<int>>> blocks; // per layer, per request: pool blocks in order
    uint8_t *ws = nullptr;
    size_t ws_bytes = 0;
    int forced_splits = 0;
    int decode_path = KVQ_DECODE_MMA_SYNC;   // kvq_set_decode_path
    int sm_count = 0;
    int device = -1;
    bool status_clear = false;   // status word zeroed on the device since the last bind
    // paged INT2/INT4 plans
    struct PagedLayer {
        std::vector<int> n2g, n4, np;            // per request
        std::vector<std::vector<int>> rec2;      // INT2 record ids per request, in group order
        std::vector<std::vector<int>> page4;     // INT4 main page ids per request, in order
        int next2 = 0, next4 = 0;                // bump allocators of the two pools
    };
    long long n2_cap = 0, n4_main_cap = 0, n4_cap = 0;
    int P_cap = 0, pend_base = 0, inv_stride = 0;
    long long rec2_bytes = 0, page4_bytes = 0, inv_off = 0;
    std::vector<long long> pool2_off, pool4_off, staging_off, table_off;
    std::vector<PagedLayer> pl;
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

// The layer's device length table (per-layer plans): [B] lengths, or [B] old lengths then
// [B] counts for an append.
int *lens_table(const kvq_handle *h, int layer) {
    return reinterpret_cast<int *>(h->ws + h->lens_off) + 2LL * h->desc.batch * layer;
}

// A decode launch of `layer` on stream st may copy its first cache blocks before its
// PDL wait unless one of the two previous launches of this handle on st wrote that
// layer's cache.  Every launch is noted, with the layer whose cache it writes or -1.
int may_start_early(const kvq_handle *h, cudaStream_t st, int layer) {
    const auto it = h->last_write.find(static_cast<const void *>(st));
    if (it == h->last_write.end()) return 1;
    return (it->second.first != layer && it->second.second != layer) ? 1 : 0;
}
// Block pools: the device block table of `layer` ([B][cap_blk] int32), or null.
const int *block_table(const kvq_handle *h, int layer) {
    return h->pools ? reinterpret_cast<const int *>(h->ws + h->btab_off[layer]) : nullptr;
}

// Block pools: take from the layer's free stack the blocks that every request's new
// length L_new[b] needs (request order) and list the new table entries (index b * cap_blk
// + i, value = pool block) in idx / val.  KVQ_ECAPACITY, with nothing taken, if the pool
// has too few free blocks.
int reserve_blocks(kvq_handle *h, int layer, const std::vector<int> &L_new, std::vector<int> &idx,
                   std::vector<int> &val) {
    if (!h->pools) return KVQ_OK;
    auto &fb = h->free_blocks[layer];
    auto &bl = h->blocks[layer];
    long long need = 0;
    for (int b = 0; b < h->desc.batch; ++b)
        need += std::max(0LL, static_cast<long long>((L_new[b] + 31) / 32) - static_cast<long long>(bl[b].size()));
    if (need > static_cast<long long>(fb.size()))
        return fail(KVQ_ECAPACITY, "layer %d: block pool exhausted (%lld more blocks needed, %zu of %d free)", layer,
                    need, fb.size(), h->desc.pool_blocks);
    for (int b = 0; b < h->desc.batch; ++b)
        while (static_cast<int>(bl[b].size()) < (L_new[b] + 31) / 32) {
            const int pid = fb.back();
            fb.pop_back();
            idx.push_back(b * h->cap_blk + static_cast<int>(bl[b].size()));
            val.push_back(pid);
            bl[b].push_back(pid);
        }
    return KVQ_OK;
}

// Block pools: return the blocks of request b beyond its first `keep` to the free stack.
void release_blocks(kvq_handle *h, int layer, int b, int keep) {
    if (!h->pools) return;
    auto &v = h->blocks[layer][b];
    while (static_cast<int>(v.size()) > keep) {
        h->free_blocks[layer].push_back(v.back());
        v.pop_back();
    }
}

void note_write(kvq_handle *h, cudaStream_t st, int layer);

// Block pools: write new table entries on the stream (a launch that writes the layer's
// table: the next decode of the layer starts no copy before its wait).
int upload_blocks(kvq_handle *h, int layer, const std::vector<int> &idx, const std::vector<int> &val,
                  cudaStream_t st) {
    if (idx.empty()) return KVQ_OK;
    int *tab = reinterpret_cast<int *>(h->ws + h->btab_off[layer]);
    cudaError_t e = kvq::launch_scatter_table(tab, idx.data(), val.data(), static_cast<int>(idx.size()), st);
    if (e != cudaSuccess) return cuda_fail(e, "block table launch");
    for (size_t i = 0; i < idx.size(); i += 500) note_write(h, st, layer);
    return KVQ_OK;
}

void note_write(kvq_handle *h, cudaStream_t st, int layer) {

    auto it = h->last_write.find(static_cast<const void *>(st));
    if (it == h->last_write.end()) {
        h->last_write[static_cast<const void *>(st)] = {layer, -1};
    } else {
        it->second.second = it->second.first;
        it->second.first = layer;
    }
}


// Per-layer maxima of the fp16 scales {K, V}, kept in two slots by the parity of the
// layer's append count v: an append reads slot v & 1, writes slot (v + 1) & 1 (carrying
// the other slot forward) and makes v + 1; a decode reads slot v & 1.  A launch that
// appends and decodes reads slot v and writes slot v + 1, which nothing else touches
// during it.  Paged plans use slot 0 only.
unsigned *smax_slot(const kvq_handle *h, int layer, int parity) {
    return reinterpret_cast<unsigned *>(h->ws + h->smax_off) + 4 * layer + 2 * (parity & 1);
}

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

// Estimated time of a per-layer decode launch, in units of one block's processing by a
// warp.  CTAs are handed to SMs as slots free up, so the launch lasts about as long as
// the busiest SM's share: ceil(CTAs / SMs) CTAs, of which `occ` run at once; with fewer
// than `occ` an SM is not full and the CTAs' own latency decides.  A CTA costs its
// blocks per warp plus about two blocks of fixed latency (first copy, q set-up,
// combine); with a single stage per warp the copy latency of every block after the
// first is exposed too (about 0.6 of a block each).  Splitting adds the partial writes and
// the merge by each unit's last CTA.
double decode_cost(int units, int nblk, int S, int nstage, int occ, int sms) {
    const int bps = (nblk + S - 1) / S;
    const int sreal = (nblk + bps - 1) / bps;
    const double per_sm = std::ceil(static_cast<double>(units) * sreal / std::max(1, sms));
    const double load = std::max(1.0, per_sm / std::max(1, occ));
    const double bpw = std::ceil(static_cast<double>(bps) / kvq::kDecodeWarps);
    const double per_cta = bpw + 2.0 + (nstage == 1 ? 0.6 * (bpw - 1.0) : 0.0);
    return load * per_cta * (1.0 + 0.002 * sreal) + (sreal > 1 ? 0.5 : 0.0);
}

}  // namespace

namespace kvq {
int host_fail(int code, const char *msg) { return fail(code, "%s", msg); }
int host_ok() { return ok(); }
}  // namespace kvq

extern "C" {

const char *kvq_last_error(void) { return g_err.c_str(); }

int kvq_plan(const kvq_plan_desc *d, kvq_handle **out) {
    if (!d || !out) return fail(KVQ_EINVAL, "null argument");
    *out = nullptr;
    if (d->num_layers < 1 || d->batch < 1 || d->n_kv_heads < 1 || d->n_q_heads < 1 || d->max_ctx < 1)
        return fail(KVQ_EINVAL, "num_layers, batch, heads and max_ctx must be positive");
    if (d->n_q_heads % d->n_kv_heads)
        return fail(KVQ_EINVAL, "n_q_heads (%d) must be a multiple of n_kv_heads (%d)", d->n_q_heads, d->n_kv_heads);
    if (d->max_ctx > (1 << 30)) return fail(KVQ_EUNSUPPORTED, "max_ctx %d above 2^30 tokens", d->max_ctx);
    const int G = d->n_q_heads / d->n_kv_heads;
    if (G > 8) return fail(KVQ_EUNSUPPORTED, "GQA group %d > 8 not supported", G);
    if (d->group != kvq::kGroup) return fail(KVQ_EUNSUPPORTED, "group must be 32 (got %d)", d->group);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(KVQ_EUNSUPPORTED, "head_dim %d not supported (64 or 128)", d->head_dim);
    if (!d->paged && !d->layers) return fail(KVQ_EINVAL, "null layer map");
    if (d->paged) {
        if (d->head_dim != 128) return fail(KVQ_EUNSUPPORTED, "paged plans need head_dim 128");
        if (!(G == 1 || G == 2 || G == 4)) return fail(KVQ_EUNSUPPORTED, "paged plans need G in {1, 2, 4}");
        if (d->batch > kvq::kMaxPagedBatch) return fail(KVQ_EUNSUPPORTED, "paged plans take at most %d requests", kvq::kMaxPagedBatch);
        if (d->page_tokens != 16) return fail(KVQ_EUNSUPPORTED, "page_tokens must be 16");
        if (!(d->avg_bits >= 2.0f && d->avg_bits <= 4.0f)) return fail(KVQ_EINVAL, "avg_bits must be in [2, 4]");
    }
    const long long max_units = static_cast<long long>(d->batch) * d->n_kv_heads;
    if (max_units > 65535LL * 65535LL) return fail(KVQ_EUNSUPPORTED, "too many (batch, head) units");
    if (d->batch > 65535 || d->n_kv_heads > 65535) return fail(KVQ_EUNSUPPORTED, "batch/heads exceed grid limits");

    auto *h = new kvq_handle();
    h->desc = *d;
    if (d->layers) h->cfg.assign(d->layers, d->layers + d->num_layers);
    h->desc.layers = nullptr;
    if (d->paged) {
        // INT2 and INT4 pools of one region per (layer, kv head), split at an offset from
        // the expected mean bits: a fraction f2 = (4 - avg_bits)/2 of the tokens is INT2.
        const int D = d->head_dim;
        const double f2 = (4.0 - d->avg_bits) / 2.0;
        const double tokens = static_cast<double>(d->batch) * d->max_ctx;
        h->rec2_bytes = kvq::paged_rec2_bytes(D);
        h->page4_bytes = kvq::paged_page4_bytes(D);
        h->n2_cap = static_cast<long long>(std::ceil(f2 * tokens * 1.03 / 32.0)) + d->batch;
        h->n4_main_cap = static_cast<long long>(std::ceil((1.0 - f2) * tokens * 1.03 / 16.0)) + d->batch;
        // page tables hold int32 indices into the pools
        if (h->n2_cap >= (1LL << 31) || h->n4_main_cap + 2LL * d->batch >= (1LL << 31)) {
            delete h;
            return fail(KVQ_EUNSUPPORTED, "paged plan too large: pool pages exceed int32 page-table indices");
        }
        h->pend_base = static_cast<int>(h->n4_main_cap);
        h->n4_cap = h->n4_main_cap + 2LL * d->batch;
        h->P_cap = (d->max_ctx + 31) / 32 + (d->max_ctx + 15) / 16 + 1;
        h->inv_stride = d->max_ctx;
        h->status_off = 0;
        h->smax_off = 256;
        h->arrive_off = align256(256 + 16LL * d->num_layers);
        h->meta_bytes = align256(h->arrive_off + 4LL * d->batch * d->n_kv_heads);
        long long off = h->meta_bytes;
        for (int l = 0; l < d->num_layers; ++l) {
            h->pool2_off.push_back(off);
            off = align256(off + h->n2_cap * h->rec2_bytes * d->n_kv_heads);
            h->pool4_off.push_back(off);
            off = align256(off + h->n4_cap * h->page4_bytes * d->n_kv_heads);
            h->staging_off.push_back(off);
            off = align256(off + 2LL * d->batch * d->n_kv_heads * 32 * D * 2);
            h->table_off.push_back(off);
            off = align256(off + 4LL * d->batch * h->P_cap);
            LayerGeom g{};
            g.bk = 2;
            g.bv = 2;
            h->geom.push_back(g);
        }
        h->inv_off = off;
        off = align256(off + 2LL * 4 * d->batch * h->inv_stride);
        const long long rows = static_cast<long long>(d->batch) * d->n_q_heads;
        h->part_acc_off = off;
        off = align256(off + rows * kvq::kMaxSplits * D * 4);
        h->part_ml_off = off;
        off = align256(off + rows * kvq::kMaxSplits * 2 * 4);
        h->total = off;
        h->len.assign(d->num_layers, 0);
    h->ver.assign(d->num_layers, 0u);
        h->pl.assign(d->num_layers, kvq_handle::PagedLayer{});
        for (auto &x : h->pl) {
            x.n2g.assign(d->batch, 0);
            x.n4.assign(d->batch, 0);
            x.np.assign(d->batch, 0);
            x.rec2.assign(d->batch, {});
            x.page4.assign(d->batch, {});
        }
        *out = h;
        return ok();
    }
    h->cap_blk = (d->max_ctx + 31) / 32;
    if (d->pool_blocks < 0) {
        delete h;
        return fail(KVQ_EINVAL, "pool_blocks must be >= 0 (got %d)", d->pool_blocks);
    }
    h->pools = d->pool_blocks > 0;

    const int D = d->head_dim;
    h->status_off = 0;
    h->smax_off = 256;                                             // after the status word
    h->arrive_off = align256(256 + 16LL * d->num_layers);         // {K, V} max scale per layer and parity
    h->meta_bytes = align256(h->arrive_off + 4LL * d->batch * d->n_kv_heads);   // split arrival counters
    long long off = h->meta_bytes;
    // per-request length tables of batches above kvq::kMaxRagged (one per layer, so calls
    // on different layers never share one)
    h->lens_off = off;
    off = align256(off + 8LL * d->batch * d->num_layers);
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
        if (h->pools) {   // the layer's pool: pool_blocks blocks of one record per kv head
            off = align256(off + g.rec_bytes * d->n_kv_heads * static_cast<long long>(d->pool_blocks));
            h->btab_off.push_back(off);
            off = align256(off + 4LL * d->batch * h->cap_blk);
        } else {
            off = align256(off + g.unit_bytes * max_units);
        }
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
    h->ver.assign(d->num_layers, 0u);
    h->rlen.assign(d->num_layers, std::vector<int>(d->batch, 0));
    if (h->pools) {
        h->free_blocks.assign(d->num_layers, {});
        h->blocks.assign(d->num_layers, std::vector<std::vector<int>>(d->batch));
    }

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
    std::fill(h->ver.begin(), h->ver.end(), 0u);
    for (auto &r : h->rlen) std::fill(r.begin(), r.end(), 0);
    for (auto &x : h->pl) {
        std::fill(x.n2g.begin(), x.n2g.end(), 0);
        std::fill(x.n4.begin(), x.n4.end(), 0);
        std::fill(x.np.begin(), x.np.end(), 0);
        for (auto &v : x.rec2) v.clear();
        for (auto &v : x.page4) v.clear();
        x.next2 = x.next4 = 0;
    }
    if (h->pools) {   // every block free (taken from the stack's end: block 0 first)
        for (int l = 0; l < h->desc.num_layers; ++l) {
            auto &fb = h->free_blocks[l];
            fb.resize(h->desc.pool_blocks);
            for (int i = 0; i < h->desc.pool_blocks; ++i) fb[i] = h->desc.pool_blocks - 1 - i;
            for (auto &v : h->blocks[l]) v.clear();
        }
    }
    h->last_write.clear();
    return ok();
}

}  // extern "C"

namespace {

// Whether the requests of a per-layer plan's layer have different lengths.
bool layer_ragged(const kvq_handle *h, int layer) {
    const auto &r = h->rlen[layer];
    return std::any_of(r.begin(), r.end(), [&](int x) { return x != r[0]; });
}

// Append n[b] tokens to request b (n == nullptr: n_max to every request); K, V hold
// n_max token slots per (b, kv head).
int append_impl(kvq_handle *h, int layer, const void *K, const void *V, const int *n, int n_max, void *stream) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if ((rc = check_bound(h))) return rc;
    if (!K || !V) return fail(KVQ_EINVAL, "null K or V");
    if (!aligned(K, 16) || !aligned(V, 16)) return fail(KVQ_EALIGN, "K and V must be 16-byte aligned");
    if (n_max < 1) return fail(KVQ_EINVAL, "n_new must be >= 1 (got %d)", n_max);
    if (h->desc.paged) return fail(KVQ_EINVAL, "paged plans append with kvq_append_tagged");
    const int B = h->desc.batch;
    std::vector<int> Lo(h->rlen[layer]), nn(B, n_max);
    if (n)
        for (int b = 0; b < B; ++b) {
            if (n[b] < 0 || n[b] > n_max) return fail(KVQ_EINVAL, "request %d: n_new %d outside [0, %d]", b, n[b], n_max);
            nn[b] = n[b];
        }
    for (int b = 0; b < B; ++b)
        if (static_cast<long long>(Lo[b]) + nn[b] > h->desc.max_ctx)
            return fail(KVQ_ECAPACITY, "layer %d request %d: %d + %d tokens exceed max_ctx %d", layer, b, Lo[b], nn[b],
                        h->desc.max_ctx);
    const bool uniform = !layer_ragged(h, layer) && std::all_of(nn.begin(), nn.end(), [&](int x) { return x == nn[0]; });
    const LayerGeom &g = h->geom[layer];
    const int units = B * h->desc.n_kv_heads;
    kvq::AppendParams p{};
    p.K = static_cast<const uint16_t *>(K);
    p.V = static_cast<const uint16_t *>(V);
    p.smax = smax_slot(h, layer, static_cast<int>(h->ver[layer] + 1));
    p.smax_prev = smax_slot(h, layer, static_cast<int>(h->ver[layer]));
    p.rec = h->ws + g.rec_off;
    p.res = g.res_off >= 0 ? reinterpret_cast<uint16_t *>(h->ws + g.res_off) : nullptr;
    p.B = B;
    p.Hkv = h->desc.n_kv_heads;
    p.D = h->desc.head_dim;
    p.bk = g.bk;
    p.bv = g.bv;
    p.kmode = g.kmode;
    p.n = n_max;
    p.cap_blk = h->cap_blk;
    p.rec_bytes = g.rec_bytes;
    p.kc = g.kc;
    p.ks = g.ks;
    p.vc = g.vc;
    if (uniform) {
        const int L_old = Lo[0], L_new = L_old + nn[0];
        p.L_old = L_old;
        p.hb0 = L_old / 16;
        p.nhb = nn[0] > 0 ? (L_new - 1) / 16 - p.hb0 + 1 : 0;
        p.g0 = L_old / 32;
        p.ng = L_new / 32 - L_old / 32;
        if (nn[0] != n_max) {   // every request appends the same n < n_max: the ragged path
            p.ragged = 1;
        }
    } else {
        p.ragged = 1;
    }
    std::vector<int> table;   // [B] old lengths, then [B] counts (batches above kMaxRagged)
    if (p.ragged) {
        int nhb = 0, ng = 0;
        if (B > kvq::kMaxRagged) {
            table.assign(Lo.begin(), Lo.end());
            table.insert(table.end(), nn.begin(), nn.end());
        }
        for (int b = 0; b < B; ++b) {
            if (B <= kvq::kMaxRagged) {
                p.L_old_r[b] = Lo[b];
                p.n_r[b] = nn[b];
            }
            const int L_new = Lo[b] + nn[b];
            if (nn[b] > 0) nhb = std::max(nhb, (L_new - 1) / 16 - Lo[b] / 16 + 1);
            ng = std::max(ng, L_new / 32 - Lo[b] / 32);
        }
        p.nhb = nhb;
        p.ng = ng;
    }
    const long long nV = static_cast<long long>(units) * p.nhb;
    const long long nK = g.kmode == KVQ_PER_TOKEN ? nV : static_cast<long long>(units) * std::max(p.ng, 1);
    if (nV + nK > 0x7FFFFFFFLL) return fail(KVQ_EUNSUPPORTED, "append too large for one launch");
    p.nV = static_cast<int>(nV);
    p.nK = static_cast<int>(nK);
    if (p.nV + p.nK == 0) return ok();   // no token appended: nothing changes (the slot neither)
    std::vector<int> bidx, bval;         // block pools: new table entries
    {
        std::vector<int> L_new(B);
        for (int b = 0; b < B; ++b) L_new[b] = Lo[b] + nn[b];
        if ((rc = reserve_blocks(h, layer, L_new, bidx, bval))) return rc;
    }
    p.btab = block_table(h, layer);
    if ((rc = prepare_status(h, static_cast<cudaStream_t>(stream)))) return rc;
    if ((rc = upload_blocks(h, layer, bidx, bval, static_cast<cudaStream_t>(stream)))) return rc;
    if (!table.empty()) {

        int *dev = lens_table(h, layer);
        cudaError_t e = kvq::launch_set_table(dev, table.data(), static_cast<int>(table.size()),
                                              static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "length table launch");
        for (size_t i = 0; i < table.size(); i += 1000) note_write(h, static_cast<cudaStream_t>(stream), -1);
        p.ragged_dev = dev;
    }
    cudaError_t e = kvq::launch_append(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    note_write(h, static_cast<cudaStream_t>(stream), layer);
    int mx = 0;
    for (int b = 0; b < B; ++b) {
        h->rlen[layer][b] = Lo[b] + nn[b];
        mx = std::max(mx, h->rlen[layer][b]);
    }
    h->len[layer] = mx;
    ++h->ver[layer];
    return ok();
}

// Decode parameters' per-request lengths (ragged layers), each request's length plus
// `extra`: in the parameters, or (batches above kMaxRagged) in the layer's device table,
// written on `st`.  KVQ_EINVAL if a request would be empty.
int fill_lengths(kvq_handle *h, int layer, kvq::DecodeParams &p, int extra, cudaStream_t st) {
    p.ragged = 0;
    p.lens_dev = nullptr;
    if (!layer_ragged(h, layer)) return KVQ_OK;
    p.ragged = 1;
    const int B = h->desc.batch;
    std::vector<int> lens(B);
    for (int b = 0; b < B; ++b) {
        lens[b] = h->rlen[layer][b] + extra;
        if (lens[b] < 1) return fail(KVQ_EINVAL, "layer %d: request %d is empty", layer, b);
        if (B <= kvq::kMaxRagged) p.lens[b] = lens[b];
    }
    if (B > kvq::kMaxRagged) {
        int *dev = lens_table(h, layer);
        cudaError_t e = kvq::launch_set_table(dev, lens.data(), B, st);
        if (e != cudaSuccess) return cuda_fail(e, "length table launch");
        for (int i = 0; i < B; i += 1000) note_write(h, st, -1);
        p.lens_dev = dev;
    }
    return KVQ_OK;
}

}  // namespace

extern "C" {

int kvq_append(kvq_handle *h, int layer, const void *K, const void *V, int n_new, void *stream) {
    return append_impl(h, layer, K, V, nullptr, n_new, stream);
}

int kvq_append_ragged(kvq_handle *h, int layer, const void *K, const void *V, const int32_t *n_new, int n_max,
                      void *stream) {
    if (!n_new) return fail(KVQ_EINVAL, "null n_new");
    return append_impl(h, layer, K, V, n_new, n_max, stream);
}

int kvq_append_tagged(kvq_handle *h, int layer, const void *K, const void *V, int n_new,
                      const uint8_t *host_tags, const uint8_t *dev_tags, void *stream) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if ((rc = check_bound(h))) return rc;
    if (!h->desc.paged) return fail(KVQ_EINVAL, "kvq_append_tagged needs a paged plan");
    if (!K || !V || !host_tags || !dev_tags) return fail(KVQ_EINVAL, "null K, V or tags");
    if (!aligned(K, 16) || !aligned(V, 16)) return fail(KVQ_EALIGN, "K and V must be 16-byte aligned");
    if (n_new < 1) return fail(KVQ_EINVAL, "n_new must be >= 1 (got %d)", n_new);
    if (static_cast<long long>(h->len[layer]) + n_new > h->desc.max_ctx)
        return fail(KVQ_ECAPACITY, "layer %d: %d + %d tokens exceed max_ctx %d", layer, h->len[layer], n_new,
                    h->desc.max_ctx);
    const int B = h->desc.batch;
    auto &P = h->pl[layer];
    kvq::PagedAppendParams a{};
    int next2 = P.next2, next4 = P.next4;
    a.cta4_off[0] = a.cta2_off[0] = 0;
    for (int b = 0; b < B; ++b) {
        int k2 = 0, k4 = 0;
        for (int j = 0; j < n_new; ++j) {
            const uint8_t tg = host_tags[static_cast<long long>(b) * n_new + j];
            if (tg == 2) ++k2;
            else if (tg == 4) ++k4;
            else return fail(KVQ_EINVAL, "tag %d of request %d is %u (must be 2 or 4)", j, b, tg);
        }
        kvq::PagedReq &r = a.req[b];
        r.n2g_old = P.n2g[b];
        r.n4_old = P.n4[b];
        r.np_old = P.np[b];
        r.k2 = k2;
        r.k4 = k4;
        const int c0 = 32 * r.n2g_old + r.np_old, c1 = c0 + k2;
        r.ng = c1 / 32 - c0 / 32;
        r.base2 = next2;
        next2 += r.ng;
        const int n4p_old = (r.n4_old + 15) / 16, n4p_new = (r.n4_old + k4 + 15) / 16;
        r.base4 = next4;
        next4 += n4p_new - n4p_old;
        r.last4 = (r.n4_old % 16 && k4 > 0) ? P.page4[b].back() : -1;
        r.c4 = k4 > 0 ? (r.n4_old + k4 - 1) / 16 - r.n4_old / 16 + 1 : 0;
        r.c2 = std::max(r.ng, k2 > 0 ? 1 : 0);
        if (r.n2g_old + r.ng + n4p_new > h->P_cap)
            return fail(KVQ_ECAPACITY, "request %d: page table full", b);
        a.cta4_off[b + 1] = a.cta4_off[b] + r.c4;
        a.cta2_off[b + 1] = a.cta2_off[b] + r.c2;
    }
    if (next2 > h->n2_cap)
        return fail(KVQ_ECAPACITY, "INT2 pool full (%d of %lld records): the tags hold more INT2 tokens than avg_bits planned for",
                    next2, h->n2_cap);
    if (next4 > h->n4_main_cap)
        return fail(KVQ_ECAPACITY, "INT4 pool full (%d of %lld pages): the tags hold more INT4 tokens than avg_bits planned for",
                    next4, h->n4_main_cap);
    const int D = h->desc.head_dim;
    a.K = static_cast<const uint16_t *>(K);
    a.V = static_cast<const uint16_t *>(V);
    a.tags = dev_tags;
    a.inv2 = reinterpret_cast<const int *>(h->ws + h->inv_off);
    a.inv4 = a.inv2 + static_cast<long long>(B) * h->inv_stride;
    a.inv_stride = h->inv_stride;
    a.pool2 = h->ws + h->pool2_off[layer];
    a.pool4 = h->ws + h->pool4_off[layer];
    a.n2_cap = h->n2_cap;
    a.n4_cap = h->n4_cap;
    a.table = reinterpret_cast<int *>(h->ws + h->table_off[layer]);
    a.P_cap = h->P_cap;
    a.pend_base = h->pend_base;
    a.staging = reinterpret_cast<uint16_t *>(h->ws + h->staging_off[layer]);
    a.smax = smax_slot(h, layer, 0);
    a.B = B;
    a.Hkv = h->desc.n_kv_heads;
    a.D = D;
    a.n = n_new;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = prepare_status(h, st))) return rc;
    if (n_new > 1) {
        cudaError_t e = kvq::launch_paged_scan(dev_tags, B, n_new, const_cast<int *>(a.inv2), const_cast<int *>(a.inv4),
                                               h->inv_stride, st);
        if (e != cudaSuccess) return cuda_fail(e, "tag scan launch");
        note_write(h, st, -1);

    }
    const long long grid = static_cast<long long>(a.cta4_off[B] + a.cta2_off[B]) * a.Hkv;
    if (grid > 0x7FFFFFFFLL) return fail(KVQ_EUNSUPPORTED, "append too large for one launch");
    cudaError_t e = kvq::launch_paged_append(a, static_cast<int>(grid), st);
    if (e != cudaSuccess) return cuda_fail(e, "paged append launch");
    note_write(h, st, layer);
    // commit the host-side tables
    for (int b = 0; b < B; ++b) {
        const kvq::PagedReq &r = a.req[b];
        for (int i = 0; i < r.ng; ++i) P.rec2[b].push_back(r.base2 + i);
        const int n4p_old = (r.n4_old + 15) / 16, n4p_new = (r.n4_old + r.k4 + 15) / 16;
        for (int i = 0; i < n4p_new - n4p_old; ++i) P.page4[b].push_back(r.base4 + i);
        P.n2g[b] += r.ng;
        P.n4[b] += r.k4;
        P.np[b] = (32 * r.n2g_old + r.np_old + r.k2) % 32;
    }
    P.next2 = next2;
    P.next4 = next4;
    h->len[layer] += n_new;
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

// Split count and stages per warp of a per-layer decode launch: every split count and
// every stage count from 1 to the most that fit is costed with the occupancy it allows
// (deep rings fit fewer CTAs per SM; short sequences gain more from one wave than from
// prefetch depth).
// Split count S, stages per warp and extra stages (for the warps with the most blocks
// when one stage per warp is used) of a per-layer decode launch.
static int splits_for(kvq_handle *h, int layer, int *S_out, int *nstage_out, int *nextra_out) {
    const LayerGeom &g = h->geom[layer];
    const int L = h->len[layer];
    const int nblk = (L + 31) / 32;
    const int G = h->desc.n_q_heads / h->desc.n_kv_heads;
    const int ns_max = kvq::decode_stages(g.rec_bytes, h->desc.head_dim, G);
    int rc = ensure_device_info(h);
    if (rc) return rc;
    const int units = h->desc.batch * h->desc.n_kv_heads;
    const int smax = std::min(kvq::kMaxSplits, nblk);
    double best = 1e300;
    *S_out = 1;
    *nstage_out = ns_max;
    *nextra_out = 0;
    constexpr int NW = kvq::kDecodeWarps;
    for (int ns = 1; ns <= ns_max; ++ns)
        for (int nx = 0; nx < (ns == 1 ? NW : 1); ++nx) {
            int per_sm = 1;
            cudaError_t e =
                kvq::decode_occupancy(h->desc.head_dim, g.bk, g.bv, g.kmode, G, g.rec_bytes, ns, nx, &per_sm);
            if (e != cudaSuccess) return cuda_fail(e, "decode occupancy");
            for (int S = 1; S <= smax; ++S) {
                if (h->forced_splits > 0 && S != std::min(h->forced_splits, smax)) continue;
                const int bps = (nblk + S - 1) / S;
                const int sreal = (nblk + bps - 1) / bps;
                if (h->forced_splits <= 0 && sreal != S) continue;
                // extra stages: for exactly the warps with two blocks (warps 0 .. bps % NW
                // - 1) when every other warp has one, so that no warp waits for a copy
                // issued after its previous block
                if (nx > 0 && !(bps > NW && bps < 2 * NW && nx == bps % NW)) continue;
                const double c = decode_cost(units, nblk, S, nx > 0 ? 2 : ns, per_sm, h->sm_count);
                if (c < best - 1e-9) {
                    best = c;
                    *S_out = S;
                    *nstage_out = ns;
                    *nextra_out = nx;
                }
            }
        }
    return KVQ_OK;
}

// Early block copies pay only for short launches: one wave of CTAs whose warps hold one
// or two blocks each (the copies then land during the previous kernel's tail).  In longer
// launches they only put the q rows behind a CTA's block copies (measured on one B200:
// context-4096 and -8192 layers 3-7% slower with them, the 128-256-token layers of the
// batch-64 Llama shape 9% faster).
static bool early_pays(kvq_handle *h, int layer, const kvq::DecodeParams &p) {
    const LayerGeom &g = h->geom[layer];
    int occ = 1;
    if (kvq::decode_occupancy(h->desc.head_dim, g.bk, g.bv, g.kmode, p.G, g.rec_bytes, p.nstage, p.nextra, &occ) !=
        cudaSuccess)
        return false;
    const long long ctas = static_cast<long long>(p.B) * p.Hkv * p.S;
    return ctas <= static_cast<long long>(occ) * h->sm_count && (p.bps + kvq::kDecodeWarps - 1) / kvq::kDecodeWarps <= 2;
}

// ------------------------------------------------------------------ paged plans
static void paged_units(const kvq_handle *h, int layer, int *u2, int *u4) {
    const auto &P = h->pl[layer];
    *u2 = *u4 = 0;
    for (int b = 0; b < h->desc.batch; ++b) {
        *u2 = std::max(*u2, P.n2g[b]);
        // INT4 work items: pairs of full pages, the odd full page, the partial main and
        // pending pages
        const int F = P.n4[b] / 16 + P.np[b] / 16;
        *u4 = std::max(*u4, F / 2 + F % 2 + (P.n4[b] % 16 ? 1 : 0) + (P.np[b] % 16 ? 1 : 0));
    }
}

// INT2 and INT4 split counts: minimise (waves) x (slowest CTA), an INT2 unit (32 tokens,
// 2-bit record) weighing 1 and an INT4 item (mostly a pair of 16-token pages) 1.2.
static int paged_splits(kvq_handle *h, int layer, int *S2, int *S4) {
    int u2, u4;
    paged_units(h, layer, &u2, &u4);
    int rc = ensure_device_info(h);
    if (rc) return rc;
    int per_sm = 1;
    cudaError_t e = kvq::decode_paged_occupancy(kvq::decode_paged_stages(), &per_sm);
    if (e != cudaSuccess) return cuda_fail(e, "paged decode occupancy");
    const int slots = std::max(1, per_sm) * h->sm_count;
    const int units = h->desc.batch * h->desc.n_kv_heads;
    if (h->forced_splits > 0) {
        const int f = std::min(h->forced_splits, kvq::kMaxSplits);
        *S2 = u2 > 0 ? std::max(1, std::min(u2, (f + 1) / 2)) : 0;
        *S4 = u4 > 0 ? std::max(1, std::min(u4, f - *S2 > 0 ? f - *S2 : 1)) : 0;
        return KVQ_OK;
    }
    double best = 1e300;
    *S2 = u2 > 0 ? 1 : 0;
    *S4 = u4 > 0 ? 1 : 0;
    for (int a = (u2 > 0 ? 1 : 0); a <= (u2 > 0 ? std::min(32, u2) : 0); ++a)
        for (int c = (u4 > 0 ? 1 : 0); c <= (u4 > 0 ? std::min(48, u4) : 0); ++c) {
            if (a + c < 1 || a + c > kvq::kMaxSplits) continue;
            const double t2 = a ? std::ceil(std::ceil(static_cast<double>(u2) / a) / kvq::kDecodeWarps) : 0.0;
            const double t4 = c ? 1.2 * std::ceil(std::ceil(static_cast<double>(u4) / c) / kvq::kDecodeWarps) : 0.0;
            const double waves = std::ceil(static_cast<double>(units) * (a + c) / slots);
            const double cost = waves * (std::max(t2, t4) + 1.0) * (1.0 + 0.002 * (a + c));
            if (cost < best - 1e-9) {
                best = cost;
                *S2 = a;
                *S4 = c;
            }
        }
    return KVQ_OK;
}

static int decode_paged(kvq_handle *h, int layer, const void *q, void *out, int out_fp32, cudaStream_t st,
                        float *part_acc, float *part_ml) {
    int S2 = 0, S4 = 0;
    int rc = paged_splits(h, layer, &S2, &S4);
    if (rc) return rc;
    const auto &P = h->pl[layer];
    kvq::PagedDecodeParams p{};
    p.pool2 = h->ws + h->pool2_off[layer];
    p.pool4 = h->ws + h->pool4_off[layer];
    p.n2_cap = h->n2_cap;
    p.n4_cap = h->n4_cap;
    p.table = reinterpret_cast<const int *>(h->ws + h->table_off[layer]);
    p.P_cap = h->P_cap;
    p.pend_base = h->pend_base;
    for (int b = 0; b < h->desc.batch; ++b) p.cnt[b] = kvq::PagedCounts{P.n2g[b], P.n4[b], P.np[b], 0};
    p.q = static_cast<const uint16_t *>(q);
    p.smax = smax_slot(h, layer, 0);
    p.out = out;
    p.part_acc = part_acc;
    p.part_ml = part_ml;
    p.sstride = kvq::kMaxSplits;
    p.status = reinterpret_cast<unsigned *>(h->ws + h->status_off);
    p.B = h->desc.batch;
    p.Hkv = h->desc.n_kv_heads;
    p.G = h->desc.n_q_heads / h->desc.n_kv_heads;
    p.S2 = S2;
    p.S4 = S4;
    p.arrive = S2 + S4 >= kvq::kInLaunchMergeSplits ? reinterpret_cast<unsigned *>(h->ws + h->arrive_off) : nullptr;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.nstage = kvq::decode_paged_stages();
    if ((rc = prepare_status(h, st))) return rc;
    cudaError_t e = kvq::launch_decode_paged(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "paged decode launch");
    note_write(h, st, -1);
    if (S2 + S4 > 1 && !p.arrive) {
        kvq::MergeParams m{};
        m.part_acc = part_acc;
        m.part_ml = part_ml;
        m.out = out;
        m.B = p.B;
        m.Hq = h->desc.n_q_heads;
        m.D = h->desc.head_dim;
        m.S = S2 + S4;
        m.out_fp32 = p.out_fp32;
        m.sstride = p.sstride;
        e = kvq::launch_merge(m, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge launch");
        note_write(h, st, -1);
    }
    return ok();
}

// Split count of the tcgen05 decode: the one with the fewest CTA waves times chunks (4
// blocks) per CTA, one chunk of set-up counted per CTA; a forced count is taken as given.
static int umma_splits(kvq_handle *h, int layer, int *S_out) {
    const LayerGeom &g = h->geom[layer];
    const int nblk = (h->len[layer] + 31) / 32;
    int rc = ensure_device_info(h);
    if (rc) return rc;
    int occ = 1;
    cudaError_t e = kvq::decode_umma_occupancy(g.bk, g.bv, h->desc.n_q_heads / h->desc.n_kv_heads, g.kmode, &occ);
    if (e != cudaSuccess) return cuda_fail(e, "tcgen05 decode occupancy");
    const long long units = static_cast<long long>(h->desc.batch) * h->desc.n_kv_heads;
    const long long slots = static_cast<long long>(std::max(occ, 1)) * h->sm_count;
    const int smax = std::min(kvq::kMaxSplits, nblk);
    if (h->forced_splits > 0) {
        *S_out = std::min(h->forced_splits, smax);
        return KVQ_OK;
    }
    double best = 1e300;
    *S_out = 1;
    for (int S = 1; S <= smax; ++S) {
        const int bps = (nblk + S - 1) / S;
        if ((nblk + bps - 1) / bps != S) continue;
        const double waves = static_cast<double>((units * S + slots - 1) / slots);
        const double c = waves * ((bps + 3) / 4 + 1);
        if (c < best - 1e-9) {
            best = c;
            *S_out = S;
        }
    }
    return KVQ_OK;
}

// kvq_decode_attn on the tcgen05 kernel (head_dim 128, G <= 8, either key mode).
static int decode_umma(kvq_handle *h, int layer, const void *q, void *out, int out_fp32, cudaStream_t st) {
    const LayerGeom &g = h->geom[layer];
    const int G = h->desc.n_q_heads / h->desc.n_kv_heads;
    if (h->desc.head_dim != 128 || G > 8)
        return fail(KVQ_EUNSUPPORTED,
                    "the tcgen05 decode path takes head_dim 128 and at most 8 query heads per kv head (layer %d: "
                    "head_dim %d, %d heads per kv head)",
                    layer, h->desc.head_dim, G);
    const int L = h->len[layer];
    const int nblk = (L + 31) / 32;
    int S = 1, rc;
    if ((rc = umma_splits(h, layer, &S))) return rc;
    kvq::DecodeParams p{};
    p.rec = h->ws + g.rec_off;
    p.res = g.res_off >= 0 ? reinterpret_cast<const uint16_t *>(h->ws + g.res_off) : nullptr;
    p.q = static_cast<const uint16_t *>(q);
    p.smax = smax_slot(h, layer, static_cast<int>(h->ver[layer]));
    if ((rc = fill_lengths(h, layer, p, 0, st))) return rc;
    p.out = out;
    p.part_acc = reinterpret_cast<float *>(h->ws + h->part_acc_off);
    p.part_ml = reinterpret_cast<float *>(h->ws + h->part_ml_off);
    p.sstride = kvq::kMaxSplits;
    p.status = reinterpret_cast<unsigned *>(h->ws + h->status_off);
    p.B = h->desc.batch;
    p.Hkv = h->desc.n_kv_heads;
    p.G = G;
    p.L = L;
    p.cap_blk = h->cap_blk;
    p.bps = (nblk + S - 1) / S;
    p.S = (nblk + p.bps - 1) / p.bps;
    p.out_fp32 = out_fp32 ? 1 : 0;
    p.rec_bytes = g.rec_bytes;
    p.btab = block_table(h, layer);
    if ((rc = prepare_status(h, st))) return rc;
    cudaError_t e = kvq::launch_decode_umma(p, g.bk, g.bv, g.kmode, st);
    if (e != cudaSuccess) return cuda_fail(e, "tcgen05 decode launch");
    note_write(h, st, -1);
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
        m.sstride = p.sstride;
        e = kvq::launch_merge(m, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge launch");
        note_write(h, st, -1);
    }
    return ok();
}

int kvq_decode_attn(kvq_handle *h, int layer, const void *q, void *out, int out_fp32, void *stream) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if ((rc = check_bound(h))) return rc;
    if (!q || !out) return fail(KVQ_EINVAL, "null q or out");
    if (!aligned(q, 16) || !aligned(out, 16)) return fail(KVQ_EALIGN, "q and out must be 16-byte aligned");
    const int L = h->len[layer];
    if (L < 1) return fail(KVQ_EINVAL, "layer %d is empty", layer);
    if (h->desc.paged)
        return decode_paged(h, layer, q, out, out_fp32, static_cast<cudaStream_t>(stream),
                            reinterpret_cast<float *>(h->ws + h->part_acc_off),
                            reinterpret_cast<float *>(h->ws + h->part_ml_off));
    if (h->decode_path == KVQ_DECODE_TCGEN05)
        return decode_umma(h, layer, q, out, out_fp32, static_cast<cudaStream_t>(stream));
    int S = 1, nstage = 2, nextra = 0;
    if ((rc = splits_for(h, layer, &S, &nstage, &nextra))) return rc;
    const LayerGeom &g = h->geom[layer];
    const int nblk = (L + 31) / 32;
    kvq::DecodeParams p{};
    p.rec = h->ws + g.rec_off;
    p.res = g.res_off >= 0 ? reinterpret_cast<const uint16_t *>(h->ws + g.res_off) : nullptr;
    p.q = static_cast<const uint16_t *>(q);
    p.smax = smax_slot(h, layer, static_cast<int>(h->ver[layer]));
    if ((rc = fill_lengths(h, layer, p, 0, static_cast<cudaStream_t>(stream)))) return rc;
    p.out = out;
    p.part_acc = reinterpret_cast<float *>(h->ws + h->part_acc_off);
    p.part_ml = reinterpret_cast<float *>(h->ws + h->part_ml_off);
    p.sstride = kvq::kMaxSplits;
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
    p.nextra = nextra;
    p.rec_bytes = g.rec_bytes;
    p.arrive = p.S >= kvq::kInLaunchMergeSplits ? reinterpret_cast<unsigned *>(h->ws + h->arrive_off) : nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = prepare_status(h, st))) return rc;
    p.btab = block_table(h, layer);
    p.early = !p.lens_dev && may_start_early(h, st, layer) && early_pays(h, layer, p);
    cudaError_t e = kvq::launch_decode(p, h->desc.head_dim, g.bk, g.bv, g.kmode, st, nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    note_write(h, st, -1);
    if (p.S > 1 && !p.arrive) {
        kvq::MergeParams m{};
        m.part_acc = p.part_acc;
        m.part_ml = p.part_ml;
        m.out = out;
        m.B = p.B;
        m.Hq = h->desc.n_q_heads;
        m.D = h->desc.head_dim;
        m.S = p.S;
        m.out_fp32 = p.out_fp32;
        m.sstride = p.sstride;
        e = kvq::launch_merge(m, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge launch");
        note_write(h, st, -1);
    }
    return ok();
}

int kvq_append_decode(kvq_handle *h, int layer, const void *K, const void *V, const void *q, void *out,
                      int out_fp32, void *stream) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if ((rc = check_bound(h))) return rc;
    if (!K || !V || !q || !out) return fail(KVQ_EINVAL, "null K, V, q or out");
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(q, 16) || !aligned(out, 16))
        return fail(KVQ_EALIGN, "K, V, q and out must be 16-byte aligned");
    if (h->desc.paged) return fail(KVQ_EINVAL, "paged plans append with kvq_append_tagged");
    const int L_old = h->len[layer];
    const int B = h->desc.batch;
    for (int b = 0; b < B; ++b)
        if (static_cast<long long>(h->rlen[layer][b]) + 1 > h->desc.max_ctx)
            return fail(KVQ_ECAPACITY, "layer %d request %d: %d + 1 tokens exceed max_ctx %d", layer, b,
                        h->rlen[layer][b], h->desc.max_ctx);
    const LayerGeom &g = h->geom[layer];
    const int L = L_old + 1;
    bool completes = false;   // the token completes some request's key group
    for (int b = 0; b < B; ++b) completes = completes || (h->rlen[layer][b] + 1) % 32 == 0;
    if (g.kmode == KVQ_PER_CHANNEL && completes) {
        // the group is quantized by the append kernel
        if ((rc = kvq_append(h, layer, K, V, 1, stream))) return rc;
        return kvq_decode_attn(h, layer, q, out, out_fp32, stream);
    }
    std::vector<int> bidx, bval;   // block pools: a token that opens a block takes one
    {
        std::vector<int> L_new(B);
        for (int b = 0; b < B; ++b) L_new[b] = h->rlen[layer][b] + 1;
        if ((rc = reserve_blocks(h, layer, L_new, bidx, bval))) return rc;
    }
    h->len[layer] = L;   // the schedule is chosen for the new length
    int S = 1, nstage = 2, nextra = 0;
    if ((rc = splits_for(h, layer, &S, &nstage, &nextra))) {
        h->len[layer] = L_old;
        return rc;
    }
    const int nblk = (L + 31) / 32;
    kvq::DecodeParams p{};
    p.rec = h->ws + g.rec_off;
    p.res = g.res_off >= 0 ? reinterpret_cast<const uint16_t *>(h->ws + g.res_off) : nullptr;
    p.q = static_cast<const uint16_t *>(q);
    p.smax = smax_slot(h, layer, static_cast<int>(h->ver[layer]));
    if ((rc = fill_lengths(h, layer, p, 1, static_cast<cudaStream_t>(stream)))) {
        h->len[layer] = L_old;
        return rc;
    }
    p.out = out;
    p.part_acc = reinterpret_cast<float *>(h->ws + h->part_acc_off);
    p.part_ml = reinterpret_cast<float *>(h->ws + h->part_ml_off);
    p.sstride = kvq::kMaxSplits;
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
    p.nextra = nextra;
    p.rec_bytes = g.rec_bytes;
    p.arrive = p.S >= kvq::kInLaunchMergeSplits ? reinterpret_cast<unsigned *>(h->ws + h->arrive_off) : nullptr;
    p.k_new = static_cast<const uint16_t *>(K);
    p.v_new = static_cast<const uint16_t *>(V);
    p.rec_w = h->ws + g.rec_off;
    p.res_w = g.res_off >= 0 ? reinterpret_cast<uint16_t *>(h->ws + g.res_off) : nullptr;
    p.smax_out = smax_slot(h, layer, static_cast<int>(h->ver[layer] + 1));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = prepare_status(h, st))) {
        h->len[layer] = L_old;
        return rc;
    }
    if ((rc = upload_blocks(h, layer, bidx, bval, st))) {
        h->len[layer] = L_old;
        return rc;
    }
    p.btab = block_table(h, layer);
    p.early = !p.lens_dev && may_start_early(h, st, layer) && early_pays(h, layer, p);

    cudaError_t e = kvq::launch_decode(p, h->desc.head_dim, g.bk, g.bv, g.kmode, st, nullptr);
    if (e != cudaSuccess) {
        h->len[layer] = L_old;
        return cuda_fail(e, "fused append + decode launch");
    }
    note_write(h, st, layer);
    for (int b = 0; b < B; ++b) ++h->rlen[layer][b];
    ++h->ver[layer];
    if (p.S > 1 && !p.arrive) {
        kvq::MergeParams m{};
        m.part_acc = p.part_acc;
        m.part_ml = p.part_ml;
        m.out = out;
        m.B = p.B;
        m.Hq = h->desc.n_q_heads;
        m.D = h->desc.head_dim;
        m.S = p.S;
        m.out_fp32 = p.out_fp32;
        m.sstride = p.sstride;
        e = kvq::launch_merge(m, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge launch");
        note_write(h, st, -1);
    }
    return ok();
}

int kvq_set_decode_path(kvq_handle *h, int path) {
    if (!h) return fail(KVQ_EINVAL, "null handle");
    if (path != KVQ_DECODE_MMA_SYNC && path != KVQ_DECODE_TCGEN05) return fail(KVQ_EINVAL, "unknown decode path %d", path);
    h->decode_path = path;
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
    if (h->desc.paged) {
        int S2 = 0, S4 = 0;
        if ((rc = paged_splits(h, layer, &S2, &S4))) return rc;
        *num_splits = S2 + S4;
        return ok();
    }
    int S = 1, nstage = 2, nextra = 0;
    const int G = h->desc.n_q_heads / h->desc.n_kv_heads;
    if (h->decode_path == KVQ_DECODE_TCGEN05 && h->desc.head_dim == 128 && G <= 8) {
        if ((rc = umma_splits(h, layer, &S))) return rc;
    } else if ((rc = splits_for(h, layer, &S, &nstage, &nextra))) {
        return rc;
    }
    const int nblk = (L + 31) / 32;
    const int bps = (nblk + S - 1) / S;
    *num_splits = (nblk + bps - 1) / bps;
    return ok();
}

static int export_paged(const kvq_handle *h, int layer, void *host_buf, size_t bytes, size_t *needed) {
    const int B = h->desc.batch, Hkv = h->desc.n_kv_heads, D = h->desc.head_dim, nj = D / 32;
    const auto &P = h->pl[layer];
    const long long REC2 = h->rec2_bytes, PAGE4 = h->page4_bytes, STG = 2LL * 32 * D * 2;
    std::vector<long long> unit_bytes(B);
    long long total = 0;
    for (int b = 0; b < B; ++b) {
        unit_bytes[b] = P.n2g[b] * REC2 + ((P.n4[b] + 15) / 16 + 2) * PAGE4 + STG;
        total += unit_bytes[b] * Hkv;
    }
    *needed = static_cast<size_t>(total);
    if (!host_buf) return ok();
    if (bytes < *needed) return fail(KVQ_EINVAL, "export buffer too small: %zu < %zu", bytes, *needed);
    int rc = check_bound(h);
    if (rc) return rc;
    if (!h->status_clear) return fail(KVQ_EINVAL, "nothing appended since the workspace was bound");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    std::vector<uint8_t> pool2(static_cast<size_t>(h->n2_cap * REC2 * Hkv));
    std::vector<uint8_t> pool4(static_cast<size_t>(h->n4_cap * PAGE4 * Hkv));
    std::vector<uint8_t> stg(static_cast<size_t>(STG * B * Hkv));
    e = cudaMemcpy(pool2.data(), h->ws + h->pool2_off[layer], pool2.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(pool4.data(), h->ws + h->pool4_off[layer], pool4.size(), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(stg.data(), h->ws + h->staging_off[layer], stg.size(), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy (paged pools)");
    // zero the scale/zero entries of absent tokens u >= r of a 16-token page
    auto zero_absent = [&](uint8_t *page, int r) {
        for (int u = r; u < 16; ++u)
            for (int j = 0; j < nj; ++j) {
                const long long so = 8LL * nj * (u / 2) + 4LL * j + 2LL * (u % 2);
                for (long long area : {2LL * D * 4, 2LL * D * 4 + 2LL * D + 2LL * D * 4}) {
                    std::memset(page + area + so, 0, 2);
                    std::memset(page + area + so + 4LL * nj, 0, 2);
                }
            }
    };
    uint8_t *dst = static_cast<uint8_t *>(host_buf);
    for (int b = 0; b < B; ++b)
        for (int h2 = 0; h2 < Hkv; ++h2) {
            uint8_t *img = dst;
            for (int g = 0; g < P.n2g[b]; ++g)
                std::memcpy(img + g * REC2, pool2.data() + (static_cast<long long>(h2) * h->n2_cap + P.rec2[b][g]) * REC2, REC2);
            uint8_t *pg = img + P.n2g[b] * REC2;
            const int n4p = (P.n4[b] + 15) / 16;
            for (int i = 0; i < n4p; ++i) {
                std::memcpy(pg + i * PAGE4, pool4.data() + (static_cast<long long>(h2) * h->n4_cap + P.page4[b][i]) * PAGE4, PAGE4);
                if (i == n4p - 1 && P.n4[b] % 16) zero_absent(pg + i * PAGE4, P.n4[b] % 16);
            }
            uint8_t *pend = pg + n4p * PAGE4;
            const int np = P.np[b];
            for (int i = 0; i < 2; ++i) {
                if (np > 16 * i) {
                    std::memcpy(pend + i * PAGE4, pool4.data() + (static_cast<long long>(h2) * h->n4_cap + h->pend_base + 2 * b + i) * PAGE4, PAGE4);
                    if (np < 16 * (i + 1)) zero_absent(pend + i * PAGE4, np - 16 * i);
                } else {
                    std::memset(pend + i * PAGE4, 0, PAGE4);
                }
            }
            uint8_t *sg = pend + 2 * PAGE4;
            const uint8_t *src = stg.data() + (static_cast<long long>(b) * Hkv + h2) * STG;
            std::memset(sg, 0, STG);
            std::memcpy(sg, src, 2LL * np * D);                            // keys of slots [0, np)
            std::memcpy(sg + STG / 2, src + STG / 2, 2LL * np * D);        // values
            dst += unit_bytes[b];
        }
    return ok();
}

int kvq_export_layer(const kvq_handle *h, int layer, void *host_buf, size_t bytes, size_t *needed) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if (!needed) return fail(KVQ_EINVAL, "null argument");
    if (h->desc.paged) return export_paged(h, layer, host_buf, bytes, needed);
    const LayerGeom &g = h->geom[layer];
    const int D = h->desc.head_dim, Hkv = h->desc.n_kv_heads;
    const long long res_bytes = g.kmode == KVQ_PER_CHANNEL ? 64LL * D : 0;
    const int units = h->desc.batch * Hkv;
    auto unit_len = [&](int u) { return h->rlen[layer][u / Hkv]; };
    auto unit_img = [&](int u) { return (unit_len(u) + 31) / 32 * g.rec_bytes + res_bytes; };
    long long total = 0;
    for (int u = 0; u < units; ++u) total += unit_img(u);
    *needed = static_cast<size_t>(total);
    if (!host_buf) return ok();
    if (bytes < *needed) return fail(KVQ_EINVAL, "export buffer too small: %zu < %zu", bytes, *needed);
    if ((rc = check_bound(h))) return rc;
    if (!h->status_clear) return fail(KVQ_EINVAL, "nothing appended since the workspace was bound");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    uint8_t *img = static_cast<uint8_t *>(host_buf);
    const int nj = D / 32;
    for (int u = 0; u < units; img += unit_img(u), ++u) {
        const int L = unit_len(u), nblk = (L + 31) / 32, r = L % 32;
        if (nblk > 0 && !h->pools) {
            e = cudaMemcpy(img, h->ws + g.rec_off + u * g.unit_bytes, nblk * g.rec_bytes, cudaMemcpyDeviceToHost);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy (records)");
        }
        for (int blk = 0; blk < nblk && h->pools; ++blk) {   // gathered through the block table
            const long long ri = static_cast<long long>(h->blocks[layer][u / Hkv][blk]) * Hkv + u % Hkv;
            e = cudaMemcpy(img + blk * g.rec_bytes, h->ws + g.rec_off + ri * g.rec_bytes, g.rec_bytes,
                           cudaMemcpyDeviceToHost);
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

int kvq_seq_lens(const kvq_handle *h, int layer, int32_t *L) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if (!L) return fail(KVQ_EINVAL, "null argument");
    if (h->desc.paged) return fail(KVQ_EUNSUPPORTED, "paged plans report one length per layer");
    for (int b = 0; b < h->desc.batch; ++b) L[b] = h->rlen[layer][b];
    return ok();
}

int kvq_truncate(kvq_handle *h, int layer, int L) {
    int rc = check_layer(h, layer);
    if (rc) return rc;
    if (h->desc.paged) return fail(KVQ_EUNSUPPORTED, "paged plans cannot be truncated");
    const int shortest = *std::min_element(h->rlen[layer].begin(), h->rlen[layer].end());
    if (L < 0 || L > shortest) return fail(KVQ_EINVAL, "truncate length %d outside [0, %d]", L, shortest);
    if (L % 32) return fail(KVQ_EINVAL, "truncate length must be a multiple of 32 (got %d)", L);
    h->len[layer] = L;
    std::fill(h->rlen[layer].begin(), h->rlen[layer].end(), L);
    for (int b = 0; b < h->desc.batch; ++b) release_blocks(h, layer, b, L / 32);
    return ok();
}

int kvq_reset_sequences(kvq_handle *h, const int32_t *seqs, int n) {
    if (!h || (n > 0 && !seqs)) return fail(KVQ_EINVAL, "null argument");
    if (h->desc.paged) return fail(KVQ_EUNSUPPORTED, "paged plans cannot reset single sequences");
    if (n < 0) return fail(KVQ_EINVAL, "n must be >= 0 (got %d)", n);
    for (int i = 0; i < n; ++i)
        if (seqs[i] < 0 || seqs[i] >= h->desc.batch)
            return fail(KVQ_EINVAL, "sequence %d out of range [0, %d)", seqs[i], h->desc.batch);
    for (int l = 0; l < h->desc.num_layers; ++l) {
        for (int i = 0; i < n; ++i) {
            h->rlen[l][seqs[i]] = 0;
            release_blocks(h, l, seqs[i], 0);
        }
        h->len[l] = *std::max_element(h->rlen[l].begin(), h->rlen[l].end());
    }
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
    if (h->desc.paged) return fail(KVQ_EUNSUPPORTED, "paged plans are not supported by kvq_decode_attn_noalloc");
    int S = 1, nstage = 2, nextra = 0;
    if ((rc = splits_for(h, layer, &S, &nstage, &nextra))) return rc;
    const LayerGeom &g = h->geom[layer];
    const int nblk = (L + 31) / 32;
    const int bps = (nblk + S - 1) / S;
    S = (nblk + bps - 1) / bps;
    const long long rows = static_cast<long long>(h->desc.batch) * h->desc.n_q_heads;
    // partials packed at the launch's own split count: [B][Hq][S][D] then [B][Hq][S][2]
    const long long acc_bytes = (rows * S * h->desc.head_dim * 4 + 255) / 256 * 256;
    const long long need = S > 1 ? acc_bytes + rows * S * 2 * 4 : 0;
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
    p.smax = smax_slot(h, layer, static_cast<int>(h->ver[layer]));
    if ((rc = fill_lengths(h, layer, p, 0, static_cast<cudaStream_t>(stream)))) return rc;
    p.out = out;
    p.part_acc = static_cast<float *>(scratch);
    p.part_ml = reinterpret_cast<float *>(static_cast<unsigned char *>(scratch) + acc_bytes);
    p.sstride = S;
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
    p.nextra = nextra;
    p.rec_bytes = g.rec_bytes;
    p.arrive = p.S >= kvq::kInLaunchMergeSplits ? reinterpret_cast<unsigned *>(h->ws + h->arrive_off) : nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = prepare_status(h, st))) return rc;
    p.btab = block_table(h, layer);
    p.early = !p.lens_dev && may_start_early(h, st, layer) && early_pays(h, layer, p);
    cudaError_t e = kvq::launch_decode(p, h->desc.head_dim, g.bk, g.bv, g.kmode, st, nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    note_write(h, st, -1);
    if (p.S > 1 && !p.arrive) {
        kvq::MergeParams m{};
        m.part_acc = p.part_acc;
        m.part_ml = p.part_ml;
        m.out = out;
        m.B = p.B;
        m.Hq = h->desc.n_q_heads;
        m.D = h->desc.head_dim;
        m.S = p.S;
        m.out_fp32 = p.out_fp32;
        m.sstride = p.sstride;
        e = kvq::launch_merge(m, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge launch");
        note_write(h, st, -1);
    }
    return ok();
}

}  // extern "C"
