/* A plain C99 consumer of include/kvq.h: the host-side entry points only (planning,
 * workspace sizes, argument errors, the per-tag allocator), so it runs without a GPU.
 * Prints one line per check and exits non-zero on the first failure. */
#include <stdio.h>
#include <string.h>

#include "kvq.h"

#define CHECK(cond, what)                                      \
    do {                                                       \
        if (!(cond)) {                                         \
            printf("FAIL %s (%s)\n", what, kvq_last_error());  \
            return 1;                                          \
        }                                                      \
        printf("ok %s\n", what);                               \
    } while (0)

int main(void) {
    kvq_layer_cfg layers[2] = {{8, 4, KVQ_PER_CHANNEL, KVQ_PER_TOKEN}, {4, 2, KVQ_PER_TOKEN, KVQ_PER_TOKEN}};
    kvq_plan_desc d;
    kvq_handle *h = NULL;
    size_t ws = 0, ws_pool = 0, calib = 0;
    int bits[3];
    double total = -1.0;
    const double D2[3] = {0.5, 0.1, 2.0}, D4[3] = {0.2, 0.05, 0.1};
    const int64_t counts[3] = {10, 10, 0};

    memset(&d, 0, sizeof d);
    d.num_layers = 2;
    d.batch = 4;
    d.n_kv_heads = 2;
    d.n_q_heads = 8;
    d.head_dim = 128;
    d.group = 32;
    d.max_ctx = 300;
    d.layers = layers;
    CHECK(kvq_plan(&d, &h) == KVQ_OK && h != NULL, "plan");
    CHECK(kvq_workspace_bytes(h, &ws) == KVQ_OK && ws > 0 && ws % 256 == 0, "workspace bytes");
    CHECK(kvq_set_decode_path(h, KVQ_DECODE_TCGEN05) == KVQ_OK, "decode path");
    CHECK(kvq_set_decode_path(h, 7) == KVQ_EINVAL, "unknown decode path refused");
    CHECK(kvq_decode_attn(h, 0, NULL, NULL, 0, NULL) != KVQ_OK, "decode without workspace refused");
    CHECK(strlen(kvq_last_error()) > 0, "error message");
    kvq_destroy(h);

    d.pool_blocks = 10;   /* block pools smaller than the 4 x 10 slab records */
    CHECK(kvq_plan(&d, &h) == KVQ_OK, "plan with block pools");
    CHECK(kvq_workspace_bytes(h, &ws_pool) == KVQ_OK && ws_pool < ws, "pools take less than slabs");
    kvq_destroy(h);

    d.pool_blocks = 0;
    d.n_q_heads = 7;      /* not a multiple of n_kv_heads */
    CHECK(kvq_plan(&d, &h) == KVQ_EINVAL, "bad head counts refused");
    d.n_q_heads = 8;
    d.group = 16;
    CHECK(kvq_plan(&d, &h) == KVQ_EUNSUPPORTED, "group 16 refused");

    CHECK(kvq_tag_distortion_workspace_bytes(2, 1, 8, 2, 128, 256, 3, &calib) == KVQ_OK && calib > 0,
          "calibration workspace bytes");
    /* 20 tokens in two tags at 3 bits: one tag can take INT2; tag 1 adds less distortion */
    CHECK(kvq_tag_allocate(3, D2, D4, counts, 3.0, bits, &total) == KVQ_OK, "allocate");
    CHECK(bits[0] == 4 && bits[1] == 2 && bits[2] == 4 && total == 0.1 + 0.2, "allocation");
    CHECK(kvq_tag_allocate(3, D2, D4, counts, 1.0, bits, &total) == KVQ_EINVAL, "budget below 2 bits refused");
    printf("all ok\n");
    return 0;
}
