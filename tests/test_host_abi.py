"""C-ABI library on the CPU: it loads, exports every symbol include/kvq.h declares, and
its host-side checks reject bad plans and arguments before any CUDA call."""
import ctypes

import pytest

from layer_wise_mixed_b200 import build as kbuild
from layer_wise_mixed_b200 import kvq


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kvq.load()


def test_exports_every_declared_symbol(lib):
    names = kvq.header_functions()
    assert {"kvq_plan", "kvq_append", "kvq_decode_attn", "kvq_export_layer", "kvq_bind",
            "kvq_workspace_bytes", "kvq_destroy", "kvq_last_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def desc(**kw):
    a = dict(num_layers=2, batch=2, n_kv_heads=2, n_q_heads=4, head_dim=64, max_ctx=100,
             layer_bits=[(4, 2), (8, 8)])
    kmodes = kw.pop("kmodes", None)
    a.update(kw)
    return kvq.make_desc(a["num_layers"], a["batch"], a["n_kv_heads"], a["n_q_heads"], a["head_dim"],
                         a["max_ctx"], a["layer_bits"], kmodes)


def plan_rc(d):
    h = ctypes.c_void_p()
    rc = kvq.load().kvq_plan(ctypes.byref(d), ctypes.byref(h))
    if rc == 0:
        kvq.kvq_destroy(h.value)
    return rc


def test_plan_validation(lib):
    assert plan_rc(desc()) == kvq.KVQ_OK
    assert plan_rc(desc(layer_bits=[(3, 2), (8, 8)])) == kvq.KVQ_EINVAL
    assert plan_rc(desc(layer_bits=[(4, 16), (8, 8)])) == kvq.KVQ_EINVAL
    assert plan_rc(desc(n_q_heads=5)) == kvq.KVQ_EINVAL
    assert plan_rc(desc(head_dim=96)) == kvq.KVQ_EUNSUPPORTED
    assert plan_rc(desc(n_q_heads=18)) == kvq.KVQ_EUNSUPPORTED          # G = 9
    assert plan_rc(desc(batch=0)) == kvq.KVQ_EINVAL
    assert plan_rc(desc(max_ctx=(1 << 31) - 1)) == kvq.KVQ_EUNSUPPORTED   # block counts would wrap
    assert plan_rc(desc(kmodes=[1, 0])) == kvq.KVQ_OK
    assert plan_rc(desc(kmodes=[1, 0], n_q_heads=6)) == kvq.KVQ_EUNSUPPORTED   # per-token keys, G = 3
    d = desc()
    d.group = 64
    assert plan_rc(d) == kvq.KVQ_EUNSUPPORTED
    d = desc()
    d.layers[0].vmode = kvq.KVQ_PER_CHANNEL
    assert plan_rc(d) == kvq.KVQ_EUNSUPPORTED
    assert "per token" in kvq.kvq_last_error()


def test_workspace_layout(lib):
    d = desc(layer_bits=[(4, 2), (8, 8)], kmodes=[0, 1])
    h = kvq.kvq_plan(d)
    try:
        D, B, Hkv, Hq, cap = 64, 2, 2, 4, (100 + 31) // 32
        rec0 = 4 * D * 4 + 4 * D + 4 * D * 2 + 4 * D
        rec1 = 4 * D * 8 + 4 * D + 4 * D * 8 + 4 * D
        al = lambda x: (x + 255) // 256 * 256
        expect = al(256 + 16 * 2)                      # status word + {K, V} max scale per layer and parity
        expect = al(expect + 4 * B * Hkv)               # split arrival counters per (b, kv head)
        expect = al(expect + 8 * B * 2)                 # per-layer [2][B] length tables (large ragged batches)
        expect = al(expect + rec0 * cap * B * Hkv)
        expect = al(expect + 64 * D * B * Hkv)          # residual of the per-channel layer
        expect = al(expect + rec1 * cap * B * Hkv)
        expect = al(expect + B * Hq * 64 * D * 4)
        expect = al(expect + B * Hq * 64 * 2 * 4)
        assert kvq.kvq_workspace_bytes(h) == expect
    finally:
        kvq.kvq_destroy(h)


def test_argument_checks_before_any_launch(lib):
    h = kvq.kvq_plan(desc())
    L = kvq.load()
    try:
        # not bound yet
        assert L.kvq_append(h, 0, 4096, 4096, 1, None) == kvq.KVQ_EUNBOUND
        n = kvq.kvq_workspace_bytes(h)
        assert L.kvq_bind(h, 4096 + 16, n) == kvq.KVQ_EALIGN
        assert L.kvq_bind(h, 4096, n - 1) == kvq.KVQ_EUNBOUND
        fake = 1 << 40                      # never dereferenced: every call below fails on the host
        assert L.kvq_bind(h, fake, n) == kvq.KVQ_OK
        assert L.kvq_append(h, 2, fake, fake, 1, None) == kvq.KVQ_EINVAL      # layer
        assert L.kvq_append(h, 0, None, fake, 1, None) == kvq.KVQ_EINVAL      # null
        assert L.kvq_append(h, 0, fake + 8, fake, 1, None) == kvq.KVQ_EALIGN
        assert L.kvq_append(h, 0, fake, fake, 0, None) == kvq.KVQ_EINVAL      # n_new
        assert L.kvq_append(h, 0, fake, fake, 101, None) == kvq.KVQ_ECAPACITY
        assert L.kvq_decode_attn(h, 0, fake, fake, 0, None) == kvq.KVQ_EINVAL  # empty layer
        assert L.kvq_decode_attn(h, 0, fake + 4, fake, 0, None) == kvq.KVQ_EALIGN
        assert "16-byte" in kvq.kvq_last_error()
        assert L.kvq_append_decode(h, 0, fake, fake + 8, fake, fake, 0, None) == kvq.KVQ_EALIGN
        assert L.kvq_append_decode(h, 0, fake, None, fake, fake, 0, None) == kvq.KVQ_EINVAL
        assert L.kvq_append_decode(h, 5, fake, fake, fake, fake, 0, None) == kvq.KVQ_EINVAL
        assert kvq.kvq_seq_len(h, 1) == 0
        need = ctypes.c_size_t()
        assert L.kvq_export_layer(h, 0, None, 0, ctypes.byref(need)) == kvq.KVQ_OK
        assert need.value == (2 * 2) * 32 * 64 * 2     # empty layer: a 32 x 64 bf16 residual per unit
        assert L.kvq_truncate(h, 0, 1) == kvq.KVQ_EINVAL
        assert L.kvq_set_num_splits(h, -1) == kvq.KVQ_EINVAL
        assert L.kvq_set_num_splits(h, 3) == kvq.KVQ_OK
        assert L.kvq_set_decode_path(None, kvq.KVQ_DECODE_TCGEN05) == kvq.KVQ_EINVAL
        assert L.kvq_set_decode_path(h, 2) == kvq.KVQ_EINVAL
        assert L.kvq_set_decode_path(h, kvq.KVQ_DECODE_TCGEN05) == kvq.KVQ_OK
        # the tcgen05 path takes head_dim 128 only; this plan's is 64: refused on the host
        assert L.kvq_decode_attn(h, 0, fake, fake, 0, None) == kvq.KVQ_EINVAL      # still: empty layer first
        assert L.kvq_set_decode_path(h, kvq.KVQ_DECODE_MMA_SYNC) == kvq.KVQ_OK
    finally:
        kvq.kvq_destroy(h)


def test_ragged_argument_checks_before_any_launch(lib):
    import numpy as np
    L = kvq.load()
    h = kvq.kvq_plan(desc())                         # batch 2, max_ctx 100
    try:
        fake = 1 << 40
        assert L.kvq_bind(h, fake, kvq.kvq_workspace_bytes(h)) == kvq.KVQ_OK
        p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
        assert L.kvq_append_ragged(h, 0, fake, fake, None, 4, None) == kvq.KVQ_EINVAL            # null counts
        assert L.kvq_append_ragged(h, 0, fake, fake, p(np.array([5, 1], np.int32)), 4, None) == kvq.KVQ_EINVAL
        assert L.kvq_append_ragged(h, 0, fake, fake, p(np.array([-1, 1], np.int32)), 4, None) == kvq.KVQ_EINVAL
        assert L.kvq_append_ragged(h, 0, fake, fake, p(np.array([1, 101], np.int32)), 120, None) == kvq.KVQ_ECAPACITY
        assert "request 1" in kvq.kvq_last_error()
        assert L.kvq_append_ragged(h, 0, fake, fake, p(np.array([1, 1], np.int32)), 0, None) == kvq.KVQ_EINVAL
        assert list(kvq.kvq_seq_lens(h, 0, 2)) == [0, 0]
    finally:
        kvq.kvq_destroy(h)
    h = kvq.kvq_plan(desc(batch=65))                 # above 64 requests: lengths in a device table
    try:
        fake = 1 << 40
        assert L.kvq_bind(h, fake, kvq.kvq_workspace_bytes(h)) == kvq.KVQ_OK
        counts = np.ones(65, np.int32)
        counts[3] = 3                                 # outside [0, n_max]: refused before any launch
        assert L.kvq_append_ragged(h, 0, fake, fake, counts.ctypes.data_as(ctypes.c_void_p), 2, None) == \
            kvq.KVQ_EINVAL
        assert "request 3" in kvq.kvq_last_error()
        assert list(kvq.kvq_seq_lens(h, 0, 65)) == [0] * 65
    finally:
        kvq.kvq_destroy(h)

    h = kvq.kvq_plan(kvq.make_paged_desc(1, 2, 2, 8, 128, 64, 3.0))
    try:
        with pytest.raises(kvq.KvqError):
            kvq.kvq_seq_lens(h, 0, 2)
    finally:
        kvq.kvq_destroy(h)


def test_product_path_has_no_fallback(monkeypatch, tmp_path):
    """Without libkvq.so the binding raises; it never computes anything itself."""
    monkeypatch.setattr(kvq, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(kvq, "_lib", None)
    with pytest.raises(FileNotFoundError):
        kvq.load()


def paged_rc(**kw):
    a = dict(num_layers=2, batch=3, n_kv_heads=2, n_q_heads=8, head_dim=128, max_ctx=200, avg_bits=3.0)
    a.update(kw)
    d = kvq.make_paged_desc(a["num_layers"], a["batch"], a["n_kv_heads"], a["n_q_heads"], a["head_dim"],
                            a["max_ctx"], a["avg_bits"])
    return plan_rc(d)


def test_paged_plan_validation(lib):
    assert paged_rc() == kvq.KVQ_OK
    assert paged_rc(head_dim=64) == kvq.KVQ_EUNSUPPORTED
    assert paged_rc(n_q_heads=14) == kvq.KVQ_EUNSUPPORTED          # G = 7
    assert paged_rc(batch=65) == kvq.KVQ_EUNSUPPORTED
    assert paged_rc(avg_bits=5.0) == kvq.KVQ_EINVAL
    assert paged_rc(avg_bits=1.5) == kvq.KVQ_EINVAL
    # page tables hold int32 pool indices: pools past 2^31 pages are refused, not wrapped
    assert paged_rc(batch=64, max_ctx=1 << 20, avg_bits=3.0) == kvq.KVQ_OK
    assert paged_rc(batch=64, max_ctx=1 << 30, avg_bits=2.0) == kvq.KVQ_EUNSUPPORTED   # INT2 pool
    assert paged_rc(batch=64, max_ctx=1 << 30, avg_bits=4.0) == kvq.KVQ_EUNSUPPORTED   # INT4 pool
    assert "int32" in kvq.kvq_last_error()


def test_paged_host_checks(lib):
    import numpy as np
    d = kvq.make_paged_desc(1, 2, 2, 8, 128, 300, 4.0)    # avg 4 bits: the INT2 pool holds ~2 groups
    h = kvq.kvq_plan(d)
    L = kvq.load()
    try:
        n = kvq.kvq_workspace_bytes(h)
        fake = 1 << 40
        assert L.kvq_bind(h, fake, n) == kvq.KVQ_OK
        assert L.kvq_append(h, 0, fake, fake, 1, None) == kvq.KVQ_EINVAL      # needs the tagged entry
        bad = np.full((2, 3), 3, np.uint8)
        ptr = bad.ctypes.data_as(ctypes.c_void_p)
        assert L.kvq_append_tagged(h, 0, fake, fake, 3, ptr, fake, None) == kvq.KVQ_EINVAL
        assert "must be 2 or 4" in kvq.kvq_last_error()
        many2 = np.full((2, 200), 2, np.uint8)                   # 12 groups > INT2 pool
        ptr = many2.ctypes.data_as(ctypes.c_void_p)
        assert L.kvq_append_tagged(h, 0, fake, fake, 200, ptr, fake, None) == kvq.KVQ_ECAPACITY
        assert "INT2 pool full" in kvq.kvq_last_error()
        assert kvq.kvq_seq_len(h, 0) == 0                        # nothing committed
        assert L.kvq_truncate(h, 0, 0) == kvq.KVQ_EUNSUPPORTED
        need = ctypes.c_size_t()
        assert L.kvq_export_layer(h, 0, None, 0, ctypes.byref(need)) == kvq.KVQ_OK
        assert need.value == 2 * 2 * (2 * 20 * 128 + 2 * 32 * 128 * 2)   # empty: pending pages + staging
    finally:
        kvq.kvq_destroy(h)


def test_block_pool_plan_layout_and_checks(lib):
    """Block pools: the layer regions hold the pool and the block table instead of the
    slabs; an append the pool cannot hold is refused before any launch and leaves the
    lengths as they were; kvq_reset_sequences checks its arguments."""
    import numpy as np
    L = kvq.load()
    D, B, Hkv, Hq, cap, P = 64, 2, 2, 4, (100 + 31) // 32, 3
    d = kvq.make_desc(2, B, Hkv, Hq, D, 100, [(4, 2), (8, 8)], None, pool_blocks=P)
    h = kvq.kvq_plan(d)
    try:
        rec0 = 4 * D * 4 + 4 * D + 4 * D * 2 + 4 * D
        rec1 = 4 * D * 8 + 4 * D + 4 * D * 8 + 4 * D
        al = lambda x: (x + 255) // 256 * 256
        expect = al(256 + 16 * 2)
        expect = al(expect + 4 * B * Hkv)
        expect = al(expect + 8 * B * 2)
        expect = al(expect + rec0 * Hkv * P)            # layer 0 pool
        expect = al(expect + 4 * B * cap)               # layer 0 block table
        expect = al(expect + 64 * D * B * Hkv)          # residual (per-channel keys)
        expect = al(expect + rec1 * Hkv * P)
        expect = al(expect + 4 * B * cap)
        expect = al(expect + 64 * D * B * Hkv)
        expect = al(expect + B * Hq * 64 * D * 4)
        expect = al(expect + B * Hq * 64 * 2 * 4)
        assert kvq.kvq_workspace_bytes(h) == expect
        fake = 1 << 40
        assert L.kvq_bind(h, fake, expect) == kvq.KVQ_OK
        # 2 sequences x 2 blocks (64 tokens) > 3 pool blocks: refused before any launch
        assert L.kvq_append(h, 0, fake, fake, 64, None) == kvq.KVQ_ECAPACITY
        assert "block pool" in kvq.kvq_last_error()
        assert list(kvq.kvq_seq_lens(h, 0, B)) == [0, 0]
        p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
        assert L.kvq_reset_sequences(h, p(np.array([0, 2], np.int32)), 2) == kvq.KVQ_EINVAL   # out of range
        assert L.kvq_reset_sequences(h, None, 1) == kvq.KVQ_EINVAL
        assert L.kvq_reset_sequences(h, p(np.array([1], np.int32)), 1) == kvq.KVQ_OK
    finally:
        kvq.kvq_destroy(h)
    d = kvq.make_desc(1, B, Hkv, Hq, D, 100, [(4, 2)], None, pool_blocks=-1)
    assert plan_rc(d) == kvq.KVQ_EINVAL
