"""kvq_decode_attn_noalloc: decode attention for callers that cannot provide device
scratch (a host that plans every device byte up front, or code running inside another
component's memory pool).  Its split partials live in a buffer built into the library
instead of the caller's workspace.

The test calls it through the C ABI twice in a row and checks both results against
kvq_decode_attn on the same cache, within the tolerance the parity tests use.  It
needs no other test to run first: the first call on the device sets the buffer up.
"""
import numpy as np
import pytest
import torch

from layer_wise_mixed_b200 import configs, inputs, kvq

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 1e-2, 1e-3


def close(a: torch.Tensor, b: torch.Tensor):
    x = a.double().cpu().numpy()
    y = b.double().cpu().numpy()
    assert np.isfinite(x).all()
    err = x - y
    assert np.abs(err).max() <= TOL_ABS
    assert np.linalg.norm(err) / max(np.linalg.norm(y), 1e-30) <= TOL_REL


@pytest.mark.parametrize("kmode,splits", [(0, 3), (1, 5), (0, 1)])
def test_noalloc_matches_workspace_entry(kmode, splits):
    B, Hkv, G, D, L = 4, 8, 4, 128, 1000
    wl = configs.Workload("noalloc", 1, B, Hkv * G, Hkv, D, 0, 0, ((4, 2),))
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L, [(4, 2)], kmodes=[kmode])
    K, V = inputs.layer_kv(wl, 0, L, "cuda")
    cache.append(0, K, V)
    kvq.kvq_set_num_splits(cache.h, splits)
    assert kvq.kvq_get_num_splits(cache.h, 0) == splits
    q = inputs.step_q(wl, 0, 0, "cuda")
    for fp32 in (True, False):
        ref = cache.decode_attn(0, q, out_fp32=fp32)
        for _ in range(2):
            out = torch.full_like(ref, float("nan"))
            kvq.kvq_decode_attn_noalloc(cache.h, 0, q, out, fp32)
            torch.cuda.synchronize()
            close(out, ref)
    assert kvq.kvq_device_status(cache.h) == 0


def test_noalloc_split_at_batch_64():
    """The Llama-3.1-8B attention shape at batch 64 (2048 query rows) split three ways:
    the partials take 2048 x 3 x (128 + 2) x 4 bytes of the built-in buffer."""
    B, Hkv, G, D, L = 64, 8, 4, 128, 300
    wl = configs.Workload("noalloc-b64", 1, B, Hkv * G, Hkv, D, 0, 0, ((4, 2),))
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L, [(4, 2)])
    K, V = inputs.layer_kv(wl, 0, L, "cuda")
    cache.append(0, K, V)
    kvq.kvq_set_num_splits(cache.h, 3)
    q = inputs.step_q(wl, 0, 0, "cuda")
    ref = cache.decode_attn(0, q, out_fp32=True)
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        kvq.kvq_decode_attn_noalloc(cache.h, 0, q, out, True)
        torch.cuda.synchronize()
        close(out, ref)
    assert kvq.kvq_device_status(cache.h) == 0


def test_noalloc_rejects_oversized_partials():
    """A launch whose split partials exceed the built-in buffer is refused before launch
    (batch 64, 32 query heads, 40 splits: 2048 x 40 x 130 x 4 bytes > 32 MiB)."""
    B, Hkv, G, D, L = 64, 8, 4, 128, 40 * 32
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L, [(8, 8)])
    wl = configs.Workload("noalloc-big", 1, B, Hkv * G, Hkv, D, 0, 0, ((8, 8),))
    K, V = inputs.layer_kv(wl, 0, L, "cuda")
    cache.append(0, K, V)
    kvq.kvq_set_num_splits(cache.h, 40)
    q = inputs.step_q(wl, 0, 0, "cuda")
    out = torch.empty((B, Hkv * G, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attn_noalloc(cache.h, 0, q, out, False)
    assert e.value.code == kvq.KVQ_EUNSUPPORTED and "built-in scratch" in str(e.value)
