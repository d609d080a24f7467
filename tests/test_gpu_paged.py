"""GPU parity of the paged INT2/INT4 path against the oracle: the exported logical image
(INT2 records, INT4 pages, pending pages, staging) is byte-equal, and decode attention
meets the T1/T2 tolerances, for several tag patterns and append schedules."""
import numpy as np
import pytest
import torch

import oracle
from layer_wise_mixed_b200 import configs, inputs, kvq
from test_gpu_parity import bits16, check_outputs

pytestmark = pytest.mark.gpu


def tag_rows(B, L, pattern, seed=0):
    r = np.random.default_rng(seed)
    rows = []
    for b in range(B):
        p = pattern if pattern != "mix" else ["bern", "all2", "all4", "alt"][b % 4]
        if p == "all2":
            rows.append(np.full(L, 2))
        elif p == "all4":
            rows.append(np.full(L, 4))
        elif p == "alt":
            rows.append(np.where(np.arange(L) % 2 == 0, 2, 4))
        else:
            rows.append(np.where(r.random(L) < 0.5, 2, 4))
    return np.stack(rows).astype(np.uint8)


def run_paged(B, Hkv, G, chunks, tags, decode_at=None, splits=(0,), wl=None, avg_bits=None, layers=1):
    L_total = sum(chunks)
    D = 128
    if avg_bits is None:   # size the pools for the actual tag mix
        avg_bits = 4.0 - 2.0 * float((tags[:, :L_total] == 2).mean())
    wl = wl or configs.Workload("paged-case", layers, B, Hkv * G, Hkv, D, 0, 0, ((2, 2),))
    cache = kvq.Cache(layers, B, Hkv, Hkv * G, D, L_total, avg_bits=avg_bits)
    decode_at = set(decode_at or [L_total])
    dtags = torch.from_numpy(tags).cuda()
    for l in range(layers):
        K, V = inputs.layer_kv(wl, l, L_total, "cuda")
        Kb, Vb = bits16(K), bits16(V)
        L = 0
        for n in chunks:
            cache.append_tagged(l, K[:, :, L:L + n].contiguous(), V[:, :, L:L + n].contiguous(),
                                dtags[:, L:L + n].contiguous())
            L += n
            if L not in decode_at:
                continue
            q = inputs.step_q(wl, l, L, "cuda")
            img_ref, out_ref = oracle.paged_layer(Kb[:, :, :L], Vb[:, :, :L], tags[:, :L], bits16(q), G)
            img = cache.export_layer(l)
            assert img.shape == img_ref.shape, (img.shape, img_ref.shape)
            if not np.array_equal(img, img_ref):
                bad = np.flatnonzero(img != img_ref)
                pytest.fail(f"paged layer {l} L={L}: image differs at {bad.size} bytes, first {bad[:8]}")
            for S in splits:
                kvq.kvq_set_num_splits(cache.h, S)
                out32 = cache.decode_attn(l, q, out_fp32=True)
                out16 = cache.decode_attn(l, q, out_fp32=False)
                torch.cuda.synchronize()
                check_outputs(out32, out16, out_ref, f"paged layer {l} L={L} splits={S}")
            kvq.kvq_set_num_splits(cache.h, 0)
    assert kvq.kvq_device_status(cache.h) == 0
    return cache


@pytest.mark.parametrize("pattern", ["bern", "all2", "all4", "alt", "mix"])
def test_paged_bulk_then_tokens(pattern):
    """A 100-token prefill then 40 single tokens (INT2 groups complete along the way)."""
    B, L = 4, 140
    tags = tag_rows(B, L, pattern, seed=1)
    run_paged(B, 2, 4, [100] + [1] * 40, tags, decode_at=[100, 101, 117, 140], splits=(0, 1, 2, 5))


def test_paged_chunked_appends():
    B = 3
    chunks = [37, 5, 64, 1, 1, 20, 33, 2]
    tags = tag_rows(B, sum(chunks), "mix", seed=2)
    run_paged(B, 2, 4, chunks, tags, decode_at=[37, 106, 108, 128, 161, 163], splits=(0, 3))


@pytest.mark.parametrize("G", [1, 2, 4])
def test_paged_gqa(G):
    B, L = 2, 90
    tags = tag_rows(B, L, "bern", seed=3 + G)
    run_paged(B, 2, G, [60, 30], tags, decode_at=[60, 90], splits=(0, 2))


def test_paged_single_token_from_empty():
    """Token-by-token from an empty cache through two INT2 group completions."""
    B, L = 2, 70
    tags = tag_rows(B, L, "mix", seed=9)
    run_paged(B, 2, 4, [1] * L, tags, decode_at=[1, 2, 31, 32, 33, 64, 70], splits=(0,))


@pytest.mark.slow
def test_paged_c5_full_layer():
    """Full C5 size for one layer: Llama-3.1-8B shape, batch 16, context 32768 with
    Bernoulli(0.5) INT2/INT4 tags, then 17 decode steps, automatic splits."""
    wl = configs.paged_c5()
    L0, steps = wl.prefill, 17
    tags = inputs.tags(wl, L0 + steps).numpy()
    run_paged(wl.batch, wl.n_kv_heads, wl.G, [L0] + [1] * steps, tags, decode_at=[L0 + 1, L0 + steps],
              wl=wl, avg_bits=wl.avg_bits)


def test_paged_segment_tag_mask():
    """Masks with the per-tag allocation's structure: runs of 16-256 tokens share one
    precision (segment tag ids mapped by a fixed table: even ids INT2, odd INT4), so INT2
    groups complete in the middle of runs and pending pages fill from several runs;
    prompt of 1500 tokens, then 40 single tokens, splits automatic and forced."""
    B, L0, n = 4, 1500, 40
    wl = configs.Workload("paged-seg", 1, B, 2 * 4, 2, 128, 0, 0, ((2, 2),))
    ids = inputs.tag_ids(wl, L0 + n).numpy()
    tags = np.where(ids % 2 == 0, 2, 4).astype(np.uint8)
    run_paged(B, 2, 4, [L0] + [1] * n, tags, decode_at=[L0, L0 + 1, L0 + 17, L0 + n], splits=(0, 3, 6), wl=wl)
