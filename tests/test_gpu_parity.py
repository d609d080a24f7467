"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

* Packed cache (codes, scales, zeros, residual) bit-exact: the exported canonical
  image equals the oracle's image of the same token sequence.
* Decode attention within tolerance of the oracle's fp64 attention over the
  dequantized cache:
    T1 fp32 output:  max-abs <= 1e-2 and relative L2 <= 1e-3 (whole tensor and every
                     (batch, query head) row);
    T2 bf16 output:  against the oracle rounded to bf16, relative L2 <= 1e-3 and
                     max-abs <= max(1e-2, one bf16 ulp of the oracle value).
Inputs are seeded synthetic tensors (layer_wise_mixed_b200.inputs); the oracle gets
the same bytes copied from the device.
"""
import numpy as np
import pytest
import torch

import oracle
from layer_wise_mixed_b200 import configs, inputs, kvq

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 1e-2, 1e-3


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.bfloat16).double().numpy()


def check_outputs(out32: torch.Tensor, out16: torch.Tensor, ref: np.ndarray, what=""):
    o = out32.double().cpu().numpy()
    assert np.isfinite(o).all(), what
    err = o - ref
    assert np.abs(err).max() <= TOL_ABS, (what, np.abs(err).max())
    # relative errors where the reference is not zero; a zero reference row (all values
    # zero) must come out exactly zero
    rn = np.linalg.norm(ref, axis=-1)
    zero = rn == 0
    assert np.all(err[zero] == 0), (what, "nonzero output for an all-zero reference row")
    if not zero.all():
        rel = np.linalg.norm(err[~zero]) / np.linalg.norm(ref[~zero])
        assert rel <= TOL_REL, (what, rel)
        rows = np.linalg.norm(err, axis=-1)[~zero] / rn[~zero]
        assert rows.max() <= TOL_REL, (what, rows.max())
    # T2
    ob = out16.double().cpu().numpy()
    rb = bf16_round(ref)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(ob - rb) <= np.maximum(TOL_ABS, ulp) + 1e-12), what
    assert np.all(ob[zero] == 0), what
    if not zero.all():
        assert np.linalg.norm((ob - rb)[~zero]) / np.linalg.norm(rb[~zero]) <= TOL_REL, what


def workload(B, Hkv, G, D, n_out=8, lo=10.0, hi=20.0, name="case"):
    return configs.Workload(name, 1, B, Hkv * G, Hkv, D, 0, 0, ((4, 2),), n_outlier=n_out,
                            outlier_lo=lo, outlier_hi=hi)


def run_case(B, Hkv, G, D, layer_bits, kmode, chunks, decode_at=None, splits=(0,), wl=None, tag="case",
             paths=(kvq.KVQ_DECODE_MMA_SYNC,)):
    """Append the token sequence in `chunks` (sizes), checking the image and decode output
    against the oracle whenever the running length is in decode_at (default: the end),
    on each decode path in `paths` and each split count in `splits`."""
    L_total = sum(chunks)
    wl = wl or workload(B, Hkv, G, D, name=tag)
    nl = len(layer_bits)
    cache = kvq.Cache(nl, B, Hkv, Hkv * G, D, L_total, layer_bits, kmodes=[kmode] * nl)
    decode_at = set(decode_at or [L_total])
    for l, (bk, bv) in enumerate(layer_bits):
        K, V = inputs.layer_kv(wl, l, L_total, "cuda")
        Kb, Vb = bits16(K), bits16(V)
        L = 0
        for n in chunks:
            cache.append(l, K[:, :, L:L + n].contiguous(), V[:, :, L:L + n].contiguous())
            L += n
            if L not in decode_at:
                continue
            q = inputs.step_q(wl, l, L, "cuda")
            img_ref, out_ref = oracle.layer(Kb[:, :, :L], Vb[:, :, :L], bits16(q), G, bk, bv, kmode)
            img = cache.export_layer(l)
            assert img.shape == img_ref.shape
            if not np.array_equal(img, img_ref):
                bad = np.flatnonzero(img != img_ref)
                pytest.fail(f"{tag} layer {l} L={L}: image differs at {bad.size} bytes, first {bad[:8]}")
            for path in paths:
                kvq.kvq_set_decode_path(cache.h, path)
                for S in splits:
                    kvq.kvq_set_num_splits(cache.h, S)
                    out32 = cache.decode_attn(l, q, out_fp32=True)
                    out16 = cache.decode_attn(l, q, out_fp32=False)
                    torch.cuda.synchronize()
                    check_outputs(out32, out16, out_ref, f"{tag} layer {l} L={L} path={path} splits={S}")
            kvq.kvq_set_decode_path(cache.h, kvq.KVQ_DECODE_MMA_SYNC)
            kvq.kvq_set_num_splits(cache.h, 0)
    assert kvq.kvq_device_status(cache.h) == 0
    return cache


def test_tiny_config():
    """Tiny: 1 layer, batch 1, 2 kv / 4 q heads, D = 64, 256 prompt tokens + 1 decode
    step, K4V2 per-channel keys, 4 outlier key channels per head x15."""
    wl = configs.tiny()
    run_case(1, 2, 2, 64, [(4, 2)], 0, [256, 1], decode_at=[256, 257], splits=(0, 1, 2, 3, 7), wl=wl,
             tag="tiny")


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("L", [1, 2, 15, 16, 17, 31, 32, 33, 64, 65, 100])
def test_edge_lengths(kmode, L):
    """Ragged lengths around the 16-token halves and 32-token groups; the first half of
    the tokens arrives in one append, the rest one by one."""
    first = max(1, L // 2)
    chunks = [first] + [1] * (L - first)
    run_case(2, 2, 2, 64, [(4, 2), (2, 8)], kmode, chunks, decode_at=[first, L], splits=(0, 1, 2),
             tag=f"edge{L}")


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("bk", [2, 4, 8])
@pytest.mark.parametrize("bv", [2, 4, 8])
def test_all_bit_pairs(kmode, bk, bv):
    run_case(2, 2, 4, 128, [(bk, bv)], kmode, [90, 7], decode_at=[97], splits=(0, 2), tag=f"K{bk}V{bv}m{kmode}")


@pytest.mark.parametrize("G,kmode", [(1, 0), (2, 0), (3, 0), (4, 0), (7, 0), (8, 0), (1, 1), (2, 1), (4, 1)])
def test_gqa_groups(G, kmode):
    run_case(2, 2, G, 128, [(8, 4)], kmode, [150, 30, 20], decode_at=[150, 200], splits=(0, 3), tag=f"G{G}")


@pytest.mark.parametrize("kmode", [0, 1])
def test_many_short_units(kmode):
    """Many (batch, kv head) units with few blocks each (64 units; 3, 4 and 5 blocks per
    unit at L = 65, 97, 129, with residual tails of 1 token), automatic splits; every
    decode is done twice (fp32, bf16) on the same cache."""
    run_case(16, 4, 2, 64, [(4, 2)], kmode, [65, 32, 32], decode_at=[65, 97, 129], splits=(0,),
             tag=f"spans{kmode}")


def test_chunked_equals_bulk():
    """Incremental appends (ragged chunks) give the same bytes as the oracle's image of
    the whole sequence, which is also what one bulk append gives."""
    wl = workload(2, 2, 4, 128, name="chunked-vs-bulk")
    for kmode in (0, 1):
        chunks = [5, 27, 1, 64, 3, 100, 33, 1, 1, 65]
        c1 = run_case(2, 2, 4, 128, [(4, 2)], kmode, chunks, wl=wl, tag="chunks")
        c2 = run_case(2, 2, 4, 128, [(4, 2)], kmode, [sum(chunks)], wl=wl, tag="bulk")
        assert np.array_equal(c1.export_layer(0), c2.export_layer(0))


def test_llama_c2_shape_schedule():
    """Llama-3.1-8B attention shape (32 q / 8 kv heads, D = 128), prompt 128 then 128
    decode steps token by token (group flushes at 160, 192, 224, 256), K8V8 and K8V4;
    batch reduced to 4 to keep the oracle fast."""
    wl = configs.llama_c2((8, 4))
    wl = configs.Workload(wl.name, 2, 4, 32, 8, 128, 128, 128, ((8, 8), (8, 4)))
    run_case(4, 8, 4, 128, [(8, 8), (8, 4)], 0, [128] + [1] * 128, decode_at=[128, 129, 159, 160, 161, 256],
             splits=(0,), wl=wl, tag="c2")


@pytest.mark.slow
def test_llama_c3_full_layers():
    """Full C3 size for one K4V4 and one K4V2 layer: batch 64, 8 kv heads, context 4096
    then 32 decode steps (residual lengths 1..31 and a flush), automatic splits."""
    wl = configs.llama_c3()
    run_case(64, 8, 4, 128, [(4, 4), (4, 2)], 0, [4096] + [1] * 32, decode_at=[4097, 4128], wl=wl, tag="c3")


@pytest.mark.slow
def test_qwen_c4_full_layers():
    """Full C4 size for one K8V2 and one K4V2 layer: Qwen2.5-7B shape (28 q / 4 kv
    heads, GQA 7), batch 32, context 8192 then 32 decode steps, 16 outlier key channels
    per head x30, automatic splits."""
    wl = configs.qwen_c4()
    run_case(32, 4, 7, 128, [(8, 2), (4, 2)], 0, [8192] + [1] * 32, decode_at=[8193, 8224], wl=wl, tag="c4")
