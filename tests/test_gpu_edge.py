"""GPU parity on the quantizer's and the decoder's boundary cases, against the oracle.

The asymmetric group quantizer ("TriAxialKV per-role mixed-precision KV quantization",
Facts: asymmetric groupwise quantizer, group 32) computes s = fp16((max - min)/(2^b - 1)),
z = fp16(min) and code = clamp(rne((x - z)/s)).  Its boundaries are: constant groups
(s = 0, every code 0), all-zero tensors, scales and zeros below fp16's normal range,
magnitudes near fp16's limit, quotients exactly halfway between two codes (ties to
even), and queries far outside fp16's range on either side (the decoder's fp16 operand
prescales).  Each case (inputs.edge_kv / inputs.edge_q) runs through the C ABI for every
bit pair and both key modes; the exported cache must equal the oracle's image byte for
byte and the decode output must meet T1/T2 (as in test_gpu_parity):
    T1 fp32 output:  max-abs <= 1e-2 and relative L2 <= 1e-3 (whole tensor and every row);
    T2 bf16 output:  against the oracle rounded to bf16, relative L2 <= 1e-3 and
                     max-abs <= max(1e-2, one bf16 ulp of the oracle value).
The paged INT2/INT4 path and the fused one-token append + decode take the same inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from layer_wise_mixed_b200 import configs, inputs, kvq
from test_gpu_parity import bits16, check_outputs

pytestmark = pytest.mark.gpu

BITS = [(bk, bv) for bk in (2, 4, 8) for bv in (2, 4, 8)]
CHUNKS = [40, 1, 1, 23, 1, 31]   # single tokens, a bulk flush at 64, a second one at 96


def _wl(name, B, Hkv, G, D=128):
    return configs.Workload(name, 1, B, Hkv * G, Hkv, D, 0, 0, ((4, 2),))


def _check_image(cache, l, img_ref, what):
    img = cache.export_layer(l)
    assert img.shape == img_ref.shape, what
    if not np.array_equal(img, img_ref):
        bad = np.flatnonzero(img != img_ref)
        pytest.fail(f"{what}: image differs at {bad.size} bytes, first {bad[:8]}")


def _decode_check(cache, l, q, out_ref, what, splits=(0, 2)):
    for S in splits:
        kvq.kvq_set_num_splits(cache.h, S)
        out32 = cache.decode_attn(l, q, out_fp32=True)
        out16 = cache.decode_attn(l, q, out_fp32=False)
        torch.cuda.synchronize()
        check_outputs(out32, out16, out_ref, f"{what} splits={S}")
    kvq.kvq_set_num_splits(cache.h, 0)


@pytest.mark.parametrize("bits", BITS, ids=[f"K{a}V{b}" for a, b in BITS])
@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("kind", inputs.EDGE_KINDS)
def test_edge_case(kind, kmode, bits):
    """Appends in chunks (single tokens and bulk, through two key-group flushes); image
    and decode output checked at 40 and 97 tokens."""
    bk, bv = bits
    B, Hkv, G, D = 2, 2, 4, 128
    wl = _wl(f"edge-{kind}-{kmode}-K{bk}V{bv}", B, Hkv, G, D)
    L_total = sum(CHUNKS)
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L_total, [bits], kmodes=[kmode])
    K, V = inputs.edge_kv(kind, wl, 0, L_total, "cuda", bits=bits, kmode=kmode)
    Kb, Vb = bits16(K), bits16(V)
    L = 0
    for n in CHUNKS:
        cache.append(0, K[:, :, L:L + n].contiguous(), V[:, :, L:L + n].contiguous())
        L += n
        if L not in (40, L_total):
            continue
        q = inputs.edge_q(kind, wl, 0, L, "cuda", bits=bits)
        img_ref, out_ref = oracle.layer(Kb[:, :, :L], Vb[:, :, :L], bits16(q), G, bk, bv, kmode)
        _check_image(cache, 0, img_ref, f"{kind} m{kmode} K{bk}V{bv} L={L}")
        _decode_check(cache, 0, q, out_ref, f"{kind} m{kmode} K{bk}V{bv} L={L}")
    assert kvq.kvq_device_status(cache.h) == 0


@pytest.mark.parametrize("bits", [(4, 2), (8, 4), (2, 8)], ids=["K4V2", "K8V4", "K2V8"])
@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("kind", inputs.EDGE_KINDS)
def test_edge_fused(kind, kmode, bits):
    """The fused one-token append + decode launch on the same inputs, token by token
    from 30 to 70 tokens (a group completion at 64 takes the two-launch path)."""
    bk, bv = bits
    B, Hkv, G, D = 2, 2, 4, 128
    wl = _wl(f"edgef-{kind}-{kmode}-K{bk}V{bv}", B, Hkv, G, D)
    L0, L1 = 30, 70
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L1, [bits], kmodes=[kmode])
    K, V = inputs.edge_kv(kind, wl, 0, L1, "cuda", bits=bits, kmode=kmode)
    Kb, Vb = bits16(K), bits16(V)
    cache.append(0, K[:, :, :L0].contiguous(), V[:, :, :L0].contiguous())
    out32 = torch.empty((B, Hkv * G, D), dtype=torch.float32, device="cuda")
    for L in range(L0 + 1, L1 + 1):
        q = inputs.edge_q(kind, wl, 0, L, "cuda", bits=bits)
        kvq.kvq_append_decode(cache.h, 0, K[:, :, L - 1:L].contiguous(), V[:, :, L - 1:L].contiguous(), q, out32,
                              True, torch.cuda.current_stream())
        if L in (31, 32, 47, 48, 63, 64, 65, 70):
            torch.cuda.synchronize()
            img_ref, out_ref = oracle.layer(Kb[:, :, :L], Vb[:, :, :L], bits16(q), G, bk, bv, kmode)
            _check_image(cache, 0, img_ref, f"fused {kind} m{kmode} K{bk}V{bv} L={L}")
            out16 = cache.decode_attn(0, q, out_fp32=False)
            torch.cuda.synchronize()
            check_outputs(out32, out16, out_ref, f"fused {kind} m{kmode} K{bk}V{bv} L={L}")
    assert kvq.kvq_device_status(cache.h) == 0


PAGED_KINDS = [k for k in inputs.EDGE_KINDS if k != "ties"]


@pytest.mark.parametrize("kind", PAGED_KINDS)
def test_edge_paged(kind):
    """The paged INT2/INT4 path (INT2 keys per channel, INT4 keys and values per token)
    on the same edge inputs, Bernoulli(0.5) tags, bulk and single-token appends."""
    B, Hkv, G, D = 2, 2, 4, 128
    wl = _wl(f"edgep-{kind}", B, Hkv, G, D)
    chunks = [150, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 40]
    L_total = sum(chunks)
    r = np.random.default_rng(7)
    tags = np.where(r.random((B, L_total)) < 0.5, 2, 4).astype(np.uint8)
    avg = 4.0 - 2.0 * float((tags == 2).mean())
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L_total, avg_bits=avg)
    K, V = inputs.edge_kv(kind, wl, 0, L_total, "cuda", bits=(2, 2), kmode=0)
    Kb, Vb = bits16(K), bits16(V)
    dtags = torch.from_numpy(tags).cuda()
    L = 0
    for n in chunks:
        cache.append_tagged(0, K[:, :, L:L + n].contiguous(), V[:, :, L:L + n].contiguous(),
                            dtags[:, L:L + n].contiguous())
        L += n
        if L not in (150, 155, L_total):
            continue
        q = inputs.edge_q(kind, wl, 0, L, "cuda", bits=(2, 2))
        img_ref, out_ref = oracle.paged_layer(Kb[:, :, :L], Vb[:, :, :L], tags[:, :L], bits16(q), G)
        _check_image(cache, 0, img_ref, f"paged {kind} L={L}")
        _decode_check(cache, 0, q, out_ref, f"paged {kind} L={L}", splits=(0, 3))
    assert kvq.kvq_device_status(cache.h) == 0


@pytest.mark.parametrize("bits", BITS, ids=[f"K{a}V{b}" for a, b in BITS])
@pytest.mark.parametrize("kmode,G", [(0, 8), (0, 7), (1, 4)])
def test_single_token(kmode, G, bits):
    """L = 1 (one token in the cache: the residual alone for per-channel keys) with the
    largest query groups at head_dim 128, then 2 and 33 tokens; plain and constant inputs."""
    bk, bv = bits
    B, Hkv, D = 2, 2, 128
    for kind in ("plain", "const"):
        wl = _wl(f"one-{kind}-{kmode}-{G}-K{bk}V{bv}", B, Hkv, G, D)
        cache = kvq.Cache(1, B, Hkv, Hkv * G, D, 33, [bits], kmodes=[kmode])
        if kind == "plain":
            K, V = inputs.layer_kv(wl, 0, 33, "cuda")
        else:
            K, V = inputs.edge_kv("const", wl, 0, 33, "cuda", bits=bits, kmode=kmode)
        Kb, Vb = bits16(K), bits16(V)
        L = 0
        for n in (1, 1, 31):
            cache.append(0, K[:, :, L:L + n].contiguous(), V[:, :, L:L + n].contiguous())
            L += n
            q = inputs.step_q(wl, 0, L, "cuda")
            img_ref, out_ref = oracle.layer(Kb[:, :, :L], Vb[:, :, :L], bits16(q), G, bk, bv, kmode)
            _check_image(cache, 0, img_ref, f"one {kind} m{kmode} G{G} K{bk}V{bv} L={L}")
            _decode_check(cache, 0, q, out_ref, f"one {kind} m{kmode} G{G} K{bk}V{bv} L={L}", splits=(0, 1))
        assert kvq.kvq_device_status(cache.h) == 0
