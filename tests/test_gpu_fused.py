"""GPU parity of kvq_append_decode (one-token append and decode attention in one launch)
against the CPU oracle.

Every step appends one token through the fused entry point; at the checked lengths the
exported cache image must equal the oracle's image of the same token sequence byte for
byte, and the step's fp32 output (and a bf16 decode at the same length) must meet the
T1/T2 tolerances of the parity tests.  Steps that complete a 32-token per-channel key
group take the two-launch path inside the call and are covered too.
"""
import numpy as np
import pytest
import torch

import oracle
from layer_wise_mixed_b200 import configs, inputs, kvq

from test_gpu_parity import bits16, check_outputs, workload

pytestmark = pytest.mark.gpu


def run_fused(B, Hkv, G, D, bits, kmode, prefill, steps, check_at, splits=0, wl=None, tag="fused"):
    bk, bv = bits
    L_total = prefill + steps
    wl = wl or workload(B, Hkv, G, D, name=tag)
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L_total, [bits], kmodes=[kmode])
    kvq.kvq_set_num_splits(cache.h, splits)
    K, V = inputs.layer_kv(wl, 0, L_total, "cuda")
    Kb, Vb = bits16(K), bits16(V)
    if prefill:
        cache.append(0, K[:, :, :prefill].contiguous(), V[:, :, :prefill].contiguous())
    check_at = set(check_at)
    for L in range(prefill + 1, L_total + 1):
        q = inputs.step_q(wl, 0, L, "cuda")
        out32 = cache.append_decode(0, K[:, :, L - 1:L].contiguous(), V[:, :, L - 1:L].contiguous(), q,
                                    out_fp32=True)
        assert cache.seq_len(0) == L
        if L not in check_at:
            continue
        out16 = cache.decode_attn(0, q, out_fp32=False)
        torch.cuda.synchronize()
        img_ref, out_ref = oracle.layer(Kb[:, :, :L], Vb[:, :, :L], bits16(q), G, bk, bv, kmode)
        img = cache.export_layer(0)
        if not np.array_equal(img, img_ref):
            bad = np.flatnonzero(img != img_ref)
            pytest.fail(f"{tag} L={L}: image differs at {bad.size} bytes, first {bad[:8]}")
        check_outputs(out32, out16, out_ref, f"{tag} L={L} splits={splits}")
    assert kvq.kvq_device_status(cache.h) == 0


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("splits", [0, 1, 2, 3])
def test_fused_from_empty(kmode, splits):
    """Token by token from an empty cache: first token of a half (16, 48), of a block
    (32, 64 with per-channel flushes), ragged lengths in between."""
    run_fused(2, 2, 2, 64, (4, 2), kmode, 0, 70, [1, 2, 15, 16, 17, 31, 32, 33, 48, 49, 63, 64, 65, 70],
              splits=splits, tag=f"empty{kmode}{splits}")


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("bk", [2, 4, 8])
@pytest.mark.parametrize("bv", [2, 4, 8])
def test_fused_bit_pairs(kmode, bk, bv):
    run_fused(2, 2, 4, 128, (bk, bv), kmode, 90, 40, [91, 96, 97, 112, 113, 128, 129, 130],
              tag=f"K{bk}V{bv}m{kmode}")


@pytest.mark.parametrize("G,kmode", [(1, 0), (3, 0), (7, 0), (8, 0), (1, 1), (4, 1)])
def test_fused_gqa(G, kmode):
    run_fused(2, 2, G, 128, (8, 4), kmode, 150, 20, [151, 160, 170], splits=0, tag=f"G{G}m{kmode}")


def test_fused_llama_c2_schedule():
    """Llama-3.1-8B attention shape, prompt 128 then 128 fused steps (K8V4, flushes at
    160, 192, 224, 256 through the two-launch path); batch 4 to keep the oracle fast."""
    wl = configs.Workload("fused-c2", 1, 4, 32, 8, 128, 128, 128, ((8, 4),))
    run_fused(4, 8, 4, 128, (8, 4), 0, 128, 128, [129, 144, 145, 159, 160, 161, 200, 255, 256], wl=wl, tag="c2")


def test_fused_matches_two_launches():
    """The fused step leaves the same cache bytes as kvq_append followed by
    kvq_decode_attn, and both outputs agree within the parity tolerance."""
    B, Hkv, G, D, L0, n = 3, 4, 4, 128, 100, 40
    wl = workload(B, Hkv, G, D, name="fused-vs-two")
    K, V = inputs.layer_kv(wl, 0, L0 + n, "cuda")
    a = kvq.Cache(1, B, Hkv, Hkv * G, D, L0 + n, [(4, 2)])
    b = kvq.Cache(1, B, Hkv, Hkv * G, D, L0 + n, [(4, 2)])
    for c in (a, b):
        c.append(0, K[:, :, :L0].contiguous(), V[:, :, :L0].contiguous())
    for L in range(L0 + 1, L0 + n + 1):
        q = inputs.step_q(wl, 0, L, "cuda")
        k1, v1 = K[:, :, L - 1:L].contiguous(), V[:, :, L - 1:L].contiguous()
        oa = a.append_decode(0, k1, v1, q, out_fp32=True)
        b.append(0, k1, v1)
        ob = b.decode_attn(0, q, out_fp32=True)
        torch.cuda.synchronize()
        assert np.array_equal(a.export_layer(0), b.export_layer(0)), L
        d = (oa - ob).double().abs().max().item()
        assert d <= 1e-4, (L, d)


@pytest.mark.parametrize("kmode", [0, 1])
def test_fused_in_launch_merge(kmode):
    """Five splits: the split partials are merged by the last CTA of each (b, kv head)
    inside the fused launch, step after step (the arrival counters reset themselves)."""
    run_fused(2, 2, 4, 128, (4, 2), kmode, 150, 40, [151, 160, 161, 175, 190], splits=5, tag=f"merge{kmode}")


def test_fused_c2_full_size_graphs():
    """The default bench workload at full size (Llama-3.1-8B shape, batch 64, 8 kv heads,
    GQA 4, K8V4, per-channel keys; 2 of its 32 layers), in the bench's launch
    configuration: prompt 128, then every decode step of each layer captured into a CUDA
    graph (fused append + decode; steps completing a key group take two launches inside
    the call) and replayed.  At the checked lengths the step's graph is replayed a second
    time: replays are idempotent (same image, same output)."""
    wl = configs.llama_c2((8, 4))
    B, Hkv, G, D, NL, P = wl.batch, wl.n_kv_heads, wl.G, wl.head_dim, 2, wl.prefill
    steps = 128
    cache = kvq.Cache(NL, B, Hkv, Hkv * G, D, P + steps, [(8, 4)] * NL)
    KV = [inputs.layer_kv(wl, l, P + steps, "cuda") for l in range(NL)]
    for l in range(NL):
        cache.append(l, KV[l][0][:, :, :P].contiguous(), KV[l][1][:, :, :P].contiguous())
    stream = torch.cuda.Stream()
    check = {129, 144, 159, 160, 161, 200, 255, 256}
    for L in range(P + 1, P + steps + 1):
        qs = [inputs.step_q(wl, l, L, "cuda") for l in range(NL)]
        ks = [KV[l][0][:, :, L - 1:L].contiguous() for l in range(NL)]
        vs = [KV[l][1][:, :, L - 1:L].contiguous() for l in range(NL)]
        outs = [torch.empty((B, Hkv * G, D), dtype=torch.float32, device="cuda") for _ in range(NL)]
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for l in range(NL):
                cache.append_decode(l, ks[l], vs[l], qs[l], outs[l], out_fp32=True, stream=stream.cuda_stream)
        g.replay()
        torch.cuda.synchronize()
        if L not in check:
            continue
        first = [o.clone() for o in outs]
        imgs = [cache.export_layer(l) for l in range(NL)]
        g.replay()
        torch.cuda.synchronize()
        for l in range(NL):
            assert torch.equal(first[l], outs[l]), (L, l)
            assert np.array_equal(imgs[l], cache.export_layer(l)), (L, l)
            Kb, Vb = bits16(KV[l][0][:, :, :L]), bits16(KV[l][1][:, :, :L])
            img_ref, out_ref = oracle.layer(Kb, Vb, bits16(qs[l]), G, 8, 4, 0)
            if not np.array_equal(imgs[l], img_ref):
                bad = np.flatnonzero(imgs[l] != img_ref)
                pytest.fail(f"c2 full L={L} layer {l}: image differs at {bad.size} bytes, first {bad[:8]}")
            out16 = cache.decode_attn(l, qs[l], out_fp32=False)
            torch.cuda.synchronize()
            check_outputs(outs[l], out16, out_ref, f"c2 full L={L} layer {l}")
        del g
    assert kvq.kvq_device_status(cache.h) == 0


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("bits", [(8, 4), (4, 2)], ids=["K8V4", "K4V2"])
def test_fused_split_value_scale_jump(kmode, bits):
    """Fused steps whose new value row is 2^4 to 2^11 times larger than every value before
    it, under forced splits: the CTA that appends the token takes a smaller value
    prescale than the other splits of the same (b, kv head) (it sees the new scale, they
    see the layer's old maxima), and the split merge must weigh the partials by their
    true maxima (a sum over tokens split into parts: the KVTuner summary's flash-decoding
    kernels and the TriAxialKV page's LSE merge of splits)."""
    bk, bv = bits
    B, Hkv, G, D = 2, 2, 4, 128
    prefill = 100
    wl = workload(B, Hkv, G, D, name=f"jump{kmode}{bk}{bv}")
    jumps = [(2, 5), (3, 9), (5, 12)]   # (splits, log2 of the new row's scale-up)
    L_total = prefill + len(jumps)
    K, V = inputs.layer_kv(wl, 0, L_total, "cuda")
    V = V.float()
    V[:, :, :prefill] *= 2.0                                  # value scales near 1
    for i, (_, e) in enumerate(jumps):
        V[:, :, prefill + i] *= 2.0 ** e
    V = V.to(torch.bfloat16)
    Kb, Vb = bits16(K), bits16(V)
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L_total, [bits], kmodes=[kmode])
    cache.append(0, K[:, :, :prefill].contiguous(), V[:, :, :prefill].contiguous())
    for i, (S, _) in enumerate(jumps):
        L = prefill + i + 1
        kvq.kvq_set_num_splits(cache.h, S)
        q = inputs.step_q(wl, 0, L, "cuda")
        out32 = cache.append_decode(0, K[:, :, L - 1:L].contiguous(), V[:, :, L - 1:L].contiguous(), q,
                                    out_fp32=True)
        torch.cuda.synchronize()
        img_ref, out_ref = oracle.layer(Kb[:, :, :L], Vb[:, :, :L], bits16(q), G, bk, bv, kmode)
        img = cache.export_layer(0)
        if not np.array_equal(img, img_ref):
            bad = np.flatnonzero(img != img_ref)
            pytest.fail(f"L={L}: image differs at {bad.size} bytes, first {bad[:8]}")
        check_outputs(out32, out32.to(torch.bfloat16), out_ref, f"jump splits={S} L={L}")
    assert kvq.kvq_device_status(cache.h) == 0
