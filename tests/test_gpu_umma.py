"""GPU parity of the tcgen05 decode path (kvq_set_decode_path(h, KVQ_DECODE_TCGEN05))
against the CPU oracle: both contractions of the per-layer decode on tcgen05.mma with
tensor-memory accumulators, for both key modes and head_dim 128 (the flash-decoding splits merged by log-sum-exp of the "TriAxialKV per-role
mixed-precision KV quantization" page, Facts: decode path), up to 8 query heads per kv
head.  The same T1/T2 bounds as the mma.sync path; layers outside the path's scope are
refused without a launch."""
import numpy as np
import pytest
import torch

import oracle
from layer_wise_mixed_b200 import configs, inputs, kvq

from test_gpu_parity import bits16, check_outputs, run_case, workload

pytestmark = pytest.mark.gpu

UMMA = (kvq.KVQ_DECODE_TCGEN05,)
BOTH = (kvq.KVQ_DECODE_MMA_SYNC, kvq.KVQ_DECODE_TCGEN05)


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("bk", [2, 4, 8])
@pytest.mark.parametrize("bv", [2, 4, 8])
def test_umma_bit_pairs(bk, bv, kmode):
    """Every precision pair and key mode: 3 full blocks and a 1-token tail, then 9 full
    blocks and a 12-token tail (three 4-block chunks, the last one partial), forced splits."""
    run_case(2, 2, 4, 128, [(bk, bv)], kmode, [97, 203], decode_at=[97, 300], splits=(0, 1, 2, 3, 5), paths=BOTH,
             tag=f"umma-K{bk}V{bv}m{kmode}")


@pytest.mark.parametrize("G,kmode", [(g, 0) for g in range(1, 9)] + [(1, 1), (2, 1), (4, 1)])
def test_umma_gqa(G, kmode):
    run_case(2, 2, G, 128, [(8, 4)], kmode, [150, 30, 20], decode_at=[150, 200], splits=(0, 3), paths=UMMA,
             tag=f"umma-G{G}m{kmode}")


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("L", [1, 2, 31, 32, 33, 64, 127, 128, 129, 131, 160, 257])
def test_umma_lengths(L, kmode):
    """Tail-only units, whole groups without a tail, 4-block chunk boundaries."""
    first = max(1, L - 3)
    run_case(2, 2, 4, 128, [(4, 2)], kmode, [first] + [1] * (L - first), decode_at=[first, L], splits=(0, 1, 2),
             paths=UMMA, tag=f"umma-L{L}m{kmode}")


def test_umma_llama_c2_schedule():
    """Llama-3.1-8B attention shape, prompt 128 then decode steps through two group
    flushes (batch 4 to keep the oracle fast), K8V4."""
    wl = configs.Workload("umma-c2", 1, 4, 32, 8, 128, 128, 64, ((8, 4),))
    run_case(4, 8, 4, 128, [(8, 4)], 0, [128] + [1] * 64, decode_at=[128, 129, 159, 160, 161, 192], splits=(0,),
             wl=wl, paths=BOTH, tag="umma-c2")


def test_umma_ragged_and_pools():
    """Per-request lengths (kvq_append_ragged) and a block-pool plan on the tcgen05 path."""
    B, Hkv, G, D, bits = 4, 2, 4, 128, (4, 2)
    wl = workload(B, Hkv, G, D, name="umma-ragged")
    for pool in (0, 40):
        cache = kvq.Cache(1, B, Hkv, Hkv * G, D, 400, [bits], kmodes=[0], pool_blocks=pool)
        K, V = inputs.layer_kv(wl, 0, 400, "cuda")
        Kb, Vb = bits16(K), bits16(V)
        counts = [37, 300, 129, 5]
        n_max = max(counts)
        Kn = torch.zeros((B, Hkv, n_max, D), dtype=torch.bfloat16, device="cuda")
        Vn = torch.zeros_like(Kn)
        for b, n in enumerate(counts):
            Kn[b, :, :n] = K[b, :, :n]
            Vn[b, :, :n] = V[b, :, :n]
        cache.append_ragged(0, Kn, Vn, counts)
        q = inputs.step_q(wl, 0, 1, "cuda")
        kvq.kvq_set_decode_path(cache.h, kvq.KVQ_DECODE_TCGEN05)
        for S in (0, 2, 5):
            kvq.kvq_set_num_splits(cache.h, S)
            out32 = cache.decode_attn(0, q, out_fp32=True)
            out16 = cache.decode_attn(0, q, out_fp32=False)
            torch.cuda.synchronize()
            for b, n in enumerate(counts):
                _, ref = oracle.layer(Kb[b:b + 1, :, :n], Vb[b:b + 1, :, :n], bits16(q[b:b + 1]), G, *bits, 0)
                check_outputs(out32[b:b + 1], out16[b:b + 1], ref, f"pool={pool} splits={S} request {b} L={n}")
        assert kvq.kvq_device_status(cache.h) == 0


EDGE = ["const", "zero_k", "zero_v", "zero_kv", "tiny", "tiny_mixed", "large", "ties", "q_big", "q_huge", "q_small"]


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("kind", EDGE)
@pytest.mark.parametrize("bits", [(4, 2), (8, 8), (2, 4)], ids=["K4V2", "K8V8", "K2V4"])
def test_umma_edge(kind, bits, kmode):
    """The quantizer's and decoder's boundary inputs (constant groups, zero tensors,
    subnormal fp16 scales, |x| near 2^14, round-half-even ties, q far outside N(0, 1))."""
    B, Hkv, G, D = 2, 2, 4, 128
    wl = workload(B, Hkv, G, D, name=f"umma-edge-{kind}")
    L = 150
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L, [bits], kmodes=[kmode])
    K, V = inputs.edge_kv(kind, wl, 0, L, "cuda", bits=bits, kmode=kmode)
    cache.append(0, K, V)
    q = inputs.edge_q(kind, wl, 0, L, "cuda", bits=bits)
    _, ref = oracle.layer(bits16(K), bits16(V), bits16(q), G, bits[0], bits[1], kmode)
    kvq.kvq_set_decode_path(cache.h, kvq.KVQ_DECODE_TCGEN05)
    for S in (0, 2):
        kvq.kvq_set_num_splits(cache.h, S)
        out32 = cache.decode_attn(0, q, out_fp32=True)
        out16 = cache.decode_attn(0, q, out_fp32=False)
        torch.cuda.synchronize()
        check_outputs(out32, out16, ref, f"{kind} K{bits[0]}V{bits[1]} m{kmode} splits={S}")
    assert kvq.kvq_device_status(cache.h) == 0


@pytest.mark.parametrize("bits", [(8, 2), (4, 2), (2, 8)], ids=["K8V2", "K4V2", "K2V8"])
def test_umma_qwen_gqa7(bits):
    """Qwen2.5-7B attention shape (28 q / 4 kv heads, GQA 7) with 16 outlier key channels
    per head x30, batch 4, context 1000 then single-token steps, forced and automatic splits,
    both paths."""
    wl = configs.Workload("umma-qwen", 1, 4, 28, 4, 128, 1000, 4, (bits,), n_outlier=16, outlier_lo=30.0,
                          outlier_hi=30.0)
    run_case(4, 4, 7, 128, [bits], 0, [1000, 1, 1, 1, 1], decode_at=[1000, 1003, 1004], splits=(0, 3), wl=wl,
             paths=BOTH, tag=f"umma-qwen-K{bits[0]}V{bits[1]}")


@pytest.mark.parametrize("kind", ["const", "zero_kv", "tiny", "large", "ties", "q_huge", "q_small"])
def test_umma_edge_g8(kind):
    """The boundary inputs at 8 query heads per kv head (the 16-row key operand)."""
    B, Hkv, G, D, bits = 2, 2, 8, 128, (4, 4)
    wl = workload(B, Hkv, G, D, name=f"umma-edge8-{kind}")
    L = 100
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, L, [bits], kmodes=[0])
    K, V = inputs.edge_kv(kind, wl, 0, L, "cuda", bits=bits, kmode=0)
    cache.append(0, K, V)
    q = inputs.edge_q(kind, wl, 0, L, "cuda", bits=bits)
    _, ref = oracle.layer(bits16(K), bits16(V), bits16(q), G, bits[0], bits[1], 0)
    kvq.kvq_set_decode_path(cache.h, kvq.KVQ_DECODE_TCGEN05)
    for S in (0, 2):
        kvq.kvq_set_num_splits(cache.h, S)
        out32 = cache.decode_attn(0, q, out_fp32=True)
        out16 = cache.decode_attn(0, q, out_fp32=False)
        torch.cuda.synchronize()
        check_outputs(out32, out16, ref, f"G=8 {kind} splits={S}")
    assert kvq.kvq_device_status(cache.h) == 0


@pytest.mark.slow
def test_umma_llama_c3_full_layer():
    """Full C3 size for a K4V2 layer: batch 64, 8 kv heads, context 4096 + 4 decode
    steps, automatic splits, both paths."""
    wl = configs.llama_c3()
    run_case(64, 8, 4, 128, [(4, 2)], 0, [4096] + [1] * 4, decode_at=[4100], wl=wl, paths=BOTH, tag="umma-c3")


@pytest.mark.parametrize("kmode", [0, 1])
def test_umma_refuses_head_dim_64(kmode):
    """head_dim 64: KVQ_EUNSUPPORTED from kvq_decode_attn on the tcgen05 path, and the
    default path still decodes."""
    G, D = 4, 64
    wl = workload(1, 2, G, D, name=f"umma-refuse-{kmode}")
    cache = kvq.Cache(1, 1, 2, 2 * G, D, 64, [(4, 4)], kmodes=[kmode])
    K, V = inputs.layer_kv(wl, 0, 40, "cuda")
    cache.append(0, K[:1].contiguous(), V[:1].contiguous())
    q = inputs.step_q(wl, 0, 40, "cuda")[:1].contiguous()
    kvq.kvq_set_decode_path(cache.h, kvq.KVQ_DECODE_TCGEN05)
    with pytest.raises(kvq.KvqError) as e:
        cache.decode_attn(0, q, out_fp32=True)
    assert e.value.code == kvq.KVQ_EUNSUPPORTED
    kvq.kvq_set_decode_path(cache.h, kvq.KVQ_DECODE_MMA_SYNC)
    out = cache.decode_attn(0, q, out_fp32=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()


def test_umma_split_count_query():
    """kvq_get_num_splits answers for the handle's decode path: forced counts on both paths,
    and on the tcgen05 path the automatic count is the one its launch uses (outputs still
    match the oracle at that count)."""
    B, Hkv, G, D, bits = 2, 2, 4, 128, (4, 2)
    wl = workload(B, Hkv, G, D, name="umma-splits")
    cache = kvq.Cache(1, B, Hkv, Hkv * G, D, 300, [bits], kmodes=[0])
    K, V = inputs.layer_kv(wl, 0, 300, "cuda")
    cache.append(0, K, V)
    q = inputs.step_q(wl, 0, 1, "cuda")
    _, ref = oracle.layer(bits16(K), bits16(V), bits16(q), G, *bits, 0)
    for path in (kvq.KVQ_DECODE_MMA_SYNC, kvq.KVQ_DECODE_TCGEN05):
        kvq.kvq_set_decode_path(cache.h, path)
        kvq.kvq_set_num_splits(cache.h, 3)
        assert kvq.kvq_get_num_splits(cache.h, 0) == 3
        kvq.kvq_set_num_splits(cache.h, 0)
        S = kvq.kvq_get_num_splits(cache.h, 0)
        assert 1 <= S <= 10
        kvq.kvq_set_num_splits(cache.h, S)
        forced = cache.decode_attn(0, q, out_fp32=True)
        kvq.kvq_set_num_splits(cache.h, 0)
        auto = cache.decode_attn(0, q, out_fp32=True)
        torch.cuda.synchronize()
        assert torch.equal(forced, auto), (path, S)   # the same split count, the same launch
        check_outputs(auto, auto.to(torch.bfloat16), ref, f"path={path} splits={S}")
    assert kvq.kvq_device_status(cache.h) == 0
