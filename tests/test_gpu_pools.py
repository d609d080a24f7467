"""GPU parity of per-layer plans with block pools (desc.pool_blocks > 0), request by
request against the CPU oracle.

Each layer's 32-token records come from a pool shared by all sequences and are assigned
through a block table as sequences grow; kvq_truncate and kvq_reset_sequences return
blocks to the pool.  The exported image gathers each sequence's blocks in order, so it
must equal the oracle's image of that sequence's token stream byte for byte, and decode
must meet T1/T2 on every request (the "TriAxialKV per-role mixed-precision KV
quantization" page's paged pools sharing one address space, applied to the per-layer
records; splits merged by log-sum-exp as in its Facts on the decode path).
"""
import numpy as np
import pytest
import torch

import oracle
from layer_wise_mixed_b200 import inputs, kvq

from test_gpu_parity import bits16, check_outputs, workload

pytestmark = pytest.mark.gpu


class Pooled:
    """One layer of a block-pool plan and a token stream per sequence slot; a reset slot
    starts a new stream (a new request) at an offset into the pre-drawn tokens."""

    def __init__(self, B, Hkv, G, D, bits, kmode, max_ctx, pool_blocks, tag, nl=1):
        self.B, self.Hkv, self.G, self.D, self.bits, self.kmode, self.nl = B, Hkv, G, D, bits, kmode, nl
        self.wl = workload(B, Hkv, G, D, name=tag)
        self.cache = kvq.Cache(nl, B, Hkv, Hkv * G, D, max_ctx, [bits] * nl, kmodes=[kmode] * nl,
                               pool_blocks=pool_blocks)
        self.K, self.V = inputs.layer_kv(self.wl, 0, 2 * max_ctx, "cuda")   # streams drawn once
        self.Kb, self.Vb = bits16(self.K), bits16(self.V)
        self.start = [0] * B    # offset of each slot's current stream in the drawn tokens
        self.L = [0] * B

    def append(self, counts):
        n_max = max(max(counts), 1)
        Kn = torch.zeros((self.B, self.Hkv, n_max, self.D), dtype=torch.bfloat16, device="cuda")
        Vn = torch.zeros_like(Kn)
        for b, n in enumerate(counts):
            s = self.start[b] + self.L[b]
            Kn[b, :, :n] = self.K[b, :, s:s + n]
            Vn[b, :, :n] = self.V[b, :, s:s + n]
        for l in range(self.nl):
            self.cache.append_ragged(l, Kn, Vn, counts)
        self.L = [L + n for L, n in zip(self.L, counts)]
        assert list(self.cache.seq_lens(0)) == self.L

    def fused(self, step):
        Kn = torch.stack([self.K[b, :, self.start[b] + self.L[b]] for b in range(self.B)]).unsqueeze(2).contiguous()
        Vn = torch.stack([self.V[b, :, self.start[b] + self.L[b]] for b in range(self.B)]).unsqueeze(2).contiguous()
        q = inputs.step_q(self.wl, 0, 2000 + step, "cuda")
        out32 = self.cache.append_decode(0, Kn, Vn, q, out_fp32=True)
        for l in range(1, self.nl):
            self.cache.append_decode(l, Kn, Vn, q, out_fp32=True)
        self.L = [L + 1 for L in self.L]
        return q, out32

    def reset(self, seqs, new_start):
        kvq.kvq_reset_sequences(self.cache.h, seqs)
        for b in seqs:
            self.L[b] = 0
            self.start[b] = new_start

    def check(self, q, out32=None, splits=(0,), what="", layer=0):
        bk, bv = self.bits
        imgs, refs = [], []
        for b in range(self.B):
            s0 = self.start[b]
            img, ref = oracle.layer(self.Kb[b:b + 1, :, s0:s0 + self.L[b]], self.Vb[b:b + 1, :, s0:s0 + self.L[b]],
                                    bits16(q[b:b + 1]), self.G, bk, bv, self.kmode)
            imgs.append(img)
            refs.append(ref)
        img = self.cache.export_layer(layer)
        ref_img = np.concatenate(imgs)
        if not np.array_equal(img, ref_img):
            bad = np.flatnonzero(img != ref_img) if img.shape == ref_img.shape else []
            pytest.fail(f"{what} L={self.L}: image differs ({img.shape} vs {ref_img.shape}), first {bad[:8]}")
        outs = [] if out32 is None else [("fused", out32, None)]
        for S in splits:
            kvq.kvq_set_num_splits(self.cache.h, S)
            o32 = self.cache.decode_attn(layer, q, out_fp32=True)
            o16 = self.cache.decode_attn(layer, q, out_fp32=False)
            outs.append((f"splits={S}", o32, o16))
        kvq.kvq_set_num_splits(self.cache.h, 0)
        torch.cuda.synchronize()
        for tag, o32, o16 in outs:
            for b in range(self.B):
                o16b = o16[b:b + 1] if o16 is not None else o32[b:b + 1].to(torch.bfloat16)
                check_outputs(o32[b:b + 1], o16b, refs[b], f"{what} {tag} request {b} L={self.L[b]}")
        assert kvq.kvq_device_status(self.cache.h) == 0


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("bits", [(4, 2), (8, 4)])
def test_pools_ragged_and_fused(kmode, bits):
    """Ragged prompts, appends with zero counts, fused steps through block boundaries and
    a two-launch group completion, forced splits; the pool holds fewer blocks than the
    slabs would reserve (4 sequences x 13 blocks = 52; pool 30)."""
    r = Pooled(4, 2, 4, 128, bits, kmode, 400, 30, f"pool{kmode}{bits[0]}{bits[1]}")
    r.append([37, 150, 64, 5])
    r.check(inputs.step_q(r.wl, 0, 1, "cuda"), splits=(0, 2, 5), what="prompts")
    r.append([0, 3, 31, 27])
    r.check(inputs.step_q(r.wl, 0, 2, "cuda"), splits=(0, 3), what="appends")
    for step in range(1, 6):
        q, out32 = r.fused(step)
        if step in (1, 2, 5):
            r.check(q, out32, splits=(0,), what=f"fused {step}")


def test_pools_reset_reuse():
    """Continuous batching: a sequence leaves (kvq_reset_sequences) and a new request
    takes its slot and its freed blocks; an append the pool cannot hold is refused before
    any launch and leaves every length unchanged; truncation returns blocks too."""
    r = Pooled(3, 2, 2, 64, (4, 4), 0, 300, 12, "poolreuse", nl=2)
    r.append([100, 150, 40])                     # 4 + 5 + 2 = 11 of 12 blocks
    r.check(inputs.step_q(r.wl, 0, 1, "cuda"), splits=(0, 2), what="full pool")
    with pytest.raises(kvq.KvqError) as e:       # lengths 100, 210, 70 need 3 more blocks, 1 is free
        r.cache.append_ragged(0, torch.zeros((3, 2, 64, 64), dtype=torch.bfloat16, device="cuda"),
                              torch.zeros((3, 2, 64, 64), dtype=torch.bfloat16, device="cuda"), [0, 60, 30])
    assert e.value.code == kvq.KVQ_ECAPACITY
    assert list(r.cache.seq_lens(0)) == r.L
    r.reset([1], new_start=300)                  # request 1 leaves: its 5 blocks return
    r.append([0, 70, 0])                          # a new request in slot 1 (3 blocks)
    r.append([20, 0, 10])
    r.check(inputs.step_q(r.wl, 0, 2, "cuda"), splits=(0, 3), what="reused slot", layer=0)
    r.check(inputs.step_q(r.wl, 1, 2, "cuda"), splits=(0,), what="reused slot layer 1", layer=1)
    for step in range(1, 4):
        q, out32 = r.fused(step)
    r.check(q, out32, splits=(0,), what="fused after reuse")
    for l in range(2):
        kvq.kvq_truncate(r.cache.h, l, 32)       # keeps one block per sequence: 9 free
    r.L = [32] * 3
    r.append([60, 60, 60])                       # 3 blocks each: fits only with the freed blocks
    r.check(inputs.step_q(r.wl, 0, 3, "cuda"), splits=(0,), what="after truncation")


def test_pools_batch_96():
    """96 sequences (lengths through the device tables) in a pool of 60% of the slab
    capacity, with resets and fused steps."""
    B = 96
    r = Pooled(B, 2, 4, 128, (4, 2), 0, 200, int(B * 7 * 0.6), "pool96")
    rng = np.random.default_rng(5)
    r.append([int(x) for x in rng.integers(1, 120, B)])
    r.check(inputs.step_q(r.wl, 0, 1, "cuda"), splits=(0, 3), what="b96 prompts")
    r.reset(list(range(0, B, 3)), new_start=200)
    counts = [int(x) for x in rng.integers(1, 60, B)]
    r.append(counts)
    r.check(inputs.step_q(r.wl, 0, 2, "cuda"), splits=(0,), what="b96 after resets")
    q, out32 = r.fused(1)
    r.check(q, out32, splits=(0,), what="b96 fused")
