"""GPU parity of ragged batches (sequences of different lengths in one per-layer plan)
against the CPU oracle, request by request: kvq_append_ragged (per-request token
counts, zero included), decode over each sequence's own tokens (automatic and forced
splits, the in-launch merge among them), fused one-token steps on ragged lengths (and
the two-launch path when some sequence completes a per-channel key group), per-request
export, truncation back to equal lengths."""
import numpy as np
import pytest
import torch

import oracle
from layer_wise_mixed_b200 import inputs, kvq

from test_gpu_parity import bits16, check_outputs, workload

pytestmark = pytest.mark.gpu


class Ragged:
    """A per-layer plan of one layer and the token streams of its B sequences."""

    def __init__(self, B, Hkv, G, D, bits, kmode, max_ctx, tag):
        self.B, self.Hkv, self.G, self.D, self.bits, self.kmode = B, Hkv, G, D, bits, kmode
        self.wl = workload(B, Hkv, G, D, name=tag)
        self.cache = kvq.Cache(1, B, Hkv, Hkv * G, D, max_ctx, [bits], kmodes=[kmode])
        self.K, self.V = inputs.layer_kv(self.wl, 0, max_ctx, "cuda")   # sequence b = row b
        self.Kb, self.Vb = bits16(self.K), bits16(self.V)
        self.L = [0] * B

    def append(self, counts):
        n_max = max(max(counts), 1)
        Kn = torch.zeros((self.B, self.Hkv, n_max, self.D), dtype=torch.bfloat16, device="cuda")
        Vn = torch.zeros_like(Kn)
        for b, n in enumerate(counts):
            Kn[b, :, :n] = self.K[b, :, self.L[b]:self.L[b] + n]
            Vn[b, :, :n] = self.V[b, :, self.L[b]:self.L[b] + n]
        self.cache.append_ragged(0, Kn, Vn, counts)
        self.L = [L + n for L, n in zip(self.L, counts)]
        assert list(self.cache.seq_lens(0)) == self.L

    def fused(self, step):
        b_idx = torch.arange(self.B, device="cuda")
        pos = torch.tensor(self.L, device="cuda")
        Kn = self.K[b_idx, :, pos].unsqueeze(2).contiguous()   # [B, Hkv, 1, D]
        Vn = self.V[b_idx, :, pos].unsqueeze(2).contiguous()
        q = inputs.step_q(self.wl, 0, 1000 + step, "cuda")
        out32 = self.cache.append_decode(0, Kn, Vn, q, out_fp32=True)
        self.L = [L + 1 for L in self.L]
        return q, out32

    def check(self, q, out32=None, splits=(0,), what=""):
        bk, bv = self.bits
        imgs, refs = [], []
        for b in range(self.B):
            img, ref = oracle.layer(self.Kb[b:b + 1, :, :self.L[b]], self.Vb[b:b + 1, :, :self.L[b]],
                                    bits16(q[b:b + 1]), self.G, bk, bv, self.kmode)
            imgs.append(img)
            refs.append(ref)
        img = self.cache.export_layer(0)
        ref_img = np.concatenate(imgs)
        if not np.array_equal(img, ref_img):
            bad = np.flatnonzero(img != ref_img) if img.shape == ref_img.shape else []
            pytest.fail(f"{what} L={self.L}: image differs ({img.shape} vs {ref_img.shape}), first {bad[:8]}")
        outs = [] if out32 is None else [("fused", out32, None)]
        for S in splits:
            kvq.kvq_set_num_splits(self.cache.h, S)
            o32 = self.cache.decode_attn(0, q, out_fp32=True)
            o16 = self.cache.decode_attn(0, q, out_fp32=False)
            outs.append((f"splits={S}", o32, o16))
        kvq.kvq_set_num_splits(self.cache.h, 0)
        torch.cuda.synchronize()
        for tag, o32, o16 in outs:
            for b in range(self.B):
                o16b = o16[b:b + 1] if o16 is not None else o32[b:b + 1].to(torch.bfloat16)
                check_outputs(o32[b:b + 1], o16b, refs[b], f"{what} {tag} request {b} L={self.L[b]}")
        assert kvq.kvq_device_status(self.cache.h) == 0


@pytest.mark.parametrize("kmode", [0, 1])
@pytest.mark.parametrize("bits", [(4, 2), (8, 4), (2, 8)])
def test_ragged_appends_and_decode(kmode, bits):
    r = Ragged(4, 2, 4, 128, bits, kmode, 400, f"ragged{kmode}{bits[0]}{bits[1]}")
    r.append([37, 100, 64, 5])
    r.check(inputs.step_q(r.wl, 0, 1, "cuda"), splits=(0, 2, 5), what="prompts")
    r.append([0, 3, 1, 27])                     # one request appends nothing
    r.append([31, 0, 32, 2])                    # group completions in some requests only
    r.check(inputs.step_q(r.wl, 0, 2, "cuda"), splits=(0, 3, 5), what="appends")


@pytest.mark.parametrize("kmode", [0, 1])
def test_ragged_fused_steps(kmode):
    """One-token fused steps on ragged lengths; lengths 31/63 make some request complete a
    key group at the next step (two-launch path for per-channel keys)."""
    r = Ragged(3, 2, 4, 128, (4, 2), kmode, 300, f"ragfused{kmode}")
    r.append([29, 61, 100])
    for step in range(1, 8):
        q, out32 = r.fused(step)
        if step in (1, 2, 3, 4, 7):
            r.check(q, out32, splits=(0, 4), what=f"fused step {step}")


def test_ragged_truncate_and_equal_again():
    """Truncation cuts every sequence to the same length; appends then take the uniform
    path and the results still match the oracle."""
    r = Ragged(3, 2, 2, 64, (4, 4), 0, 300, "ragtrunc")
    r.append([70, 45, 96])
    kvq.kvq_truncate(r.cache.h, 0, 32)
    r.L = [32] * 3
    assert list(r.cache.seq_lens(0)) == r.L
    r.append([20, 20, 20])
    r.check(inputs.step_q(r.wl, 0, 3, "cuda"), splits=(0, 2), what="truncated")
    with pytest.raises(kvq.KvqError):
        kvq.kvq_truncate(r.cache.h, 0, 64)      # longer than the sequences


@pytest.mark.parametrize("splits", [1, 3, 5])
def test_ragged_noalloc_matches_workspace_entry(splits):
    """The entry point without caller scratch gives the same bytes on a ragged layer."""
    r = Ragged(4, 2, 4, 128, (8, 4), 0, 400, f"ragnoalloc{splits}")
    r.append([130, 33, 200, 1])
    kvq.kvq_set_num_splits(r.cache.h, splits)
    q = inputs.step_q(r.wl, 0, 9, "cuda")
    a = r.cache.decode_attn(0, q, out_fp32=True)
    b = torch.empty_like(a)
    kvq.kvq_decode_attn_noalloc(r.cache.h, 0, q, b, True)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    r.check(q, splits=(splits,), what="noalloc")


@pytest.mark.parametrize("kmode", [0, 1])
def test_ragged_batch_96(kmode):
    """96 requests of different lengths (above the 64 whose lengths fit the kernel
    parameters: the lengths go through the layer's device table): ragged appends with
    zero counts and group completions, decode with automatic and forced splits, fused
    one-token steps (and the two-launch path), the entry point without caller scratch."""
    B = 96
    r = Ragged(B, 2, 4, 128, (4, 2), kmode, 260, f"ragged96-{kmode}")
    rng = np.random.default_rng(96 + kmode)
    r.append([int(x) for x in rng.integers(1, 160, B)])
    r.check(inputs.step_q(r.wl, 0, 1, "cuda"), splits=(0, 3, 5), what="b96 prompts")
    counts = [int(x) for x in rng.integers(0, 40, B)]
    counts[0] = 0
    r.append(counts)
    r.check(inputs.step_q(r.wl, 0, 2, "cuda"), splits=(0, 4), what="b96 appends")
    for step in range(1, 4):
        q, out32 = r.fused(step)
        r.check(q, out32, splits=(0,), what=f"b96 fused {step}")
    q = inputs.step_q(r.wl, 0, 7, "cuda")
    kvq.kvq_set_num_splits(r.cache.h, 3)
    a = r.cache.decode_attn(0, q, out_fp32=True)
    b = torch.empty_like(a)
    kvq.kvq_decode_attn_noalloc(r.cache.h, 0, q, b, True)
    kvq.kvq_set_num_splits(r.cache.h, 0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
