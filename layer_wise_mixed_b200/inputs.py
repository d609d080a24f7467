"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module only draws random numbers: it holds none of the quantizer or attention
arithmetic.  Every tensor is a pure function of (workload name, layer, kind, step)
through ``configs.seed_of``, drawn with a torch generator on the requested device
and rounded to bf16.  A consumer that needs the same values on the CPU (the
oracle) copies the device tensor to the host; it never re-draws them.

Recipe (per layer l, kv head h):
  * K ~ N(0, 1); n_outlier channels of each (l, h), chosen by a seeded
    permutation, are multiplied by factors drawn from U[outlier_lo, outlier_hi]
    (fixed per (l, h, channel) for the whole sequence).
  * V ~ N(0, 1), Q ~ N(0, 1).
  * Tags (paged workloads): per (batch row, token) INT2 with probability
    int2_prob, else INT4, shared by all layers and heads.
  * Tag ids (per-tag allocation): each sequence is cut into segments (16-256 tokens;
    calibration sets 16-64);
    a segment's id is (temporal * 2 + modal) * 7 + semantic with temporal = the
    quarter of the sequence it starts in, modal = 1 (image) with probability 0.3 and
    semantic uniform in 0..6: 56 possible ids, of which a sequence uses some.
"""
from __future__ import annotations

import torch

from .configs import Workload, seed_of


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed_of(*parts))
    return g


def key_channel_scale(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """[Hkv, D] float32 per-channel multiplier (1 except the outlier channels)."""
    g = _gen("cpu", w.name, layer, "outliers")
    scale = torch.ones(w.n_kv_heads, w.head_dim)
    for h in range(w.n_kv_heads):
        ch = torch.randperm(w.head_dim, generator=g)[: w.n_outlier]
        f = w.outlier_lo + (w.outlier_hi - w.outlier_lo) * torch.rand(w.n_outlier, generator=g)
        scale[h, ch] = f
    return scale.to(device)


def layer_kv(w: Workload, layer: int, n_tokens: int, device="cpu", batch=None, tag="prefill"):
    """K, V bf16 [B, Hkv, n_tokens, D] for the prefill tokens of one layer."""
    B = w.batch if batch is None else batch
    g = _gen(device, w.name, layer, tag, "KV", B, n_tokens)
    shape = (B, w.n_kv_heads, n_tokens, w.head_dim)
    K = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    K.mul_(key_channel_scale(w, layer, device)[None, :, None, :])
    V = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return K.to(torch.bfloat16), V.to(torch.bfloat16)


def step_kv(w: Workload, layer: int, step: int, device="cpu", batch=None, n=1):
    """K, V bf16 [B, Hkv, n, D] for decode step ``step`` of one layer."""
    return layer_kv(w, layer, n, device, batch, tag=f"step{step}")


def step_q(w: Workload, layer: int, step: int, device="cpu", batch=None):
    """Q bf16 [B, Hq, D] for decode step ``step`` of one layer."""
    B = w.batch if batch is None else batch
    g = _gen(device, w.name, layer, f"step{step}", "Q", B)
    q = torch.randn((B, w.n_q_heads, w.head_dim), generator=g, device=device, dtype=torch.float32)
    return q.to(torch.bfloat16)


def tags(w: Workload, n_tokens: int, tag="prefill", batch=None) -> torch.Tensor:
    """uint8 [B, n_tokens]: 2 (INT2) with probability int2_prob, else 4 (INT4).
    Drawn on the CPU: tags are host-side scheduling metadata."""
    B = w.batch if batch is None else batch
    g = _gen("cpu", w.name, tag, "tags", B, n_tokens)
    u = torch.rand((B, n_tokens), generator=g)
    return torch.where(u < w.int2_prob, 2, 4).to(torch.uint8)


def prefill_q(w: Workload, layer: int, n_tokens: int, device="cpu", batch=None, tag="prefill"):
    """Q bf16 [B, Hq, n_tokens, D] for the prefill tokens of one layer (calibration)."""
    B = w.batch if batch is None else batch
    g = _gen(device, w.name, layer, tag, "Qp", B, n_tokens)
    q = torch.randn((B, w.n_q_heads, n_tokens, w.head_dim), generator=g, device=device, dtype=torch.float32)
    return q.to(torch.bfloat16)


def tag_ids(w: Workload, n_tokens: int, tag="prefill", batch=None, seg=(16, 256)) -> torch.Tensor:
    """int32 [B, n_tokens] segment tag ids in [0, 56) (recipe in the module docstring;
    segment lengths uniform in seg)."""
    B = w.batch if batch is None else batch
    g = _gen("cpu", w.name, tag, "tagids", B, n_tokens, seg[0], seg[1])
    out = torch.empty((B, n_tokens), dtype=torch.int32)
    for b in range(B):
        t = 0
        while t < n_tokens:
            n = int(torch.randint(seg[0], seg[1] + 1, (1,), generator=g))
            temporal = min(3, 4 * t // n_tokens)
            modal = int(torch.rand(1, generator=g) < 0.3)
            semantic = int(torch.randint(0, 7, (1,), generator=g))
            out[b, t:t + n] = (temporal * 2 + modal) * 7 + semantic
            t += n
    return out

