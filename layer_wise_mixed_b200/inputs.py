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



# ---------------------------------------------------------------- structured edge cases
# Inputs with the structure of the quantizer's and the decoder's boundary cases.  They
# are built from seeded draws, constants, powers of two and half-integers; nothing here
# computes a scale, a code or an attention value.
EDGE_KINDS = ("const", "zero_k", "zero_v", "zero_kv", "tiny", "tiny_mixed", "large", "ties", "q_big", "q_huge",
              "q_small")


def _tile_const(x: torch.Tensor, g: torch.Generator, frac: float = 0.5) -> torch.Tensor:
    """Set a seeded fraction of the 32-token x 32-channel tiles of x [B, H, L, D] to one
    seeded constant each (so those tiles' 32-token channel groups and 32-channel token
    groups are constant)."""
    B, H, L, D = x.shape
    nt, nc = (L + 31) // 32, D // 32
    pick = torch.rand((B, H, nt, nc), generator=g, device=x.device) < frac
    val = torch.randn((B, H, nt, nc), generator=g, device=x.device)
    full = pick.repeat_interleave(32, 2)[:, :, :L].repeat_interleave(32, 3)
    cval = val.repeat_interleave(32, 2)[:, :, :L].repeat_interleave(32, 3)
    return torch.where(full, cval, x)


def _half_grid(bits: int, device) -> torch.Tensor:
    """Multiples of 1/2 in [0, 2^bits - 1] that bf16 holds exactly."""
    c = torch.arange(0, 2 * (2 ** bits - 1) + 1, device=device, dtype=torch.float32) / 2
    return c[c.to(torch.bfloat16).float() == c]


def _grid_groups(shape, axis: int, bits: int, g: torch.Generator, device) -> torch.Tensor:
    """Values on the half-integer grid of [0, 2^bits - 1] with, in every group of 32
    along `axis` (tokens: 2, channels: 3), one element at 0 and one at 2^bits - 1 at
    seeded positions; the other elements mostly halfway between two integers."""
    grid = _half_grid(bits, device)
    halves = grid[(grid * 2) % 2 == 1]
    x = torch.empty(shape, device=device, dtype=torch.float32)
    u = torch.rand(shape, generator=g, device=device)
    ih = torch.randint(0, halves.numel(), shape, generator=g, device=device)
    ig = torch.randint(0, grid.numel(), shape, generator=g, device=device)
    x = torch.where(u < 0.75, halves[ih], grid[ig])
    n = shape[axis]
    xm = x.movedim(axis, -1)
    for g0 in range(0, n, 32):
        w = min(32, n - g0)
        if w < 2:
            continue
        p = torch.randperm(w, generator=g, device=device)[:2].tolist()
        xm[..., g0 + p[0]] = 0.0
        xm[..., g0 + p[1]] = float(2 ** bits - 1)
    return xm.movedim(-1, axis).contiguous()


def edge_kv(kind: str, w: Workload, layer: int, n_tokens: int, device="cpu", bits=(4, 2), kmode=0):
    """K, V bf16 [B, Hkv, n_tokens, D] for one edge case (kinds in EDGE_KINDS):
      const      seeded half of the 32x32 (token, channel) tiles constant, the rest as layer_kv
      zero_k / zero_v / zero_kv   keys, values or both all zero, the rest as layer_kv
      tiny       K, V as layer_kv times 2^-20 (fp16 scales and zeros below the normal range)
      tiny_mixed half of each head's channels times 2^-18, the others as layer_kv
      large      K, V uniform in (-2^14, 2^14)
      ties       half-integer grids: per group (keys along the key mode's axis, values per
                 token) one element at 0 and one at 2^b - 1, most others at k + 1/2
      q_big      K as layer_kv times 2^-17 (with edge_q: q times 2^17)
      q_huge     K as layer_kv times 2^-40 (q times 2^40)
      q_small    K as layer_kv times 2^13 / 20, clipped below 2^15 (q times 2^-20)"""
    K, V = layer_kv(w, layer, n_tokens, device, tag=f"edge-{kind}")
    K, V = K.float(), V.float()
    B = K.shape[0]
    g = _gen(device, w.name, layer, "edge", kind, B, n_tokens)
    if kind == "const":
        K, V = _tile_const(K, g), _tile_const(V, g)
    elif kind in ("zero_k", "zero_kv"):
        K = torch.zeros_like(K)
    if kind in ("zero_v", "zero_kv"):
        V = torch.zeros_like(V)
    if kind == "tiny":
        K, V = K * 2.0 ** -20, V * 2.0 ** -20
    elif kind == "tiny_mixed":
        sel = (torch.rand((1, K.shape[1], 1, K.shape[3]), generator=g, device=device) < 0.5).float()
        K = K * (sel * 2.0 ** -18 + (1 - sel))
        V = V * (sel * 2.0 ** -18 + (1 - sel))
    elif kind == "large":
        K = (torch.rand(K.shape, generator=g, device=device) * 2 - 1) * 2.0 ** 14
        V = (torch.rand(V.shape, generator=g, device=device) * 2 - 1) * 2.0 ** 14
    elif kind == "ties":
        bk, bv = bits
        K = _grid_groups(tuple(K.shape), 2 if kmode == 0 else 3, bk, g, device)
        V = _grid_groups(tuple(V.shape), 3, bv, g, device)
    elif kind == "q_big":
        K = K * 2.0 ** -17
    elif kind == "q_huge":
        K = K * 2.0 ** -40
    elif kind == "q_small":
        K = (K * 2.0 ** 13 / 20).clamp(-(2.0 ** 15 - 256), 2.0 ** 15 - 256)
    return K.to(torch.bfloat16), V.to(torch.bfloat16)


def edge_q(kind: str, w: Workload, layer: int, step: int, device="cpu", bits=(4, 2)):
    """Q bf16 [B, Hq, D] for an edge case: step_q times a power of two that keeps the
    scores of the matching edge_kv keys of order one (q_big 2^17, q_huge 2^40, q_small
    2^-20, tiny 2^20, large 2^-14, ties 2^-bk)."""
    q = step_q(w, layer, step, device).float()
    e = {"q_big": 17, "q_huge": 40, "q_small": -20, "tiny": 20, "large": -14, "ties": -bits[0]}.get(kind, 0)
    return (q * 2.0 ** e).to(torch.bfloat16)
