"""Oracle of the per-tag bit allocation ("TriAxialKV per-role mixed-precision KV
quantization for agentic prefills", Facts: per-tag distortion, allocator, quantizer,
leftover routing).

TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``): the tests are the only
callers; the product library never imports or runs it.

Written step by step from the pages' description, in numpy fp64, with the group
quantizer of ``oracle.quant_groups`` (binary32 steps of the cache's quantizer):

- D_k(b): the tokens of tag k quantized at b bits, every other token exact; causal
  attention over the calibration prefill; mean squared output error per query head;
  max over heads, mean over requests, sum over layers.
- b = 4: K and V per token, groups of 32 channels.  b = 2: K per channel over
  consecutive 32-token groups of the tag's tokens (token order), V per token; the tag's
  last (count mod 32) tokens take the 4-bit per-token path for K and V.
- Allocation: INT2 or INT4 per tag under an average-bit budget, exhaustive for 22 tags
  or fewer, otherwise greedy by distortion added per bit saved.
"""
from __future__ import annotations

import numpy as np

from . import bf16_bits_to_f32, f16_bits_to_f64, quant_groups


def _dequant_rows(x32: np.ndarray, bits: int) -> np.ndarray:
    """Rows of 32 binary32 values -> their dequantized fp64 values."""
    s, z, c = quant_groups(x32, bits)
    return c.astype(np.float64) * f16_bits_to_f64(s)[:, None] + f16_bits_to_f64(z)[:, None]


def quantize_tag_tokens(Kf: np.ndarray, Vf: np.ndarray, toks: np.ndarray, bits: int):
    """Kf, Vf: [T, D] float32 (exact); toks: the tag's token indices in order.
    Returns fp64 copies with those tokens quantized at `bits`."""
    T, D = Kf.shape
    Kq = Kf.astype(np.float64)
    Vq = Vf.astype(np.float64)
    n = len(toks)
    full = (n // 32) * 32 if bits == 2 else 0
    for g in range(full // 32):
        rows = toks[32 * g:32 * g + 32]
        cols = Kf[rows, :].T                      # [D, 32]: one group per channel
        Kq[rows, :] = _dequant_rows(cols, 2).T
    if full:
        rows = toks[:full]
        Vq[rows, :] = _dequant_rows(Vf[rows, :].reshape(-1, 32), 2).reshape(len(rows), D)
    rest = toks[full:]
    if len(rest):
        Kq[rest, :] = _dequant_rows(Kf[rest, :].reshape(-1, 32), 4).reshape(len(rest), D)
        Vq[rest, :] = _dequant_rows(Vf[rest, :].reshape(-1, 32), 4).reshape(len(rest), D)
    return Kq, Vq


def causal_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """q, K, V: [T, D] fp64 -> softmax(q K^T / sqrt(D), causal) V, [T, D]."""
    T, D = q.shape
    s = (q @ K.T) / np.sqrt(D)
    s[np.triu_indices(T, 1)] = -np.inf
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ V) / p.sum(axis=1, keepdims=True)


def distortion(Q, K, V, tags, num_tags: int):
    """Q [NL, R, Hq, T, D], K/V [NL, R, Hkv, T, D] bf16 bits; tags [R, T].
    Returns (D2 [num_tags], D4 [num_tags], counts [num_tags])."""
    Q = np.asarray(Q, np.uint16)
    K = np.asarray(K, np.uint16)
    V = np.asarray(V, np.uint16)
    tags = np.asarray(tags)
    NL, R, Hq, T, D = Q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    counts = np.array([(tags == k).sum() for k in range(num_tags)], np.int64)
    out = {2: np.zeros(num_tags), 4: np.zeros(num_tags)}
    for k in range(num_tags):
        for bits in (2, 4):
            total = 0.0
            for l in range(NL):
                per_req = []
                for r in range(R):
                    toks = np.flatnonzero(tags[r] == k)
                    if len(toks) == 0:
                        per_req.append(0.0)
                        continue
                    worst = 0.0
                    for h in range(Hkv):
                        Kf = bf16_bits_to_f32(K[l, r, h])
                        Vf = bf16_bits_to_f32(V[l, r, h])
                        Kq, Vq = quantize_tag_tokens(Kf, Vf, toks, bits)
                        for g in range(G):
                            q = bf16_bits_to_f32(Q[l, r, h * G + g]).astype(np.float64)
                            ref = causal_attention(q, Kf.astype(np.float64), Vf.astype(np.float64))
                            got = causal_attention(q, Kq, Vq)
                            worst = max(worst, float(np.mean((got - ref) ** 2)))
                    per_req.append(worst)
                total += float(np.mean(per_req))
            out[bits][k] = total
    return out[2], out[4], counts


def allocate(D2, D4, counts, avg_bits: float):
    """bits per tag (2 or 4) and the chosen total distortion."""
    D2 = np.asarray(D2, np.float64)
    D4 = np.asarray(D4, np.float64)
    counts = np.asarray(counts, np.int64)
    K = len(counts)
    bits = np.full(K, 4, np.int64)
    present = [k for k in range(K) if counts[k] > 0]
    N = int(counts[present].sum()) if present else 0
    budget = avg_bits * N
    P = len(present)
    if P <= 22:
        # every mask at once (bit i: present tag i at INT2); sums accumulated tag by tag
        # in ascending order; the first least-distortion feasible mask
        masks = np.arange(1 << P, dtype=np.int64)
        tb = np.zeros(1 << P, np.int64)
        dist = np.zeros(1 << P, np.float64)
        for i, k in enumerate(present):
            two = ((masks >> i) & 1).astype(bool)
            tb += np.where(two, 2, 4) * int(counts[k])
            dist += np.where(two, D2[k], D4[k])
        dist[tb > budget] = np.inf
        best_mask = int(np.argmin(dist))
        for i, k in enumerate(present):
            bits[k] = 2 if (best_mask >> i) & 1 else 4
    else:
        tb = 4 * N
        while tb > budget:
            cand = [k for k in present if bits[k] == 4]
            if not cand:
                break
            rates = [(D2[k] - D4[k]) / (2.0 * counts[k]) for k in cand]
            pick = cand[int(np.argmin(rates))]   # first minimum: the lower tag index
            bits[pick] = 2
            tb -= 2 * int(counts[pick])
    total = 0.0
    for k in present:
        total += D2[k] if bits[k] == 2 else D4[k]
    return bits, total
