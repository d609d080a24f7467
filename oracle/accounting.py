"""Bit accounting for per-layer K/V precision maps (test infrastructure only).

* Equivalent precision of a map: the mean over layers of (key bits + value bits)/2
  (KVTuner summary, Key results: "3.25-bit equivalent precision"; per-layer
  sensitivity facts: a K8V2 pair is "5-bit", a K4V8 pair "6-bit").
* Storage bits per cached element of the v2 format: codes plus one fp16 scale and
  one fp16 zero per 32 elements, for keys and values alike (asymmetric groupwise
  quantizer with g = 32, TriAxialKV facts).
"""
from __future__ import annotations


def pair_bits(bk: int, bv: int) -> float:
    return (bk + bv) / 2.0


def equivalent_bits(layer_pairs) -> float:
    """layer_pairs: iterable of (bk, bv), one per layer."""
    pairs = list(layer_pairs)
    return sum(pair_bits(bk, bv) for bk, bv in pairs) / len(pairs)


def expand_map(runs) -> list:
    """[[count, [bk, bv]], ...] -> per-layer list of (bk, bv)."""
    out = []
    for count, (bk, bv) in runs:
        out += [(bk, bv)] * count
    return out


def saving_vs_8bit_pct(bits_small: float, bits_big: float) -> float:
    """Bit difference as a percentage of an 8-bit (KIVI-8) footprint."""
    return 100.0 * (bits_big - bits_small) / 8.0


def direct_saving_pct(bits_small: float, bits_big: float) -> float:
    return 100.0 * (1.0 - bits_small / bits_big)


def storage_bits(bk: int, bv: int, group: int = 32, meta_bits_per_group: int = 32) -> float:
    """Mean stored bits per K or V element: codes + (fp16 scale + fp16 zero) / group."""
    return ((bk + meta_bits_per_group / group) + (bv + meta_bits_per_group / group)) / 2.0


def reduction_vs_bf16_pct(bits: float) -> float:
    return 100.0 * (1.0 - bits / 16.0)
