"""Workload descriptions: model attention shapes, per-layer K/V precision maps and the
synthetic value distributions used by the tests and the benchmark.

The shapes are the attention shapes of the models the pages evaluate on (KVTuner
summary, Experimental setup and Measured effects table: Llama-3.1-8B-Instruct and
Qwen2.5-7B-Instruct; TriAxialKV facts: INT2/INT4 token-mixed paging, page size and
splits).  No model weights or datasets are involved: keys, values and queries are
seeded normal samples, keys with a few scaled "outlier" channels per head (the
channel-wise key outliers that motivate per-channel key quantization in the
per-layer sensitivity facts).
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import List, Tuple

PER_CHANNEL = 0
PER_TOKEN = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_layers: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    prefill: int              # tokens appended before decoding starts
    decode_steps: int         # decode steps in the full schedule
    layer_bits: Tuple[Tuple[int, int], ...]   # per-layer (bk, bv)
    kmode: int = PER_CHANNEL
    n_outlier: int = 8        # outlier key channels per (layer, kv head)
    outlier_lo: float = 10.0  # outlier multiplier range U[lo, hi]
    outlier_hi: float = 20.0
    paged: bool = False
    page_tokens: int = 16
    avg_bits: float = 0.0     # paged: average bits of the tag mask
    int2_prob: float = 0.5    # paged: probability that a token is tagged INT2
    tag_source: str = "bernoulli"   # paged: "bernoulli" mask, or "alloc" (per-tag allocation)

    @property
    def G(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def max_ctx(self) -> int:
        return self.prefill + self.decode_steps

    def equivalent_bits(self) -> float:
        """Mean of (bk + bv)/2 over layers (the pages' 'equivalent precision')."""
        return sum((bk + bv) / 2 for bk, bv in self.layer_bits) / len(self.layer_bits)


def seed_of(*parts) -> int:
    """Stable 31-bit seed from a tuple of names/ints."""
    return zlib.crc32("/".join(str(p) for p in parts).encode()) & 0x7FFFFFFF


def _seeded_layers(tag: str, n_layers: int, n_pick: int) -> List[int]:
    """n_pick distinct layer indices chosen by a seeded shuffle (pure Python)."""
    import random
    r = random.Random(seed_of("layer-map", tag))
    idx = list(range(n_layers))
    r.shuffle(idx)
    return sorted(idx[:n_pick])


def tiny() -> Workload:
    return Workload("tiny", 1, 1, 4, 2, 64, 256, 1, ((4, 2),), n_outlier=4,
                    outlier_lo=15.0, outlier_hi=15.0)


def llama_c2(bits: Tuple[int, int] = (8, 4)) -> Workload:
    """Llama-3.1-8B attention shape, batch 64, prompt 128 then 128 decode steps,
    uniform bits (K8V8 is the KIVI-8 style baseline, K8V4 the mixed pair)."""
    return Workload(f"llama8b-b64-p128-d128-K{bits[0]}V{bits[1]}", 32, 64, 32, 8, 128, 128, 128,
                    tuple([bits] * 32))


def llama_c3() -> Workload:
    """Llama-3.1-8B shape, batch 64, context 4096: 8 seeded layers K4V4 and 24 layers
    K4V2 (3.25-bit equivalent), then 32 decode steps."""
    k4v4 = set(_seeded_layers("c3", 32, 8))
    bits = tuple((4, 4) if i in k4v4 else (4, 2) for i in range(32))
    return Workload("llama8b-b64-ctx4096-map3.25", 32, 64, 32, 8, 128, 4096, 32, bits)


def qwen_c4() -> Workload:
    """Qwen2.5-7B shape (28 q / 4 kv heads, GQA 7), batch 32, context 8192:
    14 seeded layers K8V2 and 14 layers K4V2 (4.0-bit), keys with 16 outlier
    channels per head x30."""
    k8 = set(_seeded_layers("c4", 28, 14))
    bits = tuple((8, 2) if i in k8 else (4, 2) for i in range(28))
    return Workload("qwen7b-b32-ctx8192-map4.0", 28, 32, 28, 4, 128, 8192, 32, bits,
                    n_outlier=16, outlier_lo=30.0, outlier_hi=30.0)


def paged_c5() -> Workload:
    """Llama-3.1-8B shape, batch 16, context 32768, 16-token pages, INT2/INT4 per
    token from a seeded Bernoulli(0.5) mask (3-bit average)."""
    return Workload("llama8b-b16-ctx32768-paged-int2int4", 32, 16, 32, 8, 128, 32768, 17,
                    tuple([(2, 2)] * 32), paged=True, page_tokens=16, avg_bits=3.0,
                    int2_prob=0.5)


def paged_c5_alloc() -> Workload:
    """C5 with the INT2/INT4 mask from the per-tag allocation at 3.0 bits: tokens carry
    synthetic (temporal, modal, semantic) tag ids in segments; a small seeded calibration
    set of the same shape gives D_k(b); each tag's tokens take its bits."""
    return Workload("llama8b-b16-ctx32768-paged-alloc", 32, 16, 32, 8, 128, 32768, 17,
                    tuple([(2, 2)] * 32), paged=True, page_tokens=16, avg_bits=3.0,
                    tag_source="alloc")


def by_name(name: str) -> Workload:
    table = {"tiny": tiny(), "c2": llama_c2((8, 4)), "c2-k8v8": llama_c2((8, 8)),
             "c2-k8v4": llama_c2((8, 4)), "c3": llama_c3(), "c4": qwen_c4(), "c5": paged_c5(),
             "c5-alloc": paged_c5_alloc()}
    return table[name]
