"""INT2/INT4 token mask of a paged workload from the per-tag allocation.

A seeded calibration set with the workload's shapes (2 layers, 8 requests of 512 tokens
cut into short segments, so that every tag id occurs) goes through
``kvq_tag_distortion``; ``kvq_tag_allocate`` then picks INT2 or INT4 per tag under the
workload's average bits, counting the workload's own tokens per tag; every token takes
its tag's bits.  The mask is an input of the paged cache like the Bernoulli one: the
append and decode paths and their parity do not depend on how it was chosen.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

from . import inputs, kvq
from .configs import Workload

NUM_TAGS = 56   # 4 temporal x 2 modal x 7 semantic values


def calibration(w: Workload, layers=2, requests=8, T=512):
    """(Q, K, V, tags) host arrays for kvq_tag_distortion: bf16 bits and int32 ids."""
    Q = np.stack([inputs.prefill_q(w, l, T, batch=requests, tag="calib").view(torch.int16).numpy()
                  for l in range(layers)]).view(np.uint16)
    KV = [inputs.layer_kv(w, l, T, batch=requests, tag="calib") for l in range(layers)]
    K = np.stack([kv[0].view(torch.int16).numpy() for kv in KV]).view(np.uint16)
    V = np.stack([kv[1].view(torch.int16).numpy() for kv in KV]).view(np.uint16)
    tags = inputs.tag_ids(w, T, tag="calib", batch=requests, seg=(16, 64)).numpy()
    return Q, K, V, tags


@functools.lru_cache(maxsize=8)
def tag_bits(w: Workload) -> np.ndarray:
    """INT2/INT4 per tag id: distortion from the calibration set, allocation at
    w.avg_bits over the workload's own tokens per tag (its B sequences of w.max_ctx
    tokens).  A tag the calibration set lacks counts as twice the worst measured 2-bit
    distortion, so it goes to INT2 last."""
    Q, K, V, ctags = calibration(w)
    D2, D4, ccounts = kvq.kvq_tag_distortion(Q, K, V, ctags, NUM_TAGS)
    missing = ccounts == 0
    D2[missing] = 2.0 * D2[~missing].max()
    D4[missing] = 0.0
    ids = inputs.tag_ids(w, w.max_ctx).numpy()
    counts = np.bincount(ids.ravel(), minlength=NUM_TAGS).astype(np.int64)
    bits, _ = kvq.kvq_tag_allocate(D2, D4, counts, w.avg_bits)
    return np.asarray(bits, np.uint8)


def token_mask(w: Workload, n_tokens: int, tag="prefill", batch=None) -> torch.Tensor:
    """uint8 [B, n_tokens] of 2 / 4: each token takes its tag id's allocated bits."""
    ids = inputs.tag_ids(w, n_tokens, tag=tag, batch=batch).numpy()
    return torch.from_numpy(tag_bits(w)[ids])
