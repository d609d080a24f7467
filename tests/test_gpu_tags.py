"""GPU per-tag distortion (kvq_tag_distortion_device) against the oracle and the host
entry point ("TriAxialKV per-role mixed-precision KV quantization for agentic prefills",
Facts: per-tag distortion D_k(b), quantizer, leftover routing, INT2/INT4 allocator).

Both sides compute in fp64, so the bound is the order of the sums: relative 1e-9.  The
allocations chosen from the two are identical, tags without tokens give 0 exactly, and
tags whose tokens quantize exactly give 0 exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import tags as otags
from layer_wise_mixed_b200 import kvq

from test_tags import bf16, calib, levels

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def device_distortion(Q, K, V, tags, num_tags):
    return kvq.kvq_tag_distortion_device(dev(Q), dev(K), dev(V), tags, num_tags)


def close(a, b):
    return np.allclose(a, b, rtol=1e-9, atol=1e-15)


@pytest.mark.parametrize("G,D,T", [(1, 64, 80), (2, 64, 80), (4, 128, 100), (7, 128, 33)])
def test_device_distortion_matches_oracle(G, D, T):
    rng = np.random.default_rng(40 + G + T)
    NL, R, Hkv = 2, 2, 2 if G < 7 else 1
    Q, K, V = calib(rng, NL, R, Hkv * G, Hkv, T, D)
    p = np.array([0.55, 0.2, 0.15, 0.1, 0.0])   # tag 0 fills 2-bit key groups; tag 4 absent
    tags = rng.choice(5, size=(R, T), p=p).astype(np.int32)
    D2o, D4o, co = otags.distortion(Q, K, V, tags, 5)
    D2g, D4g, cg = device_distortion(Q, K, V, tags, 5)
    assert np.array_equal(co, cg)
    assert close(D2g, D2o) and close(D4g, D4o)
    assert D2g[4] == D4g[4] == 0.0
    assert D2g[0] > 0 and D4g[0] > 0
    for avg in (2.5, 3.0, 3.5):
        assert np.array_equal(otags.allocate(D2o, D4o, co, avg)[0], kvq.kvq_tag_allocate(D2g, D4g, cg, avg)[0])


def test_device_distortion_single_token_closed_form():
    """T = 1: the output is the value row, so D_k(b) is the value quantization MSE at 4
    bits for both b (one token never fills a 2-bit key group)."""
    rng = np.random.default_rng(5)
    Q, K, V = calib(rng, 1, 1, 2, 1, 1, 64)
    tags = np.array([[1]], np.int32)
    D2, D4, counts = device_distortion(Q, K, V, tags, 3)
    v = oracle.bf16_bits_to_f32(V[0, 0, 0]).reshape(-1, 32)
    s, z, c = oracle.quant_groups(v, 4)
    vh = c * oracle.f16_bits_to_f64(s)[:, None] + oracle.f16_bits_to_f64(z)[:, None]
    mse = np.mean((vh - v.astype(np.float64)) ** 2)
    assert D2[1] == pytest.approx(mse, rel=1e-12) and D4[1] == pytest.approx(mse, rel=1e-12)
    assert D2[0] == D2[2] == D4[0] == D4[2] == 0.0
    assert list(counts) == [0, 1, 0]


def test_device_distortion_zero_on_exact_levels():
    """Levels 0..3 (0 and 3 in every group) are exact at 2 bits, 0..15 at 4 bits: the
    quantized terms equal the exact ones and the distortion is 0 exactly."""
    rng = np.random.default_rng(9)
    T, D = 64, 128
    Q, _, _ = calib(rng, 1, 1, 2, 1, T, D)
    tags = np.ones((1, T), np.int32)
    Kc = levels(rng, (D, T), 3).T.copy()
    V3 = levels(rng, (T, D), 3)
    D2, _, _ = device_distortion(Q, bf16(Kc)[None, None, None], bf16(V3)[None, None, None], tags, 2)
    assert D2[1] == 0.0
    K15, V15 = levels(rng, (T, D), 15), levels(rng, (T, D), 15)
    _, D4, _ = device_distortion(Q, bf16(K15)[None, None, None], bf16(V15)[None, None, None], tags, 2)
    assert D4[1] == 0.0


def test_device_distortion_matches_host_many_tags():
    """20 tags in segments (some with two or more 2-bit key groups, some with a few tokens),
    query blocks that end inside the sequence, GQA 4 at head_dim 128: device against the
    host entry point."""
    rng = np.random.default_rng(77)
    NL, R, Hkv, G, T, D = 1, 2, 2, 4, 333, 128
    Q, K, V = calib(rng, NL, R, Hkv * G, Hkv, T, D)
    tags = np.zeros((R, T), np.int32)
    for r in range(R):
        t = 0
        while t < T:
            n = int(rng.integers(3, 90))
            tags[r, t:t + n] = rng.integers(0, 20)
            t += n
    D2h, D4h, ch = kvq.kvq_tag_distortion(Q, K, V, tags, 20)
    D2g, D4g, cg = device_distortion(Q, K, V, tags, 20)
    assert np.array_equal(ch, cg)
    assert close(D2g, D2h) and close(D4g, D4h)
    for avg in (2.4, 3.0, 3.6):
        assert np.array_equal(kvq.kvq_tag_allocate(D2h, D4h, ch, avg)[0], kvq.kvq_tag_allocate(D2g, D4g, cg, avg)[0])


def test_device_distortion_workspace_and_stream():
    """A caller workspace (one size for every call at these shapes) and a side stream give
    the same results as the binding's own workspace; a too-small workspace is refused
    before any device work."""
    rng = np.random.default_rng(3)
    Q, K, V = calib(rng, 1, 1, 4, 2, 50, 64)
    tags = rng.integers(0, 3, size=(1, 50)).astype(np.int32)
    ref = device_distortion(Q, K, V, tags, 3)
    need = kvq.kvq_tag_distortion_workspace_bytes(1, 1, 4, 2, 64, 50, 3)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())   # the inputs' copies
    got = kvq.kvq_tag_distortion_device(Qd, Kd, Vd, tags, 3, workspace=ws, stream=st)
    for a, b in zip(ref, got):
        assert np.array_equal(a, b)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_tag_distortion_device(dev(Q), dev(K), dev(V), tags, 3, workspace=ws[: need - 256])
