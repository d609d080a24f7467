"""Per-tag bit allocation (TriAxialKV per-role page, Facts: per-tag distortion D_k(b),
INT2/INT4 allocator under an average-bit budget).  CPU only: the oracle is pinned to
brute force, closed forms and exactly representable inputs; the library's host entry
points (kvq_tag_distortion, kvq_tag_allocate) must then match the oracle."""
import numpy as np
import pytest

import oracle
from oracle import tags as otags
from layer_wise_mixed_b200 import kvq


def brute_force(D2, D4, counts, avg_bits):
    """Every INT2/INT4 choice of the present tags, in ascending mask order; the first of
    least total distortion (summed in ascending tag order) within the budget."""
    present = [k for k in range(len(counts)) if counts[k] > 0]
    N = sum(counts[k] for k in present)
    best, best_bits = None, None
    for mask in range(1 << len(present)):
        bits = [4] * len(counts)
        for i, k in enumerate(present):
            if (mask >> i) & 1:
                bits[k] = 2
        if sum(counts[k] * bits[k] for k in present) > avg_bits * N:
            continue
        dist = 0.0
        for k in present:
            dist += D2[k] if bits[k] == 2 else D4[k]
        if best is None or dist < best:
            best, best_bits = dist, bits
    return best_bits, best


def random_case(rng, K):
    D4 = rng.uniform(0.0, 1.0, K)
    D2 = D4 + rng.uniform(-0.2, 2.0, K)        # sometimes INT2 is better (non-monotonic MSE)
    counts = rng.integers(0, 50, K)
    counts[rng.integers(0, K)] = 0              # a tag that never occurs
    return D2, D4, counts


@pytest.mark.parametrize("K", [1, 2, 5, 9, 12])
@pytest.mark.parametrize("avg", [2.0, 2.5, 3.0, 3.7, 4.0])
def test_allocate_exhaustive_is_brute_force(K, avg):
    rng = np.random.default_rng(1000 * K + int(avg * 10))
    for _ in range(4):
        D2, D4, counts = random_case(rng, K)
        bits_b, dist_b = brute_force(list(D2), list(D4), list(counts), avg)
        bits_o, dist_o = otags.allocate(D2, D4, counts, avg)
        assert list(bits_o) == bits_b and dist_o == dist_b
        bits_p, dist_p = kvq.kvq_tag_allocate(D2, D4, counts, avg)
        assert list(bits_p) == bits_b and dist_p == dist_b


def test_allocate_budget_extremes():
    rng = np.random.default_rng(7)
    D2, D4, counts = random_case(rng, 10)
    present = counts > 0
    bits, _ = kvq.kvq_tag_allocate(D2, D4, counts, 2.0)
    assert np.all(bits[present] == 2) and np.all(bits[~present] == 4)
    bits, _ = kvq.kvq_tag_allocate(D2, D4, counts, 4.0)   # no constraint: per-tag minimum
    assert np.array_equal(bits[present], np.where(D2[present] < D4[present], 2, 4))


def test_allocate_greedy_rule():
    """25 tags (> 22: greedy), one token each, D4 = 0 and D2 = k: each switch costs k per
    2 bits saved, so the budget 4 - 2m/25 takes tags 0 .. m-1 to INT2."""
    K, m = 25, 9
    D4 = np.zeros(K)
    D2 = np.arange(K, dtype=np.float64)
    counts = np.ones(K, np.int64)
    avg = 4.0 - 2.0 * m / K
    expect = np.where(np.arange(K) < m, 2, 4)
    bits_o, _ = otags.allocate(D2, D4, counts, avg)
    bits_p, total = kvq.kvq_tag_allocate(D2, D4, counts, avg)
    assert np.array_equal(bits_o, expect) and np.array_equal(bits_p, expect)
    assert total == float(sum(range(m)))


@pytest.mark.parametrize("K", [23, 30, 56])
def test_allocate_greedy_matches_oracle(K):
    rng = np.random.default_rng(K)
    for avg in (2.3, 3.0, 3.6):
        D2, D4, counts = random_case(rng, K)
        bits_o, dist_o = otags.allocate(D2, D4, counts, avg)
        bits_p, dist_p = kvq.kvq_tag_allocate(D2, D4, counts, avg)
        assert np.array_equal(bits_o, bits_p) and dist_o == dist_p
        assert (counts * bits_p).sum() <= avg * counts.sum()


def test_allocate_22_tags_exhaustive():
    rng = np.random.default_rng(22)
    D2, D4, counts = random_case(rng, 22)
    counts[counts == 0] = 1                      # all 22 present: 4M choices
    bits_o, dist_o = otags.allocate(D2, D4, counts, 3.0)
    bits_p, dist_p = kvq.kvq_tag_allocate(D2, D4, counts, 3.0)
    assert np.array_equal(bits_o, bits_p) and dist_o == dist_p


def test_allocate_rejects_bad_budget():
    with pytest.raises(kvq.KvqError):
        kvq.kvq_tag_allocate(np.ones(3), np.ones(3), np.ones(3, np.int64), 1.5)


# ------------------------------------------------------------------ distortion
def bf16(x):
    """float32 -> bf16 bits (round to nearest even)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def calib(rng, NL, R, Hq, Hkv, T, D):
    Q = bf16(rng.standard_normal((NL, R, Hq, T, D)).astype(np.float32))
    K = bf16((rng.standard_normal((NL, R, Hkv, T, D)) * np.where(rng.random(D) < 0.1, 8.0, 1.0)).astype(np.float32))
    V = bf16(rng.standard_normal((NL, R, Hkv, T, D)).astype(np.float32))
    return Q, K, V


def test_causal_attention_pinned_to_decode_attention():
    """The last row of the oracle's causal attention is decode attention over all tokens:
    the C oracle computes that independently."""
    rng = np.random.default_rng(3)
    T, D = 40, 64
    q = bf16(rng.standard_normal((T, D)).astype(np.float32))
    Kh = rng.standard_normal((T, D))
    Vh = rng.standard_normal((T, D))
    qf = oracle.bf16_bits_to_f32(q).astype(np.float64)
    got = otags.causal_attention(qf, Kh, Vh)[-1]
    ref = oracle.attention(q[-1:], Kh, Vh)[0]
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-13)
    # row i sees tokens 0..i only
    row5 = otags.causal_attention(qf, Kh, Vh)[5]
    assert np.allclose(row5, oracle.attention(q[5:6], Kh[:6], Vh[:6])[0], rtol=1e-12, atol=1e-13)


def test_distortion_single_token_closed_form():
    """T = 1: the output is the value row itself, so D_k(b) is the value quantization
    MSE; a single token never fills a 2-bit key group, so both b take the 4-bit path."""
    rng = np.random.default_rng(5)
    Q, K, V = calib(rng, 1, 1, 2, 1, 1, 64)
    tags = np.array([[1]], np.int32)
    D2, D4, counts = otags.distortion(Q, K, V, tags, 3)
    v = oracle.bf16_bits_to_f32(V[0, 0, 0]).reshape(-1, 32)
    s, z, c = oracle.quant_groups(v, 4)
    vh = c * oracle.f16_bits_to_f64(s)[:, None] + oracle.f16_bits_to_f64(z)[:, None]
    mse = np.mean((vh - v.astype(np.float64)) ** 2)
    assert D2[1] == pytest.approx(mse, rel=1e-12) and D4[1] == pytest.approx(mse, rel=1e-12)
    assert D2[0] == D2[2] == D4[0] == D4[2] == 0.0
    assert list(counts) == [0, 1, 0]


def levels(rng, shape, hi):
    """Integers 0..hi with 0 and hi forced into every group of 32 along the last axis."""
    x = rng.integers(0, hi + 1, shape).astype(np.float32)
    x[..., 0::32] = 0
    x[..., 1::32] = hi
    return x


def test_distortion_zero_on_exact_levels():
    """Tag 1's tokens hold only representable levels: 0..3 with 0 and 3 in every group is
    exact at 2 bits (scale 1, zero 0) and 0..15 with 0 and 15 exact at 4 bits."""
    rng = np.random.default_rng(9)
    T, D = 64, 64
    Q, _, _ = calib(rng, 1, 1, 2, 1, T, D)
    tags = np.ones((1, T), np.int32)
    # 2 bits: K per channel over the 64 tokens (two groups of 32), V per token
    Kc = levels(rng, (D, T), 3).T.copy()       # groups of 32 along tokens
    V3 = levels(rng, (T, D), 3)
    D2, _, _ = otags.distortion(Q, bf16(Kc)[None, None, None], bf16(V3)[None, None, None], tags, 2)
    assert D2[1] == 0.0
    K15, V15 = levels(rng, (T, D), 15), levels(rng, (T, D), 15)
    _, D4, _ = otags.distortion(Q, bf16(K15)[None, None, None], bf16(V15)[None, None, None], tags, 2)
    assert D4[1] == 0.0


def test_distortion_aggregation():
    """Sum over layers (two equal layers double it), mean over requests (two equal
    requests change nothing), max over heads (a copied head changes nothing)."""
    rng = np.random.default_rng(11)
    Q, K, V = calib(rng, 1, 1, 2, 1, 48, 64)
    tags = (rng.random((1, 48)) < 0.5).astype(np.int32)
    D2, D4, _ = otags.distortion(Q, K, V, tags, 2)
    D2l, D4l, _ = otags.distortion(np.concatenate([Q, Q]), np.concatenate([K, K]), np.concatenate([V, V]), tags, 2)
    assert np.allclose(D2l, 2 * D2, rtol=1e-14) and np.allclose(D4l, 2 * D4, rtol=1e-14)
    Qr, Kr, Vr = (np.concatenate([a, a], axis=1) for a in (Q, K, V))
    D2r, _, cr = otags.distortion(Qr, Kr, Vr, np.concatenate([tags, tags]), 2)
    assert np.allclose(D2r, D2, rtol=1e-14) and np.array_equal(cr, 2 * np.bincount(tags[0], minlength=2))
    Qh = np.concatenate([Q, Q], axis=2)        # G = 4 with the heads repeated
    D2h, _, _ = otags.distortion(Qh, K, V, tags, 2)
    assert np.allclose(D2h, D2, rtol=1e-14)


@pytest.mark.parametrize("G", [1, 2])
def test_distortion_library_matches_oracle(G):
    rng = np.random.default_rng(20 + G)
    NL, R, Hkv, T, D = 2, 2, 2, 80, 64
    Q, K, V = calib(rng, NL, R, Hkv * G, Hkv, T, D)
    p = np.array([0.55, 0.2, 0.15, 0.1, 0.0])   # tag 0 fills 2-bit key groups; tag 4 absent
    tags = rng.choice(5, size=(R, T), p=p).astype(np.int32)
    D2o, D4o, co = otags.distortion(Q, K, V, tags, 5)
    D2p, D4p, cp = kvq.kvq_tag_distortion(Q, K, V, tags, 5)
    assert np.array_equal(co, cp)
    assert np.allclose(D2p, D2o, rtol=1e-9, atol=1e-15) and np.allclose(D4p, D4o, rtol=1e-9, atol=1e-15)
    assert D2o[4] == D4o[4] == D2p[4] == D4p[4] == 0.0
    assert D2o[0] > 0 and D4o[0] > 0
    for avg in (2.5, 3.0, 3.5):
        assert np.array_equal(otags.allocate(D2o, D4o, co, avg)[0], kvq.kvq_tag_allocate(D2p, D4p, cp, avg)[0])


def test_distortion_argument_checks():
    Q = np.zeros((1, 1, 2, 4, 64), np.uint16)
    K = np.zeros((1, 1, 1, 4, 64), np.uint16)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_tag_distortion(Q, K, K, np.full((1, 4), 3, np.int32), 3)      # tag out of range
    with pytest.raises(kvq.KvqError):
        kvq.kvq_tag_distortion(Q[..., :48], K[..., :48], K[..., :48], np.zeros((1, 4), np.int32), 1)   # D % 32


def test_segment_tag_ids_recipe():
    """Synthetic tag ids: segments of 16-256 tokens sharing one id in [0, 56), the
    temporal axis being the quarter of the sequence the segment starts in."""
    from layer_wise_mixed_b200 import configs, inputs
    w = configs.by_name("c5-alloc")
    ids = inputs.tag_ids(w, 3000, batch=3).numpy()
    assert ids.min() >= 0 and ids.max() < 56
    for row in ids:
        cuts = np.flatnonzero(np.diff(row)) + 1
        starts = np.concatenate([[0], cuts])
        lens = np.diff(np.concatenate([starts, [len(row)]]))
        assert np.all(lens[:-1] >= 16)           # a run may span segments that drew one id
        for s0 in starts:                        # every run starts a segment: id // 14 = its quarter
            assert row[s0] // 14 == min(3, 4 * s0 // len(row))
    assert np.array_equal(ids, inputs.tag_ids(w, 3000, batch=3).numpy())   # seeded


def test_allocation_mask_meets_budget():
    """The workload's INT2/INT4 mask from the per-tag allocation keeps the average bits at
    or under the workload's budget, and every token takes its tag's bits."""
    from layer_wise_mixed_b200 import configs, inputs, tagalloc
    w = configs.by_name("c5-alloc")
    m = tagalloc.token_mask(w, w.max_ctx).numpy()
    assert set(np.unique(m)) <= {2, 4}
    assert m.astype(np.float64).mean() <= w.avg_bits + 1e-12
    ids = inputs.tag_ids(w, w.max_ctx).numpy()
    bits = tagalloc.tag_bits(w)
    assert np.array_equal(m, bits[ids])


def test_device_distortion_host_checks():
    """The device entry point's argument checks run on the host before any CUDA call
    (fake device addresses are never touched)."""
    import ctypes
    from layer_wise_mixed_b200 import build as kbuild
    kbuild.build()
    L = kvq.load()
    n = ctypes.c_size_t(0)
    assert L.kvq_tag_distortion_workspace_bytes(1, 2, 8, 2, 128, 100, 5, ctypes.byref(n)) == 0
    small = n.value
    assert L.kvq_tag_distortion_workspace_bytes(1, 2, 8, 2, 128, 200, 5, ctypes.byref(n)) == 0
    assert n.value > small and n.value % 256 == 0
    # one layer's fp64 dequantized K and V at 2 and 4 bits dominate the size
    assert n.value >= 4 * 2 * 2 * 200 * 128 * 8
    assert L.kvq_tag_distortion_workspace_bytes(1, 2, 8, 2, 96, 200, 5, ctypes.byref(n)) == -2   # EUNSUPPORTED
    assert L.kvq_tag_distortion_workspace_bytes(1, 2, 7, 2, 128, 200, 5, ctypes.byref(n)) == -1  # Hq % Hkv
    assert L.kvq_tag_distortion_workspace_bytes(1, 1, 8, 2, 128, (1 << 31) - 1, 5, ctypes.byref(n)) == -2
    tags = np.zeros((1, 4), np.int32)
    D2, D4, cnt = np.zeros(2), np.zeros(2), np.zeros(2, np.int64)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    fake = 1 << 20                      # 256-byte aligned, never dereferenced
    args = lambda q, ws, nbytes, t: (1, 1, 2, 1, 64, 4, q, fake, fake, p(t), 2, ws, nbytes, p(D2), p(D4), p(cnt), None)
    f = L.kvq_tag_distortion_device
    assert f(*args(None, fake, 1 << 30, tags)) == -1          # null Q
    assert f(*args(fake + 8, fake, 1 << 30, tags)) == -5      # EALIGN
    assert f(*args(fake, None, 1 << 30, tags)) == -4          # no workspace: EUNBOUND
    assert f(*args(fake, fake, 256, tags)) == -4              # workspace too small
    assert f(*args(fake, fake + 16, 1 << 30, tags)) == -4     # workspace not 256-byte aligned
    assert f(*args(fake, fake, 1 << 30, np.full((1, 4), 2, np.int32))) == -1   # tag out of range


@pytest.mark.parametrize("L,bits,stride", [(64, 2, 1), (70, 2, 1), (150, 2, 2), (40, 4, 1), (90, 4, 3)])
def test_tag_quantizer_matches_paged_writer(L, bits, stride):
    """The distortion oracle's quantizer for one tag is the paged cache's writer for the
    tokens of that tag (the C oracle, written separately): INT2 keys per channel over
    consecutive groups of the tag's tokens, values per token, the last count mod 32
    through the 4-bit path; INT4 per token.  Tokens of the tag every `stride` positions,
    the others tagged with the other width in the paged cache and left exact here."""
    rng = np.random.default_rng(L + bits + stride)
    D = 128
    K = bf16(rng.standard_normal((L, D)).astype(np.float32) * 3)
    V = bf16(rng.standard_normal((L, D)).astype(np.float32))
    toks = np.arange(0, L, stride)
    ptags = np.full(L, 6 - bits, np.uint8)
    ptags[toks] = bits
    _, Kp, Vp = oracle.paged_unit(K, V, ptags, D)
    Kq, Vq = otags.quantize_tag_tokens(oracle.bf16_bits_to_f32(K), oracle.bf16_bits_to_f32(V), toks, bits)
    assert np.array_equal(Kq[toks], Kp[toks]) and np.array_equal(Vq[toks], Vp[toks])
    rest = np.setdiff1d(np.arange(L), toks)
    assert np.array_equal(Kq[rest], oracle.bf16_bits_to_f32(K)[rest].astype(np.float64))
