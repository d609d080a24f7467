"""Pins for the oracle's paged INT2/INT4 token-mixed cache (TriAxialKV facts: INT2 keys
per channel and values per token with 2 bits, INT4 keys and values per token, group 32,
leftover INT2 tokens through the INT4 per-token path, INT2 pages ahead of INT4 pages)."""
import numpy as np
import pytest

import oracle
from test_oracle_pins import bf16_vals, chan_sz_off, to_bf16_bits, tok_sz_off

rng = np.random.default_rng(7)
D = 128
NJ = D // 32


def h16(buf, off):
    return oracle.f16_bits_to_f64(np.frombuffer(buf[off:off + 2].tobytes(), np.uint16))[0]


def read_paged(img, tags, L):
    """Independent reader of a paged unit image -> dequantized K^, V^ in token order."""
    tags = np.asarray(tags)
    i2 = np.flatnonzero(tags == 2)
    i4 = np.flatnonzero(tags == 4)
    n2g, np_ = len(i2) // 32, len(i2) % 32
    REC2 = oracle.paged_rec2_bytes(D)
    P4 = oracle.paged_page4_bytes(D)
    KC2, KS2, VC2 = 4 * D * 2, 4 * D, 4 * D * 2
    KC4, KS4, VC4 = 2 * D * 4, 2 * D, 2 * D * 4
    Kh = np.full((L, D), np.nan)
    Vh = np.full((L, D), np.nan)
    for g in range(n2g):
        rec = img[g * REC2:(g + 1) * REC2]
        for u in range(32):
            tok = i2[32 * g + u]
            for d in range(D):
                so, zo = chan_sz_off(d)
                Kh[tok, d] = oracle.get_code(rec[:KC2], 0, u, d, D, 2) * h16(rec, KC2 + so) + h16(rec, KC2 + zo)
                so, zo = tok_sz_off(u, d // 32, NJ)
                vs = KC2 + KS2 + VC2
                Vh[tok, d] = oracle.get_code(rec[KC2 + KS2:KC2 + KS2 + VC2], 1, u, d, D, 2) * h16(rec, vs + so) \
                    + h16(rec, vs + zo)
    base4 = n2g * REC2
    n4p = (len(i4) + 15) // 16
    toks4 = [(i4[r], base4 + (r // 16) * P4, r % 16) for r in range(len(i4))]
    pend = base4 + n4p * P4
    toks4 += [(i2[32 * n2g + r], pend + (r // 16) * P4, r % 16) for r in range(np_)]
    for tok, off, u in toks4:
        page = img[off:off + P4]
        for d in range(D):
            so, zo = tok_sz_off(u, d // 32, NJ)
            Kh[tok, d] = oracle.get_code(page[:KC4], 0, u, d, D, 4) * h16(page, KC4 + so) + h16(page, KC4 + zo)
            vs = KC4 + KS4 + VC4
            Vh[tok, d] = oracle.get_code(page[KC4 + KS4:KC4 + KS4 + VC4], 1, u, d, D, 4) * h16(page, vs + so) \
                + h16(page, vs + zo)
    return Kh, Vh, n2g, len(i4), np_


def rand_seq(L, tags):
    K = to_bf16_bits(rng.standard_normal((L, D)) * 2)
    V = to_bf16_bits(rng.standard_normal((L, D)))
    return K, V, np.asarray(tags, np.uint8)


@pytest.mark.parametrize("pattern", ["all2", "all4", "alt", "bern"])
def test_paged_image_reads_back(pattern):
    L = 75
    tags = {"all2": [2] * L, "all4": [4] * L, "alt": [2, 4] * (L // 2) + [2],
            "bern": list(np.where(rng.random(L) < 0.5, 2, 4))}[pattern]
    K, V, tags = rand_seq(L, tags)
    img, Kh, Vh = oracle.paged_unit(K, V, tags, D)
    Kr, Vr, n2g, n4, np_ = read_paged(img, tags, L)
    assert np.array_equal(Kr, Kh) and np.array_equal(Vr, Vh)
    assert n2g == int((tags == 2).sum()) // 32 and n4 == int((tags == 4).sum())
    assert len(img) == n2g * oracle.paged_rec2_bytes(D) + ((n4 + 15) // 16 + 2) * oracle.paged_page4_bytes(D) \
        + 2 * 32 * D * 2
    # staging holds the pending INT2 tokens' originals, zeros after them
    stg = img[-2 * 32 * D * 2:].view(np.uint16).reshape(2, 32, D)
    pend = np.flatnonzero(tags == 2)[32 * n2g:]
    assert np.array_equal(stg[0, :np_], K[pend]) and np.array_equal(stg[1, :np_], V[pend])
    assert not stg[:, np_:].any()


def test_bit_widths_and_leftover_routing():
    """33 INT2 tokens: the first 32 are one group (2-bit keys per channel, 2-bit values);
    the 33rd is a leftover stored 4-bit per token (error within half a 4-bit step)."""
    L = 33
    K, V, tags = rand_seq(L, [2] * L)
    _, Kh, Vh = oracle.paged_unit(K, V, tags, D)
    Kf, Vf = bf16_vals(K).astype(np.float64), bf16_vals(V).astype(np.float64)
    # group: per-channel 2-bit keys -> error <= range/3/2 of each channel's 32 tokens
    rk = (Kf[:32].max(0) - Kf[:32].min(0)) / 3
    assert np.all(np.abs(Kf[:32] - Kh[:32]) <= rk / 2 * 1.002 + 1e-12)
    # leftover: per-token 4-bit over 32 channels
    g = Kf[32].reshape(NJ, 32)
    r4 = (g.max(1) - g.min(1)) / 15
    assert np.all(np.abs(g - Kh[32].reshape(NJ, 32)) <= r4[:, None] / 2 * 1.002 + 1e-12)
    # the leftover is not a per-channel 2-bit value: its error is far below a 2-bit step
    assert np.abs(Kf[32] - Kh[32]).max() < rk.min() / 2


def test_page_order_invariance():
    """P11: attention over the INT2-first page order equals attention over token order."""
    L = 300
    K, V, tags = rand_seq(L, np.where(rng.random(L) < 0.5, 2, 4))
    _, Kh, Vh = oracle.paged_unit(K, V, tags, D)
    i2 = np.flatnonzero(tags == 2)
    n2g = len(i2) // 32
    order = np.concatenate([i2[:32 * n2g], np.flatnonzero(tags == 4), i2[32 * n2g:]])
    assert sorted(order.tolist()) == list(range(L))
    q = to_bf16_bits(rng.standard_normal((4, D)))
    a = oracle.attention(q, Kh, Vh)
    b = oracle.attention(q, Kh[order], Vh[order])
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14)


def test_prefix_stability():
    """Complete INT2 groups and full INT4 pages do not change as tokens arrive."""
    L = 260
    K, V, tags = rand_seq(L, np.where(rng.random(L) < 0.6, 2, 4))
    for L1 in (100, 180, 259):
        img1, _, _ = oracle.paged_unit(K[:L1], V[:L1], tags[:L1], D)
        img2, _, _ = oracle.paged_unit(K, V, tags, D)
        g1 = int((tags[:L1] == 2).sum()) // 32
        REC2 = oracle.paged_rec2_bytes(D)
        assert np.array_equal(img1[:g1 * REC2], img2[:g1 * REC2])
        n4_1 = int((tags[:L1] == 4).sum())
        g2 = int((tags == 2).sum()) // 32
        P4 = oracle.paged_page4_bytes(D)
        full = n4_1 // 16
        assert np.array_equal(img1[g1 * REC2:g1 * REC2 + full * P4], img2[g2 * REC2:g2 * REC2 + full * P4])


def test_paged_layer_matches_units():
    B, Hkv, G, L = 2, 2, 4, 70
    K = to_bf16_bits(rng.standard_normal((B, Hkv, L, D)))
    V = to_bf16_bits(rng.standard_normal((B, Hkv, L, D)))
    tags = np.where(rng.random((B, L)) < 0.5, 2, 4).astype(np.uint8)
    Q = to_bf16_bits(rng.standard_normal((B, Hkv * G, D)))
    img, out = oracle.paged_layer(K, V, tags, Q, G)
    off = 0
    for b in range(B):
        for h in range(Hkv):
            u, Kh, Vh = oracle.paged_unit(K[b, h], V[b, h], tags[b], D)
            assert np.array_equal(img[off:off + len(u)], u)
            off += len(u)
            assert np.allclose(out[b, h * G:(h + 1) * G], oracle.attention(Q[b, h * G:(h + 1) * G], Kh, Vh),
                               rtol=1e-13, atol=1e-14)
    assert off == len(img)


@pytest.mark.parametrize("tag,L", [(2, 64), (4, 48), (4, 37)])
def test_uniform_tags_reduce_to_uniform_layers(tag, L):
    """All tokens INT2 (a whole number of groups) is the per-layer K2V2 cache with
    per-channel keys; all tokens INT4 is K4V4 with per-token keys.  The paged writer and
    the per-layer writer are separate code, so their dequantized caches must agree
    exactly, and so must attention over them."""
    K, V, tags = rand_seq(L, [tag] * L)
    _, Kp, Vp = oracle.paged_unit(K, V, tags, D)
    kmode = 0 if tag == 2 else 1
    _, Ku, Vu = oracle.unit(K, V, D, tag, tag, kmode)
    assert np.array_equal(Kp, Ku) and np.array_equal(Vp, Vu)
    q = to_bf16_bits(rng.standard_normal((2, D)))
    assert np.array_equal(oracle.attention(q, Kp, Vp), oracle.attention(q, Ku, Vu))
