"""Pins for the CPU oracle: each test ties the oracle to something other than itself
(IEEE library conversions, closed forms, brute force, invariants, the pages' printed
accounting numbers, hand-derived format positions).  CPU only."""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import accounting

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(20260512)


def to_bf16_bits(x):
    """Round binary32 -> bf16 (RNE) with numpy integer ops (test-side helper)."""
    u = np.ascontiguousarray(np.asarray(x, np.float32)).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_vals(bits):
    return oracle.bf16_bits_to_f32(bits)


# ----------------------------------------------------------------- number formats
def test_f16_rne_matches_ieee_library():
    """Binary32 -> binary16 RNE against numpy's IEEE conversion: random normals,
    subnormals, exact ties, overflow boundary."""
    xs = [rng.standard_normal(200000).astype(np.float32) * np.float32(s)
          for s in (1e-7, 1e-5, 1e-3, 1.0, 300.0, 6e4)]
    # exact ties between two fp16 neighbours (normal and subnormal ranges)
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    ties = ((lo + hi) / 2).astype(np.float32)
    edge = np.array([65504, 65519.99, 65520, 65536, 1e30, 2 ** -24, 2 ** -25, 2 ** -25 * 1.0001,
                     3 * 2 ** -26, 0.0, -0.0, -65520], np.float32)
    x = np.concatenate(xs + [ties, edge, -ties])
    mine = oracle.f32_to_f16_bits(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(mine, ref)


def test_f16_decode_matches_library():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (h & 0x7C00) != 0x7C00
    mine = oracle.f16_bits_to_f64(h)
    ref = h.view(np.float16).astype(np.float64)
    assert np.array_equal(mine[finite], ref[finite])
    assert np.all(np.isinf(mine[(h & 0x7FFF) == 0x7C00]))


# ----------------------------------------------------------------- quantizer (Q1)
def random_groups(n, scale=1.0):
    x = (rng.standard_normal((n, 32)) * scale).astype(np.float32)
    return bf16_vals(to_bf16_bits(x)).reshape(n, 32)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_error_bound(bits):
    """P1: |x - x^| <= s*(1/2 + 2^(b-22)) whenever the stored zero equals the group
    minimum and the stored scale is a normal fp16 (or zero).  The 2^(b-22) term is the
    binary32 rounding of (x - z)/s (two correctly rounded operations on a quotient
    below 2^b); the stored-scale reading makes the code the nearest grid point of
    the grid the decoder uses."""
    x = np.concatenate([random_groups(20000), random_groups(5000, 20.0), random_groups(2000, 1e-2)])
    s16, z16, c = oracle.quant_groups(x, bits)
    s = oracle.f16_bits_to_f64(s16)[:, None]
    z = oracle.f16_bits_to_f64(z16)[:, None]
    xh = c.astype(np.float64) * s + z
    ok = (z[:, 0] == x.min(1)) & ((s[:, 0] == 0) | (s[:, 0] >= 2.0 ** -14))
    assert ok.mean() > 0.999
    err = np.abs(x.astype(np.float64) - xh)[ok]
    bound = (s * (0.5 + 2.0 ** (bits - 22)))[ok]
    assert np.all(err <= bound)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_endpoint_codes(bits):
    """P2: the group minimum codes to 0 and the maximum to 2^b-1 (normal scale)."""
    x = random_groups(20000)
    s16, z16, c = oracle.quant_groups(x, bits)
    s = oracle.f16_bits_to_f64(s16)
    ok = s >= 2.0 ** -14
    rows = np.arange(len(x))
    assert np.all(c[rows, x.argmin(1)][ok] == 0)
    assert np.all(c[rows, x.argmax(1)][ok] == 2 ** bits - 1)


@pytest.mark.parametrize("bits,m,e", [(2, -1.5, -2), (4, -1.5, -3), (8, -2.0, -6), (4, 3.0, 0),
                                      (2, 0.25, -4)])
def test_on_grid_inputs_are_lossless(bits, m, e):
    """P3 (closed form): x = m + k*2^e with k spanning 0..2^b-1 gives scale 2^e,
    zero m, codes k, and exact reconstruction."""
    qmax = 2 ** bits - 1
    ks = np.concatenate([[0, qmax], rng.integers(0, qmax + 1, 30)])
    rng.shuffle(ks)
    x = (m + ks * 2.0 ** e).astype(np.float32)
    assert np.array_equal(bf16_vals(to_bf16_bits(x)), x)   # inputs are bf16-exact
    s16, z16, c = oracle.quant_groups(x[None], bits)
    assert oracle.f16_bits_to_f64(s16)[0] == 2.0 ** e
    assert oracle.f16_bits_to_f64(z16)[0] == m
    assert np.array_equal(c[0], ks)
    xh = c[0] * oracle.f16_bits_to_f64(s16)[0] + oracle.f16_bits_to_f64(z16)[0]
    assert np.array_equal(xh, x.astype(np.float64))


def test_constant_group():
    """P4: a constant group has scale 0, codes 0 and reconstructs exactly."""
    for v in (0.0, 1.5, -3.25, 1e-3):
        x = np.full((1, 32), v, np.float32)
        for bits in (2, 4, 8):
            s16, z16, c = oracle.quant_groups(x, bits)
            assert s16[0] == 0 and np.all(c == 0)
            assert oracle.f16_bits_to_f64(z16)[0] == np.float32(v).astype(np.float16).astype(np.float64)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_codes_are_nearest_grid_point(bits):
    """Brute force: every code minimises |x - (c*s + z)| over all 2^b codes (s, z the
    stored fp16 values), except at exact ties."""
    x = random_groups(3000)
    s16, z16, c = oracle.quant_groups(x, bits)
    s = oracle.f16_bits_to_f64(s16)[:, None, None]
    z = oracle.f16_bits_to_f64(z16)[:, None, None]
    grid = np.arange(2 ** bits)[None, None, :] * s + z
    d = np.abs(x.astype(np.float64)[:, :, None] - grid)
    best = d.argmin(2)
    dsort = np.sort(d, 2)
    clear = (dsort[:, :, 1] - dsort[:, :, 0]) > 1e-9 * s[:, :, 0]
    assert np.array_equal(best[clear], c[clear].astype(np.int64))


def test_numpy_restatement_agrees():
    """Cross-check (not a pin by itself): a numpy float32 restatement of Q1."""
    x = random_groups(5000, 3.0)
    for bits in (2, 4, 8):
        s16, z16, c = oracle.quant_groups(x, bits)
        mn, mx = x.min(1), x.max(1)
        s32 = (mx - mn) / np.float32(2 ** bits - 1)
        s = s32.astype(np.float16).astype(np.float32)
        z = mn.astype(np.float16).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.rint((x - z[:, None]) / s[:, None])
        cc = np.where(s[:, None] == 0, 0, np.clip(q, 0, 2 ** bits - 1)).astype(np.uint8)
        assert np.array_equal(s16, s.astype(np.float16).view(np.uint16))
        assert np.array_equal(c, cc)


# ----------------------------------------------------------------- storage format (Q3)
def test_golden_positions():
    """Hand-derived positions of single codes (no page prints a layout)."""
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "format_v2_positions.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) > 30
    for role, D, bits, u, d, byte, bit in rows:
        area = np.zeros(2 * 2 * D * bits, np.uint8)
        word = ((2 ** bits - 1) << bit) & 0xFFFFFFFF
        area[byte:byte + 4] = np.frombuffer(np.uint32(word).tobytes(), np.uint8)
        assert oracle.get_code(area, role, u, d, D, bits) == 2 ** bits - 1, (role, D, bits, u, d)
        # neighbours in token and channel read zero
        for uu, dd in ((u ^ 1, d), (u, d ^ 1), (u ^ 8, d), (u, d ^ 8)):
            assert oracle.get_code(area, role, uu, dd, D, bits) == 0


@pytest.mark.parametrize("role", [0, 1])
@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_format_is_a_bijection(role, D, bits):
    """Every (token, channel) of a block owns `bits` distinct bits inside one 32-bit
    word, no two codes overlap, and the codes tile the code area exactly."""
    area_bits = 2 * 2 * D * bits * 8
    owner = np.full(area_bits, -1, np.int64)
    for u in range(32):
        for d in range(D):
            byte, bit = oracle.code_position(role, u, d, D, bits)
            assert byte % 4 == 0 and 0 <= bit and bit + bits <= 32
            lo = byte * 8 + bit
            assert np.all(owner[lo:lo + bits] == -1), (u, d)
            owner[lo:lo + bits] = u * D + d
    assert np.all(owner >= 0)


def test_worked_packing_examples():
    """P5: end-to-end worked examples through quantizer and packer.
    (a) 2-bit value codes 0,1,2,3 repeated across the 16 fields of lane 0's first
        word -> 0xE4E4E4E4.  (b) 4-bit key codes 0..7 in the 8 fields -> 0x76543210."""
    D = 128
    # (a) values: fields of lane 0 word 0 hold channels {0, 8, 16, 24} of tokens {0, 1, 8, 9}
    V = np.zeros((32, D), np.float32)
    for u in range(32):
        for d in (0, 8, 16, 24):
            V[u, d] = ((d // 8) % 2) + 2 * ((u // 8) % 2)
        V[u, 1], V[u, 2] = 0.0, 3.0            # group range [0, 3] -> scale 1, zero 0
        for j in range(1, D // 32):
            V[u, 32 * j], V[u, 32 * j + 1] = 0.0, 3.0
    K = np.zeros((32, D), np.float32)
    img, _, _ = oracle.unit(to_bf16_bits(K), to_bf16_bits(V), D, 4, 2, oracle.PER_TOKEN)
    rec = oracle.record_bytes(D, 4, 2)
    vcode = img[4 * D * 4 + 4 * D:]
    assert int(np.frombuffer(vcode[:4].tobytes(), np.uint32)[0]) == 0xE4E4E4E4
    # (b) keys per channel: lane 0 word 0 holds (u, d) in {0, 8} x {0, 1, 8, 9}
    K = np.zeros((32, D), np.float32)
    K[31, :] = 15.0                             # channel range [0, 15] -> scale 1, zero 0
    for (u, d), v in {(0, 0): 0, (0, 8): 1, (8, 0): 2, (8, 8): 3,
                      (0, 1): 4, (0, 9): 5, (8, 1): 6, (8, 9): 7}.items():
        K[u, d] = v
    V = np.zeros((32, D), np.float32)
    img, _, _ = oracle.unit(to_bf16_bits(K), to_bf16_bits(V), D, 4, 2, oracle.PER_CHANNEL)
    assert int(np.frombuffer(img[:4].tobytes(), np.uint32)[0]) == 0x76543210
    assert len(img) == rec + 64 * D


def chan_sz_off(d):
    """Test-side restatement of the per-channel key scale/zero placement."""
    k, e = divmod(d, 16)
    t, r, hb = (e % 8) // 2, e // 8, e % 2
    so = 16 * (4 * k + t) + 8 * r + 2 * hb
    return so, so + 4


def tok_sz_off(u, j, nj):
    """Test-side restatement of the per-token scale/zero placement."""
    so = 8 * nj * (u // 2) + 4 * j + 2 * (u % 2)
    return so, so + 4 * nj


def decode_unit_image(img, L, D, bk, bv, kmode):
    """Independent reader: codes and s/z of a unit image -> dequantized K^, V^ (fp64)."""
    REC = oracle.record_bytes(D, bk, bv)
    KC, KS, VC = 4 * D * bk, 4 * D, 4 * D * bv
    nj = D // 32
    nblk = (L + 31) // 32
    Kh = np.zeros((L, D))
    Vh = np.zeros((L, D))

    def h16(buf, off):
        return oracle.f16_bits_to_f64(np.frombuffer(buf[off:off + 2].tobytes(), np.uint16))[0]

    for tok in range(L):
        blk, u = divmod(tok, 32)
        rec = img[blk * REC:(blk + 1) * REC]
        for d in range(D):
            so, zo = tok_sz_off(u, d // 32, nj)
            s, z = h16(rec, KC + KS + VC + so), h16(rec, KC + KS + VC + zo)
            Vh[tok, d] = oracle.get_code(rec[KC + KS:KC + KS + VC], 1, u, d, D, bv) * s + z
            if kmode == oracle.PER_TOKEN:
                so, zo = tok_sz_off(u, d // 32, nj)
                Kh[tok, d] = oracle.get_code(rec[:KC], 0, u, d, D, bk) * h16(rec, KC + so) + h16(rec, KC + zo)
            elif blk < L // 32:
                so, zo = chan_sz_off(d)
                Kh[tok, d] = oracle.get_code(rec[:KC], 0, u, d, D, bk) * h16(rec, KC + so) + h16(rec, KC + zo)
            else:
                res = img[nblk * REC:]
                Kh[tok, d] = oracle.bf16_bits_to_f32(np.frombuffer(res[2 * (u * D + d):2 * (u * D + d) + 2].tobytes(), np.uint16))[0]
    return Kh, Vh


def test_golden_sz_positions():
    """Hand-derived scale/zero offsets (no page fixes a layout)."""
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "format_v2_sz_positions.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 12
    for kind, nj, index, j, so, zo in rows:
        assert oracle.sz_position(kind, index, j, nj) == (so, zo), (kind, nj, index, j)


@pytest.mark.parametrize("nj", [1, 2, 4, 8])
def test_sz_layout_is_a_bijection(nj):
    """Scales and zeros of every channel (per-channel area) and of every (token, group)
    (per-token area) occupy distinct aligned fp16 slots that tile the 4*D-byte area."""
    D = 32 * nj
    seen = set()
    for d in range(D):
        so, zo = oracle.sz_position(0, d, 0, nj)
        assert so % 2 == 0 and zo % 2 == 0 and so not in seen and zo not in seen
        seen |= {so, zo}
    assert seen == set(range(0, 4 * D, 2))
    seen = set()
    for u in range(32):
        for j in range(nj):
            so, zo = oracle.sz_position(1, u, j, nj)
            assert so not in seen and zo not in seen
            seen |= {so, zo}
    assert seen == set(range(0, 4 * D, 2))


@pytest.mark.parametrize("L,kmode,bk,bv", [(40, 0, 4, 2), (33, 1, 8, 4), (64, 0, 2, 8), (7, 0, 8, 8)])
def test_image_round_trip(L, kmode, bk, bv):
    """The image decodes (through an independent reader) to the oracle's dequantized cache."""
    D = 64
    K = to_bf16_bits(rng.standard_normal((L, D)) * 3)
    V = to_bf16_bits(rng.standard_normal((L, D)))
    img, Kh, Vh = oracle.unit(K, V, D, bk, bv, kmode)
    Kd, Vd = decode_unit_image(img, L, D, bk, bv, kmode)
    assert np.array_equal(Kd, Kh) and np.array_equal(Vd, Vh)


def test_image_edges_and_zero_fill():
    D, bk, bv = 64, 4, 2
    REC = oracle.record_bytes(D, bk, bv)
    KC, KS, VC = 4 * D * bk, 4 * D, 4 * D * bv
    nj = D // 32
    for L in (0, 1, 31, 32, 33):
        K = to_bf16_bits(rng.standard_normal((max(L, 1), D)))[:L]
        V = to_bf16_bits(rng.standard_normal((max(L, 1), D)))[:L]
        img, Kh, Vh = oracle.unit(K, V, D, bk, bv, oracle.PER_CHANNEL)
        nblk = (L + 31) // 32
        assert len(img) == nblk * REC + 64 * D
        r = L % 32
        if r:
            tail = img[(nblk - 1) * REC:nblk * REC]
            assert not tail[:KC + KS].any()                  # incomplete key group: not stored
            vsz = tail[KC + KS + VC:]
            for u in range(r, 32):                           # value s/z of absent tokens
                for j in range(nj):
                    so, zo = tok_sz_off(u, j, nj)
                    assert not vsz[so:so + 2].any() and not vsz[zo:zo + 2].any()
            res = img[nblk * REC:]
            assert not res[2 * D * r:].any()
            assert np.array_equal(Kh[L - r:], bf16_vals(K[L - r:]).astype(np.float64))
        else:
            assert not img[nblk * REC:].any()


def test_prefix_stability():
    """Complete blocks of a unit do not change when more tokens arrive (the image of
    a sequence is a function of that sequence, so incremental = bulk)."""
    D, bk, bv = 128, 8, 4
    K = to_bf16_bits(rng.standard_normal((100, D)))
    V = to_bf16_bits(rng.standard_normal((100, D)))
    REC = oracle.record_bytes(D, bk, bv)
    for kmode in (0, 1):
        a, _, _ = oracle.unit(K[:64], V[:64], D, bk, bv, kmode)
        b, _, _ = oracle.unit(K, V, D, bk, bv, kmode)
        assert np.array_equal(a[:2 * REC], b[:2 * REC])


# ----------------------------------------------------------------- attention (Q4)
def brute_attention(q, Kh, Vh):
    qf = bf16_vals(q).astype(np.float64)
    D = Kh.shape[1]
    s = qf @ Kh.T / np.sqrt(D)
    p = np.exp(s - s.max(1, keepdims=True))
    return (p @ Vh) / p.sum(1, keepdims=True)


def test_attention_brute_force():
    """P9: numpy float64 softmax attention on Tiny-sized inputs."""
    for L, G, D in ((257, 2, 64), (1, 4, 64), (33, 7, 128), (1000, 1, 32)):
        q = to_bf16_bits(rng.standard_normal((G, D)))
        Kh = rng.standard_normal((L, D)) * 2
        Vh = rng.standard_normal((L, D))
        out = oracle.attention(q, Kh, Vh)
        ref = brute_attention(q, Kh, Vh)
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    D = 64
    q = to_bf16_bits(rng.standard_normal((3, D)))
    Vh = rng.standard_normal((50, D))
    # all keys equal -> uniform weights -> mean value
    Kh = np.tile(rng.standard_normal(D), (50, 1))
    assert np.allclose(oracle.attention(q, Kh, Vh), np.tile(Vh.mean(0), (3, 1)), rtol=1e-12, atol=1e-14)
    # L = 1 -> the single value
    assert np.array_equal(oracle.attention(q, Kh[:1], Vh[:1]), np.tile(Vh[0], (3, 1)))
    # one dominant key -> its value
    q1 = to_bf16_bits(np.ones((1, D)))
    Kd = rng.standard_normal((50, D)) * 0.01
    Kd[17] = 100.0
    assert np.allclose(oracle.attention(q1, Kd, Vh), Vh[17:18], rtol=0, atol=1e-12)


def test_split_invariance():
    """P10: log-sum-exp merge of any partition equals the unsplit result."""
    L, G, D = 300, 4, 64
    q = to_bf16_bits(rng.standard_normal((G, D)))
    Kh = rng.standard_normal((L, D)) * 3
    Vh = rng.standard_normal((L, D))
    ref = oracle.attention(q, Kh, Vh)
    for _ in range(5):
        cuts = np.sort(rng.choice(np.arange(1, L), rng.integers(1, 8), replace=False))
        bounds = [0, *cuts.tolist(), L]
        parts = [oracle.attention_partial(q, Kh, Vh, a, b) for a, b in zip(bounds[:-1], bounds[1:])]
        m = np.stack([p[0] for p in parts])
        l = np.stack([p[1] for p in parts])
        acc = np.stack([p[2] for p in parts])
        assert np.allclose(oracle.merge_partials(m, l, acc), ref, rtol=1e-12, atol=1e-14)


def test_layer_gqa_mapping_and_units():
    """P13: query head hq attends kv head hq // G; G = 1 is plain multi-head attention;
    the layer image is the concatenation of the unit images."""
    B, Hkv, G, L, D = 2, 3, 2, 45, 64
    K = to_bf16_bits(rng.standard_normal((B, Hkv, L, D)))
    V = to_bf16_bits(rng.standard_normal((B, Hkv, L, D)))
    Q = to_bf16_bits(rng.standard_normal((B, Hkv * G, D)))
    img, out = oracle.layer(K, V, Q, G, 4, 2, oracle.PER_CHANNEL)
    per = oracle.unit_image_bytes(L, D, 4, 2, 0)
    for b in range(B):
        for h in range(Hkv):
            uimg, Kh, Vh = oracle.unit(K[b, h], V[b, h], D, 4, 2, 0)
            assert np.array_equal(img[(b * Hkv + h) * per:(b * Hkv + h + 1) * per], uimg)
            for g in range(G):
                assert np.allclose(out[b, h * G + g], brute_attention(Q[b, h * G + g][None], Kh, Vh)[0],
                                   rtol=1e-12, atol=1e-13)
    # G = 1: each query head uses its own kv head; permuting kv heads permutes outputs
    Q1 = to_bf16_bits(rng.standard_normal((B, Hkv, D)))
    _, o1 = oracle.layer(K, V, Q1, 1, 8, 4, 0, want_image=False)
    perm = [2, 0, 1]
    _, o2 = oracle.layer(K[:, perm], V[:, perm], Q1[:, perm], 1, 8, 4, 0, want_image=False)
    assert np.allclose(o2, o1[:, perm], rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------- pages' measurements
def test_accounting_matches_pages():
    """P6: the pages' bit accounting (tests/golden/accounting.json, with citations)."""
    g = json.load(open(os.path.join(GOLDEN, "accounting.json")))
    for key in ("llama_map_3_25", "qwen_map_4_0"):
        m = accounting.expand_map(g[key]["layers"])
        assert accounting.equivalent_bits(m) == g[key]["equivalent_bits"]
    kv = g["k8v2_vs_k4v8"]
    assert accounting.pair_bits(8, 2) == kv["k8v2_bits"]
    assert accounting.pair_bits(4, 8) == kv["k4v8_bits"]
    assert accounting.saving_vs_8bit_pct(5, 6) == kv["less_memory_pct"]
    assert abs(accounting.direct_saving_pct(5, 6) - 16.667) < 1e-3   # the other reading, not printed
    # the stored format: codes + fp16 scale and zero per 32 -> +1 bit per element
    assert accounting.storage_bits(8, 4) == 7.0
    assert accounting.reduction_vs_bf16_pct(accounting.storage_bits(8, 4)) == 56.25
    D = 128
    rec = oracle.record_bytes(D, 8, 4)
    assert rec * 8 / (32 * D * 2) == accounting.storage_bits(8, 4)
    # KVSplit's 59% cross-check corresponds to 6.5 bits (scale only, no zero)
    assert round(accounting.reduction_vs_bf16_pct(accounting.storage_bits(8, 4, meta_bits_per_group=16))) \
        == g["kvsplit_k8v4"]["memory_reduction_pct"]


def _workload_kv(wl, L):
    """Seeded CPU keys/values of layer 0 as bf16 bit patterns."""
    import torch
    from layer_wise_mixed_b200 import inputs
    K, V = inputs.layer_kv(wl, 0, L, "cpu")
    return K.view(torch.int16).numpy().view(np.uint16), V.view(torch.int16).numpy().view(np.uint16)


def test_per_channel_beats_per_token_for_outlier_keys():
    """P7 (direction of the KVTuner summary's measured relative key error, per-token
    0.012280 -> per-channel 0.004869): with channel outliers, per-channel grouping
    has the smaller relative key error, at every bit width."""
    from layer_wise_mixed_b200 import configs
    for wl in (configs.tiny(), configs.llama_c2()):
        K, V = _workload_kv(wl, 256)
        D = wl.head_dim
        for bits in (2, 4, 8):
            errs = {}
            for kmode in (0, 1):
                num = den = 0.0
                for h in range(min(wl.n_kv_heads, 4)):
                    _, Kh, _ = oracle.unit(K[0, h], V[0, h], D, bits, bits, kmode, want_image=False)
                    Kf = bf16_vals(K[0, h]).astype(np.float64).reshape(-1, D)
                    num += ((Kf - Kh) ** 2).sum()
                    den += (Kf ** 2).sum()
                errs[kmode] = np.sqrt(num / den)
            assert errs[0] < 0.7 * errs[1], (wl.name, bits, errs)


def test_keys_matter_more_k4v2_vs_k2v4():
    """P8 (direction of the KVTuner summary's relative attention-output error,
    K4V2 0.453 vs K2V4 0.892): on Tiny, K4V2 has the smaller output error."""
    from layer_wise_mixed_b200 import configs, inputs
    import torch
    wl = configs.tiny()
    K, V = _workload_kv(wl, 257)
    Q = inputs.step_q(wl, 0, 0).view(torch.int16).numpy().view(np.uint16)
    D, G = wl.head_dim, wl.G
    err = {}
    for bk, bv in ((4, 2), (2, 4)):
        num = den = 0.0
        for h in range(wl.n_kv_heads):
            _, Kh, Vh = oracle.unit(K[0, h], V[0, h], D, bk, bv, oracle.PER_CHANNEL, want_image=False)
            Kf = bf16_vals(K[0, h]).astype(np.float64).reshape(-1, D)
            Vf = bf16_vals(V[0, h]).astype(np.float64).reshape(-1, D)
            q = Q[0, h * G:(h + 1) * G]
            o_q = oracle.attention(q, Kh, Vh)
            o_f = oracle.attention(q, Kf, Vf)
            num += ((o_q - o_f) ** 2).sum()
            den += (o_f ** 2).sum()
        err[(bk, bv)] = np.sqrt(num / den)
    assert err[(4, 2)] < err[(2, 4)], err
