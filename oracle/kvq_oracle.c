/*
 * kvq_oracle.c -- plain, slow CPU oracle for layer-wise mixed-precision KV-cache
 * quantization and single-token decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or helper with the CUDA library; the only thing both sides agree
 * on is the storage format, which is written out as a specification below and
 * implemented here independently.
 *
 * Sources (web pages on the subject; cited by page title and section):
 *  [KVT]  "KVTuner: Sensitivity-Aware Layer-Wise Mixed-Precision KV Cache
 *          Quantization ..." (atlas.scime.ai summary) -- Approach; Measured effects
 *          table; Limitations (KIVI kernel, HF transformers).
 *  [MIX]  "Mixed-precision KV-cache quantization per-layer sensitivity"
 *          (llms-explorer) -- Facts: per-layer K/V precision pairs, per-channel
 *          asymmetric keys vs per-token asymmetric.
 *  [TRI]  "TriAxialKV per-role mixed-precision KV quantization for agentic
 *          prefills" (llms-explorer) -- Facts: asymmetric groupwise quantizer with
 *          group size 32; INT2 per-channel keys, per-token values; leftover INT2
 *          keys routed through the INT4 per-token path; INT2/INT4 page pools;
 *          bitwidth-homogeneous flash-decoding splits merged by log-sum-exp.
 *
 * Precision: every quantizer step is one correctly rounded IEEE binary32
 * operation (x86-64 SSE arithmetic, built with -ffp-contract=off, no fast-math);
 * dequantisation and attention are binary64.
 *
 * ---------------------------------------------------------------------------
 * Q1  Group quantizer ([TRI] Facts: asymmetric, groupwise, g = 32; [MIX] Facts:
 *     asymmetric keys per channel, values per token).  For 32 inputs x_i and
 *     bits b in {2,4,8}:
 *        mn = min x_i, mx = max x_i
 *        s32 = (mx - mn) / (2^b - 1)            binary32 subtract, then divide
 *        s16 = fp16_rne(s32), z16 = fp16_rne(mn) stored scale and zero
 *        s = float(s16), z = float(z16)
 *        code_i = 0 if s == 0, else clamp(rne((x_i - z) / s), 0, 2^b - 1)
 *        dequant  x^_i = code_i * s + z          (binary64 here)
 *     Reading: the divisor in the code formula is the stored fp16 scale (the
 *     value the decoder multiplies by), and the zero is the fp16 group minimum.
 *
 * Q2  Grouping axes.  Keys in per-channel mode: 32 consecutive tokens of one
 *     channel; the L mod 32 newest tokens are not quantized and stay in a bf16
 *     residual.  Values, and keys in per-token mode: 32 consecutive channels of
 *     one token.
 *
 * Q3  Storage format (version 2).  The pages fix no layout; this one is chosen so
 *     that a decoder thread's tensor-core operand fragments are contiguous.
 *     (Version 1 kept the scales and zeros of each area in plain index order; version
 *     2 places them in fragment order, as below.  Images of the two versions are not
 *     interchangeable.)
 *     Per (batch b, kv head h) the cache is a sequence of 32-token block records.
 *     Record of block beta (tokens 32*beta .. 32*beta+31), D = head_dim, nj = D/32:
 *        [K codes: 4*D*bk bytes][K s/z: 4*D bytes][V codes: 4*D*bv][V s/z: 4*D]
 *     Scales and zeros are fp16, placed (byte offsets inside their s/z area):
 *        per-channel K, channel d: k = d/16, e = d%16, t = (e%8)/2, r = e/8, hb = e%2:
 *           scale at 16*(4k + t) + 8r + 2hb, zero at that + 4
 *        per-token K and V, token u of the block, channel group j = d/32:
 *           scale at 8*nj*(u/2) + 4j + 2*(u%2), zero at that + 4*nj
 *     Code areas are two 16-token halves of 2*D*b bytes each.  Token u of the
 *     block lies in half eta = u/16.  Inside a half, every code belongs to one of
 *     32 "lanes" and one half-word "slot" of that lane:
 *        K (role: key operand), token u, channel d:
 *           i = (u%16)/8, gk = u%8, k = d/16, e = d%16,
 *           t = (e%8)/2, r = e/8, hb = e%2,
 *           lane = 4*gk + t, slot = (2*k + i)*2 + r
 *        V (role: value operand), token u, channel d:
 *           e = u%16, t = (e%8)/2, ch = e/8, hb = e%2,
 *           m = d/16, rho = d%16, g = rho%8, rh = rho/8,
 *           lane = 4*g + t, slot = 4*m + 2*ch + rh
 *     Each lane owns Wh = D*b/64 little-endian 32-bit words per half, holding
 *     F = 32/b fields of b bits, LSB first.  A word carries P = F/2 slots: slot
 *     p of the word uses field p for hb = 0 and field p + P for hb = 1.  So a
 *     code sits in lane word w = slot / P at field (slot % P) + hb*P, bit
 *     offset field*b.  Lane words are stored in chunks of c = min(4, Wh) words:
 *        word index in half = ((w / c)*32 + lane)*c + (w % c).
 *     Residual (per-channel K): 32 tokens x D bf16, entry (u, d) at 2*(u*D + d).
 *     Canonical image of a (b, h) unit holding L tokens: records 0..ceil(L/32)-1,
 *     then (per-channel K only) the residual; every byte that holds no token of
 *     0..L-1 is zero (the unfilled part of the last block and of the residual).
 *
 * Q5  Paged INT2/INT4 token-mixed cache ([TRI] Facts: quantizer, leftovers, page
 *     pools, decode path).  Every token carries a tag, 2 or 4.  The INT2-tagged tokens,
 *     in arrival order, form groups of 32: keys per channel with 2 bits, values per token
 *     with 2 bits (a 32-token record as in Q3, bk = bv = 2).  INT4-tagged tokens are
 *     quantized per token, keys and values with 4 bits, into 16-token pages
 *     [K codes 2*D*4 B][K s/z 2*D B][V codes 2*D*4 B][V s/z 2*D B] (the Q3 layouts of one
 *     16-token half).  The n2 mod 32 INT2 tokens after the last complete group are held
 *     the same INT4 way in two pending pages, and their bf16 originals in a 32-slot
 *     staging area (reading: the leftovers go through the INT4 per-token path, values
 *     too, so pages stay homogeneous, until their group of 32 completes).
 *     Canonical image of a (b, h) unit: the INT2 records in group order, the INT4 pages
 *     in order, the two pending pages, then the staging keys and values (32 x D bf16
 *     each); bytes that hold no token are zero.
 *
 * Q4  Attention (fp64): O[hq] = sum_t softmax_t(q . k^_t / sqrt(D)) v^_t over all L
 *     cached tokens, quantized ones and residual alike, no mask; GQA: the kv head
 *     of query head hq is hq / G.
 * ---------------------------------------------------------------------------
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_PER_CHANNEL 0
#define ORC_PER_TOKEN 1

/* ---------------- number formats (IEEE 754 definitions) ---------------- */

/* bf16 bit pattern -> binary32: the bf16 pattern is the top half of a binary32. */
static float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary16 bit pattern -> binary64, from the encoding definition. */
static double orc_f16_to_f64(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/1024) * 2^(e-15) */
    return s ? -v : v;
}

/* binary32 -> binary16, round to nearest, ties to even. */
static uint16_t orc_f32_to_f16(float f) {
    if (isnan(f)) return 0x7E00;
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    double v = fabs((double)f);
    if (v >= 65520.0) return sign | 0x7C00;        /* halfway above 65504 rounds to inf */
    if (v < ldexp(1.0, -14)) {                     /* result grid: multiples of 2^-24 */
        double n = rint(ldexp(v, 24));             /* exact scaling; rint is RNE */
        return sign | (uint16_t)n;                 /* n == 1024 encodes the min normal */
    }
    int ex;
    frexp(v, &ex);                                  /* v = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                                 /* 2^E <= v < 2^(E+1) */
    double n = rint(ldexp(v, 10 - E));              /* significand * 1024, in [1024, 2048] */
    if (n == 2048.0) { n = 1024.0; E += 1; }
    if (E > 15) return sign | 0x7C00;
    return sign | (uint16_t)(((E + 15) << 10) | ((int)n - 1024));
}

/* ---------------- Q1: group quantizer ---------------- */

/* Quantize n values x[i*xs] (binary32) with b bits; writes scale/zero (fp16 bits)
 * and codes[i*cs]. */
static void orc_quant(const float *x, int n, int xs, int bits, uint16_t *s16, uint16_t *z16,
                      uint8_t *codes, int cs) {
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; i++) {
        float v = x[i * xs];
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    float qmax = (float)((1 << bits) - 1);
    float range = mx - mn;                          /* binary32, correctly rounded */
    float s32 = range / qmax;                       /* binary32 IEEE division */
    *s16 = orc_f32_to_f16(s32);
    *z16 = orc_f32_to_f16(mn);
    float s = (float)orc_f16_to_f64(*s16);
    float z = (float)orc_f16_to_f64(*z16);
    for (int i = 0; i < n; i++) {
        uint8_t c = 0;
        if (s != 0.0f) {
            float diff = x[i * xs] - z;
            float qv = diff / s;
            float r = rintf(qv);                    /* default rounding mode: ties to even */
            if (r < 0.0f) r = 0.0f;
            if (r > qmax) r = qmax;
            c = (uint8_t)r;
        }
        codes[i * cs] = c;
    }
}

/* ---------------- Q3: storage format ---------------- */

long orc_record_bytes(int D, int bk, int bv) { return 4L * D * (bk + bv) + 8L * D; }

long orc_unit_image_bytes(int L, int D, int bk, int bv, int kmode) {
    long nblk = (L + 31) / 32;
    long r = nblk * orc_record_bytes(D, bk, bv);
    if (kmode == ORC_PER_CHANNEL) r += 64L * D;    /* residual: 32 tokens x D bf16 */
    return r;
}

/* Byte offset (inside a code area of one block) and bit offset of the code of
 * token u (0..31), channel d, for role 0 = key operand, 1 = value operand. */
static void orc_code_pos(int role, int u, int d, int D, int bits, long *byte_off, int *bit_off) {
    int eta = u / 16, lane, slot, hb;
    if (role == 0) {
        int i = (u % 16) / 8, gk = u % 8, k = d / 16, e = d % 16;
        int t = (e % 8) / 2, r = e / 8;
        hb = e % 2;
        lane = 4 * gk + t;
        slot = (2 * k + i) * 2 + r;
    } else {
        int e = u % 16, t = (e % 8) / 2, ch = e / 8;
        int m = d / 16, rho = d % 16, g = rho % 8, rh = rho / 8;
        hb = e % 2;
        lane = 4 * g + t;
        slot = 4 * m + 2 * ch + rh;
    }
    int F = 32 / bits, P = F / 2;
    int Wh = D * bits / 64;
    int c = Wh < 4 ? Wh : 4;
    int w = slot / P;
    int field = slot % P + hb * P;
    long word = ((long)(w / c) * 32 + lane) * c + (w % c);
    *byte_off = (long)eta * (2L * D * bits) + 4 * word;
    *bit_off = field * bits;
}

static void orc_put_code(uint8_t *area, int role, int u, int d, int D, int bits, unsigned code) {
    long bo;
    int bit;
    orc_code_pos(role, u, d, D, bits, &bo, &bit);
    uint32_t w;
    memcpy(&w, area + bo, 4);
    uint32_t mask = ((1u << bits) - 1u) << bit;
    w = (w & ~mask) | ((code << bit) & mask);
    memcpy(area + bo, &w, 4);
}

/* Position of the code of (u, d) inside a code area (exported for tests). */
void orc_code_position(int role, int u, int d, int D, int bits, long *byte_off, int *bit_off) {
    orc_code_pos(role, u, d, D, bits, byte_off, bit_off);
}

/* Read back the code of (u, d) from a code area (used by tests to decode images). */
unsigned orc_get_code(const uint8_t *area, int role, int u, int d, int D, int bits) {
    long bo;
    int bit;
    orc_code_pos(role, u, d, D, bits, &bo, &bit);
    uint32_t w;
    memcpy(&w, area + bo, 4);
    return (w >> bit) & ((1u << bits) - 1u);
}

/* Offsets of the scale and zero of channel d (per-channel key s/z area). */
static void orc_chan_sz_pos(int d, long *s_off, long *z_off) {
    int k = d / 16, e = d % 16, t = (e % 8) / 2, r = e / 8, hb = e % 2;
    *s_off = 16L * (4 * k + t) + 8 * r + 2 * hb;
    *z_off = *s_off + 4;
}

/* Offsets of the scale and zero of token u, channel group j (per-token s/z area). */
static void orc_tok_sz_pos(int u, int j, int nj, long *s_off, long *z_off) {
    *s_off = 8L * nj * (u / 2) + 4 * j + 2 * (u % 2);
    *z_off = *s_off + 4L * nj;
}

static void put_chan_sz(uint8_t *area, int d, uint16_t s, uint16_t z) {
    long so, zo;
    orc_chan_sz_pos(d, &so, &zo);
    memcpy(area + so, &s, 2);
    memcpy(area + zo, &z, 2);
}

static void put_tok_sz(uint8_t *area, int u, int j, int nj, uint16_t s, uint16_t z) {
    long so, zo;
    orc_tok_sz_pos(u, j, nj, &so, &zo);
    memcpy(area + so, &s, 2);
    memcpy(area + zo, &z, 2);
}

/* Exported for tests: kind 0 = per-channel (index = channel), 1 = per-token
 * (index = token, j = group). */
void orc_sz_position(int kind, int index, int j, int nj, long *s_off, long *z_off) {
    if (kind == 0) orc_chan_sz_pos(index, s_off, z_off);
    else orc_tok_sz_pos(index, j, nj, s_off, z_off);
}

/* ---------------- one (batch, kv-head) unit ---------------- */

/* Quantize one unit's K and V (bf16 bits, [L][D]) and, if img != NULL, write its
 * canonical image; if Kh/Vh != NULL, write the dequantized cache [L][D] (fp64;
 * residual keys are the bf16 inputs themselves). */
int orc_unit(const uint16_t *K, const uint16_t *V, int L, int D, int bk, int bv, int kmode,
             uint8_t *img, double *Kh, double *Vh) {
    if (D % 32 || D <= 0 || L < 0) return -1;
    const int nj = D / 32;
    const long REC = orc_record_bytes(D, bk, bv);
    const long KC = 4L * D * bk, KS = 4L * D, VC = 4L * D * bv;
    const int nblk = (L + 31) / 32;
    const int nfull = L / 32;                       /* complete per-channel key groups */
    if (img) memset(img, 0, (size_t)orc_unit_image_bytes(L, D, bk, bv, kmode));

    float x[32];
    uint8_t c[32];
    uint16_t s16, z16;

    /* values: per token, groups of 32 channels */
    for (int tok = 0; tok < L; tok++) {
        int blk = tok / 32, u = tok % 32;
        for (int j = 0; j < nj; j++) {
            for (int i = 0; i < 32; i++) x[i] = orc_bf16_to_f32(V[(long)tok * D + 32 * j + i]);
            orc_quant(x, 32, 1, bv, &s16, &z16, c, 1);
            if (img) {
                uint8_t *rec = img + blk * REC;
                put_tok_sz(rec + KC + KS + VC, u, j, nj, s16, z16);
                for (int i = 0; i < 32; i++) orc_put_code(rec + KC + KS, 1, u, 32 * j + i, D, bv, c[i]);
            }
            if (Vh) {
                double s = orc_f16_to_f64(s16), z = orc_f16_to_f64(z16);
                for (int i = 0; i < 32; i++) Vh[(long)tok * D + 32 * j + i] = c[i] * s + z;
            }
        }
    }

    if (kmode == ORC_PER_CHANNEL) {
        /* keys: per channel over each complete group of 32 tokens */
        for (int blk = 0; blk < nfull; blk++) {
            for (int d = 0; d < D; d++) {
                for (int i = 0; i < 32; i++) x[i] = orc_bf16_to_f32(K[(long)(32 * blk + i) * D + d]);
                orc_quant(x, 32, 1, bk, &s16, &z16, c, 1);
                if (img) {
                    uint8_t *rec = img + blk * REC;
                    put_chan_sz(rec + KC, d, s16, z16);
                    for (int i = 0; i < 32; i++) orc_put_code(rec, 0, i, d, D, bk, c[i]);
                }
                if (Kh) {
                    double s = orc_f16_to_f64(s16), z = orc_f16_to_f64(z16);
                    for (int i = 0; i < 32; i++) Kh[(long)(32 * blk + i) * D + d] = c[i] * s + z;
                }
            }
        }
        /* the newest L mod 32 tokens stay in the bf16 residual */
        for (int tok = 32 * nfull; tok < L; tok++) {
            int u = tok - 32 * nfull;
            if (img) memcpy(img + nblk * REC + 2L * u * D, K + (long)tok * D, 2L * D);
            if (Kh)
                for (int d = 0; d < D; d++) Kh[(long)tok * D + d] = orc_bf16_to_f32(K[(long)tok * D + d]);
        }
    } else {
        /* keys per token, groups of 32 channels, like values */
        for (int tok = 0; tok < L; tok++) {
            int blk = tok / 32, u = tok % 32;
            for (int j = 0; j < nj; j++) {
                for (int i = 0; i < 32; i++) x[i] = orc_bf16_to_f32(K[(long)tok * D + 32 * j + i]);
                orc_quant(x, 32, 1, bk, &s16, &z16, c, 1);
                if (img) {
                    uint8_t *rec = img + blk * REC;
                    put_tok_sz(rec + KC, u, j, nj, s16, z16);
                    for (int i = 0; i < 32; i++) orc_put_code(rec, 0, u, 32 * j + i, D, bk, c[i]);
                }
                if (Kh) {
                    double s = orc_f16_to_f64(s16), z = orc_f16_to_f64(z16);
                    for (int i = 0; i < 32; i++) Kh[(long)tok * D + 32 * j + i] = c[i] * s + z;
                }
            }
        }
    }
    return 0;
}

/* ---------------- Q5: paged INT2/INT4 unit ---------------- */

void orc_attention(const uint16_t *q, const double *Kh, const double *Vh, int L, int D, int G, double *out);

long orc_paged_page4_bytes(int D) { return 20L * D; }
long orc_paged_rec2_bytes(int D) { return orc_record_bytes(D, 2, 2); }

/* Counts of a tag sequence: complete INT2 groups, INT4 tokens, pending INT2 tokens. */
void orc_paged_counts(const uint8_t *tags, int L, int *n2g, int *n4, int *np) {
    int n2 = 0, c4 = 0;
    for (int i = 0; i < L; i++) {
        if (tags[i] == 2) n2++;
        else c4++;
    }
    *n2g = n2 / 32;
    *np = n2 % 32;
    *n4 = c4;
}

long orc_paged_unit_bytes(const uint8_t *tags, int L, int D) {
    int n2g, n4, np;
    orc_paged_counts(tags, L, &n2g, &n4, &np);
    return n2g * orc_paged_rec2_bytes(D) + ((n4 + 15) / 16 + 2) * orc_paged_page4_bytes(D) + 128L * D;
}

/* Per-token quantization of one token (bits) into slot u of a 16-token page half:
 * codes into the code area (role 0 keys, 1 values), scale/zero into the s/z area. */
static void orc_token_to_page(const uint16_t *row, int D, int bits, int role, uint8_t *codes_area,
                              uint8_t *sz_area, int u, double *deq) {
    const int nj = D / 32;
    float x[32];
    uint8_t c[32];
    uint16_t s16, z16;
    for (int j = 0; j < nj; j++) {
        for (int i = 0; i < 32; i++) x[i] = orc_bf16_to_f32(row[32 * j + i]);
        orc_quant(x, 32, 1, bits, &s16, &z16, c, 1);
        put_tok_sz(sz_area, u, j, nj, s16, z16);
        for (int i = 0; i < 32; i++) orc_put_code(codes_area, role, u, 32 * j + i, D, bits, c[i]);
        if (deq) {
            double s = orc_f16_to_f64(s16), z = orc_f16_to_f64(z16);
            for (int i = 0; i < 32; i++) deq[32 * j + i] = c[i] * s + z;
        }
    }
}

/* One (b, h) unit of the paged cache from its K, V ([L][D] bf16) and tags [L]. */
int orc_paged_unit(const uint16_t *K, const uint16_t *V, const uint8_t *tags, int L, int D, uint8_t *img,
                   double *Kh, double *Vh) {
    if (D % 32 || D <= 0 || D > 512 || L < 0) return -1;
    const int nj = D / 32;
    const long REC2 = orc_paged_rec2_bytes(D), PAGE4 = orc_paged_page4_bytes(D);
    const long KC2 = 4L * D * 2, KS2 = 4L * D, VC2 = 4L * D * 2;
    const long KC4 = 2L * D * 4, KS4 = 2L * D, VC4 = 2L * D * 4;
    int n2g, n4, np;
    orc_paged_counts(tags, L, &n2g, &n4, &np);
    const int n4p = (n4 + 15) / 16;
    int *i2 = (int *)malloc(sizeof(int) * (size_t)(L + 1));
    int *i4 = (int *)malloc(sizeof(int) * (size_t)(L + 1));
    int n2 = 0, c4 = 0;
    for (int i = 0; i < L; i++) {
        if (tags[i] == 2) i2[n2++] = i;
        else i4[c4++] = i;
    }
    if (img) memset(img, 0, (size_t)orc_paged_unit_bytes(tags, L, D));
    uint8_t *pg4 = img ? img + n2g * REC2 : NULL;
    uint8_t *pend = img ? pg4 + n4p * PAGE4 : NULL;
    uint8_t *stage = img ? pend + 2 * PAGE4 : NULL;
    float x[32];
    uint8_t c[32];
    uint16_t s16, z16;

    /* INT2 groups: keys per channel over the group's 32 tokens, values per token */
    for (int g = 0; g < n2g; g++) {
        uint8_t *rec = img ? img + g * REC2 : NULL;
        for (int d = 0; d < D; d++) {
            for (int u = 0; u < 32; u++) x[u] = orc_bf16_to_f32(K[(long)i2[32 * g + u] * D + d]);
            orc_quant(x, 32, 1, 2, &s16, &z16, c, 1);
            if (rec) {
                put_chan_sz(rec + KC2, d, s16, z16);
                for (int u = 0; u < 32; u++) orc_put_code(rec, 0, u, d, D, 2, c[u]);
            }
            if (Kh) {
                double s = orc_f16_to_f64(s16), z = orc_f16_to_f64(z16);
                for (int u = 0; u < 32; u++) Kh[(long)i2[32 * g + u] * D + d] = c[u] * s + z;
            }
        }
        for (int u = 0; u < 32; u++) {
            const int tok = i2[32 * g + u];
            for (int j = 0; j < nj; j++) {
                for (int i = 0; i < 32; i++) x[i] = orc_bf16_to_f32(V[(long)tok * D + 32 * j + i]);
                orc_quant(x, 32, 1, 2, &s16, &z16, c, 1);
                if (rec) {
                    put_tok_sz(rec + KC2 + KS2 + VC2, u, j, nj, s16, z16);
                    for (int i = 0; i < 32; i++) orc_put_code(rec + KC2 + KS2, 1, u, 32 * j + i, D, 2, c[i]);
                }
                if (Vh) {
                    double s = orc_f16_to_f64(s16), z = orc_f16_to_f64(z16);
                    for (int i = 0; i < 32; i++) Vh[(long)tok * D + 32 * j + i] = c[i] * s + z;
                }
            }
        }
    }
    /* INT4 tokens (main pages), then the pending INT2 tokens (pending pages + staging) */
    for (int r = 0; r < n4 + np; r++) {
        const int pending = r >= n4;
        const int tok = pending ? i2[32 * n2g + (r - n4)] : i4[r];
        const int slot = pending ? r - n4 : r;
        uint8_t *page = img ? (pending ? pend : pg4) + (slot / 16) * PAGE4 : NULL;
        const int u = slot % 16;
        uint8_t tmp_codes[4096];
        uint8_t tmp_sz[1024];
        uint8_t *kcodes = page ? page : tmp_codes, *ksz = page ? page + KC4 : tmp_sz;
        uint8_t *vcodes = page ? page + KC4 + KS4 : tmp_codes, *vsz = page ? page + KC4 + KS4 + VC4 : tmp_sz;
        orc_token_to_page(K + (long)tok * D, D, 4, 0, kcodes, ksz, u, Kh ? Kh + (long)tok * D : NULL);
        orc_token_to_page(V + (long)tok * D, D, 4, 1, vcodes, vsz, u, Vh ? Vh + (long)tok * D : NULL);
        if (pending && stage) {
            memcpy(stage + 2L * slot * D, K + (long)tok * D, 2L * D);
            memcpy(stage + 64L * D + 2L * slot * D, V + (long)tok * D, 2L * D);
        }
    }
    free(i2);
    free(i4);
    return 0;
}

/* A whole paged layer: K, V [B][Hkv][L][D], tags [B][L] (shared by heads), Q [B][Hkv*G][D].
 * img: unit images concatenated in (b, h) order; out [B][Hq][D]. */
int orc_paged_layer(const uint16_t *K, const uint16_t *V, const uint8_t *tags, const uint16_t *Q, int B, int Hkv,
                    int G, int L, int D, uint8_t *img, double *out) {
    long *off = (long *)malloc(sizeof(long) * (size_t)(B * Hkv + 1));
    off[0] = 0;
    for (int un = 0; un < B * Hkv; un++) off[un + 1] = off[un] + orc_paged_unit_bytes(tags + (long)(un / Hkv) * L, L, D);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int un = 0; un < B * Hkv; un++) {
        int b = un / Hkv, h = un % Hkv;
        double *Kh = NULL, *Vh = NULL;
        if (out) {
            Kh = (double *)malloc(sizeof(double) * (size_t)L * D);
            Vh = (double *)malloc(sizeof(double) * (size_t)L * D);
        }
        err |= orc_paged_unit(K + (long)un * L * D, V + (long)un * L * D, tags + (long)b * L, L, D,
                              img ? img + off[un] : NULL, Kh, Vh) != 0;
        if (out) {
            orc_attention(Q + ((long)b * Hkv * G + (long)h * G) * D, Kh, Vh, L, D, G,
                          out + ((long)b * Hkv * G + (long)h * G) * D);
            free(Kh);
            free(Vh);
        }
    }
    free(off);
    return err ? -1 : 0;
}

/* ---------------- Q4: attention in binary64 ---------------- */

/* Unnormalised attention of G query heads (q: [G][D] bf16 bits) over tokens
 * [t0, t1) of a dequantized cache: m = max score, l = sum exp(score - m),
 * acc[g][d] = sum exp(score - m) * v^[d].  Scores are q.k^/sqrt(D). */
void orc_attention_partial(const uint16_t *q, const double *Kh, const double *Vh, int t0, int t1,
                           int D, int G, double *m, double *l, double *acc) {
    const double scale = 1.0 / sqrt((double)D);
    double *sc = (double *)malloc(sizeof(double) * (size_t)(t1 > t0 ? t1 - t0 : 1));
    for (int g = 0; g < G; g++) {
        double mx = -INFINITY;
        for (int t = t0; t < t1; t++) {
            double s = 0.0;
            for (int d = 0; d < D; d++) s += (double)orc_bf16_to_f32(q[g * D + d]) * Kh[(long)t * D + d];
            s *= scale;
            sc[t - t0] = s;
            if (s > mx) mx = s;
        }
        double sum = 0.0;
        for (int d = 0; d < D; d++) acc[g * D + d] = 0.0;
        for (int t = t0; t < t1; t++) {
            double p = exp(sc[t - t0] - mx);
            sum += p;
            for (int d = 0; d < D; d++) acc[g * D + d] += p * Vh[(long)t * D + d];
        }
        m[g] = mx;
        l[g] = sum;
    }
    free(sc);
}

/* Log-sum-exp merge of S partials ([S][G], [S][G], [S][G][D]) into out [G][D]
 * ([TRI] Facts: splits merged by online log-sum-exp). */
void orc_merge_partials(int S, int G, int D, const double *m, const double *l, const double *acc,
                        double *out) {
    for (int g = 0; g < G; g++) {
        double M = -INFINITY;
        for (int s = 0; s < S; s++)
            if (m[s * G + g] > M) M = m[s * G + g];
        double den = 0.0;
        for (int d = 0; d < D; d++) out[g * D + d] = 0.0;
        for (int s = 0; s < S; s++) {
            if (m[s * G + g] == -INFINITY) continue;   /* empty partial */
            double w = exp(m[s * G + g] - M);
            den += w * l[s * G + g];
            for (int d = 0; d < D; d++) out[g * D + d] += w * acc[((long)s * G + g) * D + d];
        }
        for (int d = 0; d < D; d++) out[g * D + d] /= den;
    }
}

/* Softmax attention over all L tokens: out [G][D]. */
void orc_attention(const uint16_t *q, const double *Kh, const double *Vh, int L, int D, int G,
                   double *out) {
    double *m = (double *)malloc(sizeof(double) * G);
    double *l = (double *)malloc(sizeof(double) * G);
    double *acc = (double *)malloc(sizeof(double) * (size_t)G * D);
    orc_attention_partial(q, Kh, Vh, 0, L, D, G, m, l, acc);
    orc_merge_partials(1, G, D, m, l, acc, out);
    free(m);
    free(l);
    free(acc);
}

/* ---------------- a whole layer ---------------- */

/* K, V: [B][Hkv][L][D] bf16 bits; Q: [B][Hkv*G][D] bf16 bits (query head hq uses
 * kv head hq / G).  img (nullable): unit images concatenated in (b, h) order.
 * out (nullable): [B][Hkv*G][D] binary64.  Units run in parallel (OpenMP). */
int orc_layer(const uint16_t *K, const uint16_t *V, const uint16_t *Q, int B, int Hkv, int G, int L,
              int D, int bk, int bv, int kmode, uint8_t *img, double *out) {
    if (L < 1 && out) return -1;
    const long unit_img = orc_unit_image_bytes(L, D, bk, bv, kmode);
    const int units = B * Hkv;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int un = 0; un < units; un++) {
        int b = un / Hkv, h = un % Hkv;
        const uint16_t *Ku = K + (long)un * L * D;
        const uint16_t *Vu = V + (long)un * L * D;
        double *Kh = NULL, *Vh = NULL;
        if (out) {
            Kh = (double *)malloc(sizeof(double) * (size_t)L * D);
            Vh = (double *)malloc(sizeof(double) * (size_t)L * D);
        }
        err |= orc_unit(Ku, Vu, L, D, bk, bv, kmode, img ? img + un * unit_img : NULL, Kh, Vh) != 0;
        if (out) {
            orc_attention(Q + ((long)b * Hkv * G + (long)h * G) * D, Kh, Vh, L, D, G,
                          out + ((long)b * Hkv * G + (long)h * G) * D);
            free(Kh);
            free(Vh);
        }
    }
    return err ? -1 : 0;
}

/* ---------------- threads (timing only; no effect on any result) ---------------- */

#ifdef _OPENMP
#include <omp.h>
#endif
/* Threads of the OpenMP loops above (n <= 0: the runtime's default); returns the count. */
int orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ---------------- exported scalar helpers (for pins) ---------------- */

void orc_f32_to_f16_array(const float *x, uint16_t *out, long n) {
    for (long i = 0; i < n; i++) out[i] = orc_f32_to_f16(x[i]);
}
void orc_f16_to_f64_array(const uint16_t *h, double *out, long n) {
    for (long i = 0; i < n; i++) out[i] = orc_f16_to_f64(h[i]);
}
/* Quantize many groups: x [ngroups][32] binary32 -> s16, z16 [ngroups], codes [ngroups][32]. */
void orc_quant_groups(const float *x, long ngroups, int bits, uint16_t *s16, uint16_t *z16,
                      uint8_t *codes) {
    for (long g = 0; g < ngroups; g++) orc_quant(x + g * 32, 32, 1, bits, s16 + g, z16 + g, codes + g * 32, 1);
}
int orc_format_version(void) { return 2; }
