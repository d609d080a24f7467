// Device helpers shared by the append kernels: the group quantizer and the v2 storage
// format's positions (see include/kvq.h).  Each quantizer step is one correctly rounded
// binary32 operation; nothing here is contracted into FMA.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace kvq {
namespace quant {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Scale/zero of a group from its min and max (stored fp16 values and their floats).
__device__ __forceinline__ void group_params(float mn, float mx, int bits, float &s, float &z,
                                             uint16_t &s16, uint16_t &z16) {
    const float qmax = static_cast<float>((1 << bits) - 1);
    const float s32 = __fdiv_rn(__fsub_rn(mx, mn), qmax);
    const __half sh = __float2half_rn(s32);
    const __half zh = __float2half_rn(mn);
    s = __half2float(sh);
    z = __half2float(zh);
    s16 = __half_as_ushort(sh);
    z16 = __half_as_ushort(zh);
}

__device__ __forceinline__ int group_code(float x, float s, float z, int bits) {
    if (s == 0.0f) return 0;
    const int c = __float2int_rn(__fdiv_rn(__fsub_rn(x, z), s));
    return max(0, min(c, (1 << bits) - 1));
}

// Owner (token in half e, channel d) of field f of lane word w, for the key operand
// role (role 0) or the value operand role (role 1) of the v2 format.
__device__ __forceinline__ void field_owner(int role, int lane, int w, int f, int bits, int &e,
                                            int &d) {
    const int P = 16 / bits;
    const int slot = w * P + (f % P), hb = f / P;
    const int g = lane >> 2, t = lane & 3;
    if (role == 0) {   // slot = (2k + i)*2 + r ; lane = 4*(u%8) + t ; channel = 16k + 8r + 2t + hb
        const int r = slot & 1, i = (slot >> 1) & 1, k = slot >> 2;
        e = 8 * i + g;
        d = 16 * k + 8 * r + 2 * t + hb;
    } else {           // slot = 4m + 2ch + rh ; lane = 4*g + t ; token = 8ch + 2t + hb
        const int rh = slot & 1, ch = (slot >> 1) & 1, m = slot >> 2;
        e = 8 * ch + 2 * t + hb;
        d = 16 * m + g + 8 * rh;
    }
}

// Word index (inside a half's code area) and bit offset of the code of token e (0..15
// inside the half), channel d, for the key operand role (role 0) or the value operand
// role (role 1) of the v2 format: the inverse of field_owner.
__device__ __forceinline__ void code_place(int role, int e, int d, int D, int bits, int &word, int &bit) {
    const int P = 16 / bits;
    int lane, slot, hb;
    if (role == 0) {   // token e = 8i + gk, channel d = 16k + 8r + 2t + hb
        const int i = e >> 3, gk = e & 7, k = d >> 4, ee = d & 15;
        const int t = (ee & 7) >> 1, r = ee >> 3;
        hb = ee & 1;
        lane = 4 * gk + t;
        slot = (2 * k + i) * 2 + r;
    } else {           // token e = 8ch + 2t + hb, channel d = 16m + g + 8rh
        const int t = (e & 7) >> 1, ch = e >> 3, m = d >> 4, rho = d & 15;
        const int g = rho & 7, rh = rho >> 3;
        hb = e & 1;
        lane = 4 * g + t;
        slot = 4 * m + 2 * ch + rh;
    }
    const int Wh = D * bits / 64, c = Wh < 4 ? Wh : 4;
    const int w = slot / P, field = slot % P + hb * P;
    word = ((w / c) * 32 + lane) * c + (w % c);
    bit = field * bits;
}

// Byte offsets of a scale/zero pair in the s/z areas of the v2 format.
__device__ __forceinline__ int chan_sz_off(int d) {   // per-channel keys: scale; zero at +4
    const int k = d >> 4, e = d & 15;
    return 16 * (4 * k + ((e & 7) >> 1)) + 8 * (e >> 3) + 2 * (e & 1);
}
__device__ __forceinline__ int tok_sz_off(int u, int j, int nj) {   // per token: scale; zero at +4*nj
    return 8 * nj * (u >> 1) + 4 * j + 2 * (u & 1);
}

// Memory word index inside a half's code area -> (lane, lane word).
__device__ __forceinline__ void word_lane(int widx, int Wh, int &lane, int &w) {
    const int c = Wh < 4 ? Wh : 4;
    const int chunk = widx / (32 * c), rem = widx % (32 * c);
    lane = rem / c;
    w = chunk * c + rem % c;
}


}  // namespace quant
}  // namespace kvq
