// act_groups.cuh -- per-group activation preparation shared by the decode
// kernels (stream.cu, chain.cu): absmax of a group and its quantisation into
// the permuted byte order the weight unpack produces.
//   BitLinear (BitNet b1.58 page, "BitNet b1.58 介绍"): q = rne(x * rn(127/amax)).
//   OneBit (OneBit page, "1. 新的 1bit 结构"): the fixed-point image of x*g in
//   three int8 limbs (common.cuh).
#pragma once

#include <cstdint>

#include "common.cuh"
#include "decode_forms.cuh"

namespace bl {

// Quantise one 16-element ternary group (fp16 in a, b) into the permuted
// activation tile; returns the group's sum of q.
// |x * inv| <= 127 (1 + 2^-24) for inv = rn(127/amax), so the rounded value
// never leaves [-127, 127] and no clamp is needed.
__device__ __forceinline__ int quant_group_t(uint4 a, uint4 b, float inv, uint8_t* dst) {
    const uint32_t hv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    int qv[16];   // low bytes = q
#pragma unroll
    for (int e = 0; e < 16; ++e)
        qv[e] = rne_bits(__fmul_rn(hbits(hv[e >> 1] >> (16 * (e & 1))), inv));
    uint4 o;
    o.x = pack4(qv[0], qv[4], qv[8], qv[12]);
    o.y = pack4(qv[1], qv[5], qv[9], qv[13]);
    o.z = pack4(qv[2], qv[6], qv[10], qv[14]);
    o.w = pack4(qv[3], qv[7], qv[11], qv[15]);
    *reinterpret_cast<uint4*>(dst) = o;
    int sum = __dp4a((int)o.x, 0x01010101, 0);
    sum = __dp4a((int)o.y, 0x01010101, sum);
    sum = __dp4a((int)o.z, 0x01010101, sum);
    return __dp4a((int)o.w, 0x01010101, sum);
}

// Quantise one 8-element half (elements 8h .. 8h+7 of a 16-element group,
// fp16 in a) into the group's permuted bytes at dst: element 4b+j goes to byte
// 4j+b, so half h fills bytes 4j + 2h + {0,1} of every word j.  Returns the
// half's sum of q.  (The other half of the group is written by another call.)
__device__ __forceinline__ int quant_half_group_t(uint4 a, float inv, uint8_t* dst, int h) {
    const uint32_t hv[4] = {a.x, a.y, a.z, a.w};
    int qv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[e] = rne_bits(__fmul_rn(hbits(hv[e >> 1] >> (16 * (e & 1))), inv));
    // element 8h + e = 4b + j with b = 2h + (e >> 2), j = e & 3: byte 4j + 2h + (e >> 2)
    uint16_t* d16 = reinterpret_cast<uint16_t*>(dst);
    int sum = 0;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const uint32_t lo = (uint32_t)qv[jj] & 0xffu, hi = (uint32_t)qv[4 + jj] & 0xffu;
        d16[2 * jj + h] = (uint16_t)(lo | (hi << 8));
        sum += (int)(int8_t)lo + (int)(int8_t)hi;
    }
    return sum;
}

__device__ __forceinline__ uint32_t absmax_bits_t(uint4 a) {
    const uint32_t mb = __vmaxu2(__vmaxu2(a.x & 0x7fff7fffu, a.y & 0x7fff7fffu),
                                 __vmaxu2(a.z & 0x7fff7fffu, a.w & 0x7fff7fffu));
    return max(mb & 0xffffu, mb >> 16);
}

// max |x*g| over 8 elements (fp32 products, exact for fp16 inputs)
__device__ __forceinline__ float absmax_prod(uint4 a, uint4 gg) {
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {gg.x, gg.y, gg.z, gg.w};
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e)
        mx = fmaxf(mx, fabsf(__fmul_rn(hbits(av[e >> 1] >> (16 * (e & 1))),
                                       hbits(gv[e >> 1] >> (16 * (e & 1))))));
    return mx;
}

// OneBit: one 32-element group of x*g -> X = rne(x*g*inv), split into three
// int8 limbs written permuted into the limb rows dh, dh + astride, dh + 2
// astride (byte 4j+b of the group holds element 8b+j); ls receives the
// group's sum of each limb.  |x*g*inv| < kImgMax + 0.25, so no clamp is needed.
__device__ __forceinline__ void quant_group_s(const uint4 (&xa)[4], const uint4 (&ga)[4], float inv,
                                              uint8_t* dh, int astride, int (&ls)[3]) {
    uint32_t hw[8], mw[8], lw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) hw[j] = mw[j] = lw[j] = 0;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const uint32_t av[4] = {xa[v].x, xa[v].y, xa[v].z, xa[v].w};
        const uint32_t gv[4] = {ga[v].x, ga[v].y, ga[v].z, ga[v].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float pr = __fmul_rn(hbits(av[e >> 1] >> (16 * (e & 1))),
                                       hbits(gv[e >> 1] >> (16 * (e & 1))));
            const int X = rne_bits(__fmul_rn(pr, inv)) - kRneBias;   // |X| <= kImgMax
            int hi, mid, lo;
            split_limbs(X, hi, mid, lo);
            // element 8v+e goes to byte v of word e
            hw[e] |= ((uint32_t)hi & 0xffu) << (8 * v);
            mw[e] |= ((uint32_t)mid & 0xffu) << (8 * v);
            lw[e] |= ((uint32_t)lo & 0xffu) << (8 * v);
        }
    }
    int sh = 0, sm = 0, sl = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        sh = __dp4a((int)hw[j], 0x01010101, sh);
        sm = __dp4a((int)mw[j], 0x01010101, sm);
        sl = __dp4a((int)lw[j], 0x01010101, sl);
    }
    uint4* h4 = reinterpret_cast<uint4*>(dh);
    uint4* m4 = reinterpret_cast<uint4*>(dh + astride);
    uint4* l4 = reinterpret_cast<uint4*>(dh + 2 * astride);
    h4[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    h4[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    m4[0] = make_uint4(mw[0], mw[1], mw[2], mw[3]);
    m4[1] = make_uint4(mw[4], mw[5], mw[6], mw[7]);
    l4[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    l4[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    ls[0] = sh;
    ls[1] = sm;
    ls[2] = sl;
}

}  // namespace bl
