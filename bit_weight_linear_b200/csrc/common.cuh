// common.cuh -- device helpers shared by the library's kernels (sm_100a).
// Hand-written inline PTX for the legacy warp-level integer MMA and for
// streaming loads; no generated code is embedded here.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace bl {

// Bits of the per-device condition word that bl_device_status() reads and
// clears (kernels receive its address as an argument).
constexpr unsigned int kFlagTimeout = 1u;

// D = A * B + D for one m16n8k32 tile: A is u8 [16 x 32] (row), B is s8
// [32 x 8] (col), D is s32 [16 x 8].  Fragment layout per the PTX ISA:
//   a0: row g,   k 4t..4t+3      a1: row g+8, k 4t..4t+3
//   a2: row g,   k 16+4t..+3     a3: row g+8, k 16+4t..+3
//   b0: col g,   k 4t..4t+3      b1: col g,   k 16+4t..+3
//   d0,d1: row g, cols 2t,2t+1   d2,d3: row g+8, cols 2t,2t+1
// with g = lane/4 and t = lane%4.
__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte load that bypasses L1 allocation: packed weights are read exactly
// once per launch, so they should not evict the reused activations.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte read-only load through L1 (activations, reused by many CTAs).
__device__ __forceinline__ uint4 ld_ro_v4(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// A chunk of 8 elements of a OneBit input value vector; g == nullptr stands
// for g = 1 (the two-plane binary layer, whose inputs are not scaled).
__device__ __forceinline__ uint4 ld_gvec(const uint16_t* g, size_t off) {
    return g ? ld_ro_v4(g + off) : make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Round-to-nearest-even of an fp32 value t with |t| < 2^22, as the bit
// pattern of rn(t + 1.5 * 2^23): that sum has an ulp of 1, so its low mantissa
// bits hold rne(t) (ties go to the even sum, i.e. the even integer) and its
// low byte is rne(t) mod 256.  One full-rate add instead of a float-to-int
// conversion.  The add is separately rounded (__fadd_rn is never contracted
// with the preceding __fmul_rn), which keeps the two-step rounding.
__device__ __forceinline__ int rne_bits(float t) { return __float_as_int(__fadd_rn(t, 12582912.0f)); }
constexpr int kRneBias = 0x4B400000;   // the bit pattern of 1.5 * 2^23

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ long long warp_sum64(long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// OneBit fixed-point image of a token's x*g (fp32 products, exact for fp16
// inputs): X = rne(x*g * rn(kImgMax / amax')), amax' = max_k |x*g|, so
// |X| <= kImgMax = 2^22 - 1.  The fp32 product exceeds kImgMax by at most
// kImgMax * 2^-24 < 0.25 and rounds back to kImgMax; and |t| < 2^22 is the
// range in which rne_bits is exact.  The image's error is at most
// amax' / (2 kImgMax) ~ 1.2e-7 amax' per element.
constexpr int kImgMax = 4194303;
constexpr float kImgMaxF = 4194303.0f;

// Balanced base-256 digits of an image value: X = 65536 hi + 256 mid + lo with
// every digit in [-128, 127] (hi in [-64, 64] for |X| <= kImgMax), so each
// digit is an int8 MMA operand and each limb's contraction is exact in int32.
__device__ __forceinline__ void split_limbs(int X, int& hi, int& mid, int& lo) {
    const int x1 = (X + 128) >> 8;   // arithmetic shift = floor
    lo = X - 256 * x1;
    hi = (x1 + 128) >> 8;
    mid = x1 - 256 * hi;
}

// sum X*S from the three limbs' 0/1-bit contractions D_l = sum limb_l * b
// (b = (S+1)/2) and the token's image sum sum X:
//   sum X*S = 2 (65536 D_hi + 256 D_mid + D_lo) - sum X      (exact in int64)
__device__ __forceinline__ long long limb_combine(int d_hi, int d_mid, int d_lo, long long xsum) {
    const long long P = 65536ll * d_hi + 256ll * d_mid + (long long)d_lo;
    return 2 * P - xsum;
}

}  // namespace bl
