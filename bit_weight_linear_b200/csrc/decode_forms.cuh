// decode_forms.cuh -- per-form constants and small helpers shared by the
// decode-shaped kernels (stream.cu, chain.cu).
//
// Packed weight words: ternary 16 codes of 2 bits (code = t + 1), sign 32 bits
// (1 = +1).  The byte-SIMD unpack (w >> shift*j) & mask yields, in register j,
// the elements {j, P+j, 2P+j, 3P+j} of the word (P = 4 ternary, 8 sign), so the
// activations are stored permuted within 16- (ternary) or 32-byte (sign) groups:
// byte 4j+b of a group holds element P*b + j.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace bl {

template <int FORM>
struct DF;
template <>
struct DF<0> {  // ternary, 2-bit codes
    static constexpr int kPerWord = 16, kRegs = 4, kShift = 2, kStepK = 256, kChunkK = 64;
    static constexpr int kCPT = 1, kGroup = 16;
    static constexpr uint32_t kMask = 0x03030303u;
};
template <>
struct DF<1> {  // sign, 1 bit; three activation columns (int8 limbs hi, mid, lo) per token
    static constexpr int kPerWord = 32, kRegs = 8, kShift = 1, kStepK = 512, kChunkK = 128;
    static constexpr int kCPT = 3, kGroup = 32;
    static constexpr uint32_t kMask = 0x01010101u;
};

// low bytes of a, b, c, d -> one word (a in the lowest byte)
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
    const uint32_t lo = __byte_perm((uint32_t)a, (uint32_t)b, 0x0040);
    const uint32_t hi = __byte_perm((uint32_t)c, (uint32_t)d, 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

__device__ __forceinline__ float hbits(uint32_t v) {
    return __half2float(__ushort_as_half((unsigned short)(v & 0xffffu)));
}

}  // namespace bl
