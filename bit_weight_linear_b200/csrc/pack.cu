// pack.cu -- offline weight packers.
//
// Ternary: BitNet b1.58 page ("微软、国科大开启1Bit时代…"), "BitNet b1.58 介绍"
// (weights in {-1,0,1}) and "内存和延迟" (2-bit storage): one 2-bit field per
// weight holding t+1, 16 fields per 32-bit word, field i at bits 2i..2i+1.
// Sign: OneBit page ("清华、哈工大把大模型压缩到了1bit…"), "3. 通过知识蒸馏迁移原模型
// 能力" (save the post-Sign() parameters) and "讨论与分析 / 1. 效率" (one 0/1 bit
// per parameter): bit i of a word is 1 iff sign(w) = +1, sign(+-0) = +1.
//
// Both are one thread per output word with 16-byte coalesced loads; they are
// HBM-bound (ternary: 16 B read + 4 B written per word, sign: 64 B + 4 B).
#include "common.cuh"
#include "kernels.h"

namespace bl {

__global__ void __launch_bounds__(256) pack_ternary_kernel(const int8_t* __restrict__ w,
                                                           size_t nwords,
                                                           uint32_t* __restrict__ w2,
                                                           unsigned int* __restrict__ err) {
    size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    if (i >= nwords) return;
    // K % 16 == 0, so word i covers input bytes [16 i, 16 i + 16) of the row-major matrix.
    uint4 v = ld_stream_v4(w + 16 * i);
    uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t word = 0;
    bool bad = false;
#pragma unroll
    for (int b = 0; b < 16; ++b) {
        int t = (int)(int8_t)((in[b >> 2] >> (8 * (b & 3))) & 0xffu);
        bad |= (t < -1) | (t > 1);
        word |= (uint32_t)((t + 1) & 3) << (2 * b);
    }
    w2[i] = word;
    if (bad) atomicOr(err, 1u);
}

__global__ void __launch_bounds__(256) pack_sign_kernel(const uint16_t* __restrict__ w,
                                                        size_t nwords,
                                                        uint32_t* __restrict__ s1,
                                                        unsigned int* __restrict__ err) {
    size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    if (i >= nwords) return;
    const uint16_t* src = w + 32 * i;  // K % 32 == 0
    uint32_t word = 0;
    bool bad = false;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 v = ld_stream_v4(src + 8 * c);
        uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            uint32_t hbits = (in[e >> 1] >> (16 * (e & 1))) & 0xffffu;
            uint32_t mag = hbits & 0x7fffu;
            bool neg = (hbits & 0x8000u) && mag != 0;   // -0 counts as +1
            bad |= mag > 0x7c00u;                       // NaN
            word |= (neg ? 0u : 1u) << (8 * c + e);
        }
    }
    s1[i] = word;
    if (bad) atomicOr(err, 1u);
}

cudaError_t launch_pack_ternary(const int8_t* w, int N, int K, uint32_t* w2,
                                unsigned int* err_flag, cudaStream_t s) {
    size_t nwords = (size_t)N * (size_t)(K / 16);
    if (nwords == 0) return cudaSuccess;
    unsigned blocks = (unsigned)((nwords + 255) / 256);
    pack_ternary_kernel<<<blocks, 256, 0, s>>>(w, nwords, w2, err_flag);
    return cudaGetLastError();
}

cudaError_t launch_pack_sign(const uint16_t* w, int N, int K, uint32_t* s1,
                             unsigned int* err_flag, cudaStream_t s) {
    size_t nwords = (size_t)N * (size_t)(K / 32);
    if (nwords == 0) return cudaSuccess;
    unsigned blocks = (unsigned)((nwords + 255) / 256);
    pack_sign_kernel<<<blocks, 256, 0, s>>>(w, nwords, s1, err_flag);
    return cudaGetLastError();
}

}  // namespace bl
