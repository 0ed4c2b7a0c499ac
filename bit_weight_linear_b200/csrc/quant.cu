// quant.cu -- per-token activation preparation kernels.
//
// BitLinear: BitNet b1.58 page ("微软、国科大开启1Bit时代…"), "BitNet b1.58 介绍":
// activations are quantised per token to [-Qb, Qb], Qb = 127, with no zero
// point.  Exact fp32 sequence (shared with the ABI's statement of the op):
//   amax = max_k |x|, inv = 127 / amax (IEEE division), q = rne(x * inv)
//   clamped to +-127, scale = amax / 127; an all-zero token gives 0, 0.
//
// OneBit: OneBit page ("清华、哈工大把大模型压缩到了1bit…"), "1. 新的 1bit 结构":
// the input-side value vector g multiplies x before the sign contraction.  The
// product x*g (exact in fp32: two 11-bit significands) is turned into a
// per-token 23-bit fixed-point image X = rne(x*g * (2^22-1) / amax'), split
// into three signed bytes X = 65536 hi + 256 mid + lo (balanced base-256
// digits), so that the contraction with the 0/1 sign bits runs exactly in int8
// MMA, one limb at a time.
//
// One CTA per token, two passes over the token (the second hits L1/L2).
// HBM-bound: the plain/ternary kernels read 2 B and write 1 B per element.
#include "common.cuh"
#include "kernels.h"
#include "tc_prims.cuh"

namespace bl {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// max over the block of a non-negative float carried as its bit pattern
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t r = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) r = max(r, red[w]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ int block_sum_i32(int v, int* red) {
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int r = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) r += red[w];
    return r;
}

// Zero the consumer's arrival counters (CTA 0 only; called after the PDL wait,
// so the previous user of the counters has finished).
__device__ __forceinline__ void zero_words(unsigned int* zero, int n_zero) {
    if (zero != nullptr && blockIdx.x == 0)
        for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0u;
}

__device__ __forceinline__ float half_bits_to_float(uint32_t bits) {
    return __half2float(__ushort_as_half((unsigned short)(bits & 0xffffu)));
}

// |x * inv| <= 127 (1 + 2^-24) for inv = rn(127/amax): the code never leaves
// [-127, 127], so no clamp is needed
__device__ __forceinline__ int quant127(float xv, float inv) {
    return rne_bits(__fmul_rn(xv, inv)) - kRneBias;
}

// Layout 0: natural order.  Layout 1: the decode kernel's order, a 4x4 byte
// transpose inside every 16-byte group (byte 4j+b holds element 4b+j), which
// matches the byte order the 2-bit unpack (w >> 2j) & 0x03030303 produces.
template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) quant_act_kernel(const uint16_t* __restrict__ x,
                                                             int K, int8_t* __restrict__ q,
                                                             float* __restrict__ scale,
                                                             int32_t* __restrict__ qsum,
                                                             unsigned int* zero, int n_zero) {
    __shared__ uint32_t redu[kWarps];
    __shared__ int redi[kWarps];
    const int m = blockIdx.x;
    const uint16_t* row = x + (size_t)m * K;
    // programmatic dependent launch: let the consumer start streaming its
    // weights, and read x / write the outputs only after the producer of x is done
    tc::pdl_trigger();
    tc::pdl_wait();
    zero_words(zero, n_zero);

    // pass 1: amax as the max of |x| bit patterns (monotone for finite halves)
    uint32_t mx = 0;
    for (int c = threadIdx.x; c < K / 8; c += kThreads) {
        uint4 v = tc::ld_v4(row + 8 * c);
        mx = __vmaxu2(mx, v.x & 0x7fff7fffu);
        mx = __vmaxu2(mx, v.y & 0x7fff7fffu);
        mx = __vmaxu2(mx, v.z & 0x7fff7fffu);
        mx = __vmaxu2(mx, v.w & 0x7fff7fffu);
    }
    mx = max(mx & 0xffffu, mx >> 16);
    const float amax = half_bits_to_float(block_max_u32(mx, redu));
    const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;

    // pass 2: quantise 16 elements per step, store 16 bytes
    int sum = 0;
    int8_t* qrow = q + (size_t)m * K;
    for (int c = threadIdx.x; c < K / 16; c += kThreads) {
        uint4 a = tc::ld_v4(row + 16 * c);
        uint4 b = tc::ld_v4(row + 16 * c + 8);
        uint32_t hv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        int qv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            qv[e] = quant127(half_bits_to_float(hv[e >> 1] >> (16 * (e & 1))), inv);
            sum += qv[e];
        }
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t wv = 0;
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                int src = LAYOUT == 0 ? 4 * j + bb : 4 * bb + j;
                wv |= ((uint32_t)qv[src] & 0xffu) << (8 * bb);
            }
            out[j] = wv;
        }
        *reinterpret_cast<uint4*>(qrow + 16 * c) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (LAYOUT == 1) {
        int tot = block_sum_i32(sum, redi);
        if (threadIdx.x == 0) qsum[m] = tot;
    }
    if (threadIdx.x == 0) scale[m] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
}

// Register-resident variant: a 512-thread CTA per token loads the whole token
// into registers (NCH 16-element chunks per thread, all loads in flight at
// once), takes amax, then quantises from registers.  One read of x instead of
// two, and no loop-carried load latency; used while K <= 16 * 512 * 8.
constexpr int kRegThreads = 512;
constexpr int kRegMaxChunks = 8;

template <int NW>
__device__ __forceinline__ uint32_t block_max_u32_n(uint32_t v, uint32_t* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t r = red[lane < NW ? lane : 0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r = max(r, __shfl_xor_sync(0xffffffffu, r, o));
    return r;
}

template <int NW>
__device__ __forceinline__ int block_sum_i32_n(int v, int* red) {
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    return warp_sum(lane < NW ? red[lane] : 0);
}

template <int LAYOUT, int NCH>
__global__ void __launch_bounds__(kRegThreads, NCH <= 4 ? 2 : 1)
    quant_act_reg_kernel(const uint16_t* __restrict__ x, int K, int8_t* __restrict__ q,
                         float* __restrict__ scale, int32_t* __restrict__ qsum,
                         unsigned int* zero, int n_zero) {
    constexpr int NW = kRegThreads / 32;
    __shared__ uint32_t redu[NW];
    __shared__ int redi[NW];
    const int m = blockIdx.x;
    const int nc = K / 16;
    const uint16_t* row = x + (size_t)m * K;
    tc::pdl_trigger();
    tc::pdl_wait();
    zero_words(zero, n_zero);

    uint4 va[NCH], vb[NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = threadIdx.x + i * kRegThreads;
        if (c < nc) {
            va[i] = tc::ld_v4(row + 16 * c);
            vb[i] = tc::ld_v4(row + 16 * c + 8);
        } else {
            va[i] = make_uint4(0, 0, 0, 0);
            vb[i] = va[i];
        }
    }
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        mx = __vmaxu2(mx, va[i].x & 0x7fff7fffu);
        mx = __vmaxu2(mx, va[i].y & 0x7fff7fffu);
        mx = __vmaxu2(mx, va[i].z & 0x7fff7fffu);
        mx = __vmaxu2(mx, va[i].w & 0x7fff7fffu);
        mx = __vmaxu2(mx, vb[i].x & 0x7fff7fffu);
        mx = __vmaxu2(mx, vb[i].y & 0x7fff7fffu);
        mx = __vmaxu2(mx, vb[i].z & 0x7fff7fffu);
        mx = __vmaxu2(mx, vb[i].w & 0x7fff7fffu);
    }
    mx = max(mx & 0xffffu, mx >> 16);
    const float amax = half_bits_to_float(block_max_u32_n<NW>(mx, redu));
    const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;

    int sum = 0;
    int8_t* qrow = q + (size_t)m * K;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = threadIdx.x + i * kRegThreads;
        if (c >= nc) break;
        const uint32_t hv[8] = {va[i].x, va[i].y, va[i].z, va[i].w,
                                vb[i].x, vb[i].y, vb[i].z, vb[i].w};
        int qv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            qv[e] = quant127(half_bits_to_float(hv[e >> 1] >> (16 * (e & 1))), inv);
            sum += qv[e];
        }
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t wv = 0;
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int src = LAYOUT == 0 ? 4 * j + bb : 4 * bb + j;
                wv |= ((uint32_t)qv[src] & 0xffu) << (8 * bb);
            }
            out[j] = wv;
        }
        *reinterpret_cast<uint4*>(qrow + 16 * c) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (LAYOUT == 1) {
        const int tot = block_sum_i32_n<NW>(sum, redi);
        if (threadIdx.x == 0) qsum[m] = tot;
    }
    if (threadIdx.x == 0) scale[m] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
}

// Store one 32-element group's three limb bytes, permuted: byte 4j+b of the
// 32-byte group holds element 8b+j, the order the 1-bit unpack
// (w >> j) & 0x01010101 produces.  Plane stride K bytes: [hi][mid][lo].
// Returns the group's sum of X.
__device__ __forceinline__ int store_limbs_group(const int (&X)[32], int8_t* hi_dst, int K) {
    uint32_t hw[8], mw[8], lw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) hw[j] = mw[j] = lw[j] = 0u;
    int sum = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        int hi, mid, lo;
        split_limbs(X[e], hi, mid, lo);
        hw[e & 7] |= ((uint32_t)hi & 0xffu) << (8 * (e >> 3));
        mw[e & 7] |= ((uint32_t)mid & 0xffu) << (8 * (e >> 3));
        lw[e & 7] |= ((uint32_t)lo & 0xffu) << (8 * (e >> 3));
        sum += X[e];
    }
    uint4* hd = reinterpret_cast<uint4*>(hi_dst);
    uint4* md = reinterpret_cast<uint4*>(hi_dst + K);
    uint4* ld = reinterpret_cast<uint4*>(hi_dst + 2 * (size_t)K);
    hd[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    hd[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    md[0] = make_uint4(mw[0], mw[1], mw[2], mw[3]);
    md[1] = make_uint4(mw[4], mw[5], mw[6], mw[7]);
    ld[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    ld[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    return sum;
}

template <int NW>
__device__ __forceinline__ long long block_sum_i64_n(long long v, long long* red) {
    v = warp_sum64(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    return warp_sum64(lane < NW ? red[lane] : 0ll);
}

// OneBit preparation, general K (two passes over the token): the image of
// x*g in three int8 limb planes [M][3][K], the fixed-point step amax'/kImgMax
// and the token's image sum (int64; per thread at most 256 elements of
// |X| <= 2^22, so the per-thread int32 sums cannot overflow).
__global__ void __launch_bounds__(kThreads) prep_onebit_kernel(const uint16_t* __restrict__ x,
                                                               const uint16_t* __restrict__ g,
                                                               int K, int8_t* __restrict__ planes,
                                                               float* __restrict__ step,
                                                               long long* __restrict__ tsum,
                                                               unsigned int* zero, int n_zero) {
    __shared__ uint32_t redu[kWarps];
    __shared__ long long redl[kWarps];
    const int m = blockIdx.x;
    const uint16_t* row = x + (size_t)m * K;
    tc::pdl_trigger();
    tc::pdl_wait();
    zero_words(zero, n_zero);

    float mx = 0.f;
    for (int c = threadIdx.x; c < K / 8; c += kThreads) {
        uint4 v = tc::ld_v4(row + 8 * c);
        uint4 gv = ld_gvec(g, 8 * c);
        uint32_t xs[4] = {v.x, v.y, v.z, v.w}, gs[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float p = __fmul_rn(half_bits_to_float(xs[e >> 1] >> (16 * (e & 1))),
                                half_bits_to_float(gs[e >> 1] >> (16 * (e & 1))));
            mx = fmaxf(mx, fabsf(p));
        }
    }
    const float amax = __uint_as_float(block_max_u32(__float_as_uint(mx), redu));
    const float inv = amax > 0.f ? __fdiv_rn(kImgMaxF, amax) : 0.f;

    int sum = 0;
    int8_t* hi_row = planes + (size_t)m * 3 * K;
    for (int c = threadIdx.x; c < K / 32; c += kThreads) {
        int X[32];
#pragma unroll
        for (int part = 0; part < 4; ++part) {
            uint4 v = tc::ld_v4(row + 32 * c + 8 * part);
            uint4 gv = ld_gvec(g, 32 * c + 8 * part);
            uint32_t xs[4] = {v.x, v.y, v.z, v.w}, gs[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float p = __fmul_rn(half_bits_to_float(xs[e >> 1] >> (16 * (e & 1))),
                                    half_bits_to_float(gs[e >> 1] >> (16 * (e & 1))));
                X[8 * part + e] = rne_bits(__fmul_rn(p, inv)) - kRneBias;   // |X| <= kImgMax
            }
        }
        sum += store_limbs_group(X, hi_row + 32 * c, K);
    }
    const long long tot = block_sum_i64_n<kWarps>((long long)sum, redl);
    if (threadIdx.x == 0) {
        tsum[m] = tot;
        step[m] = amax > 0.f ? __fdiv_rn(amax, kImgMaxF) : 0.f;
    }
}

// Register-resident OneBit preparation: a 512-thread CTA per token keeps the
// fp32 products x*g of up to NCH 32-element groups per thread in registers,
// takes amax, then forms the limbs from registers (x and g read once).  Same
// arithmetic and output as prep_onebit_kernel.
template <int NCH>
__global__ void __launch_bounds__(kRegThreads, 1)
    prep_onebit_reg_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ g, int K,
                           int8_t* __restrict__ planes, float* __restrict__ step,
                           long long* __restrict__ tsum, unsigned int* zero, int n_zero) {
    constexpr int NW = kRegThreads / 32;
    __shared__ uint32_t redu[NW];
    __shared__ long long redl[NW];
    const int m = blockIdx.x;
    const int ng = K / 32;
    const uint16_t* row = x + (size_t)m * K;
    tc::pdl_trigger();
    tc::pdl_wait();
    zero_words(zero, n_zero);

    float pr[NCH][32];
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = threadIdx.x + i * kRegThreads;
        if (c < ng) {
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                const uint4 v = tc::ld_v4(row + 32 * c + 8 * part);
                const uint4 gv = ld_gvec(g, 32 * c + 8 * part);
                const uint32_t xs[4] = {v.x, v.y, v.z, v.w}, gs[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    pr[i][8 * part + e] = __fmul_rn(half_bits_to_float(xs[e >> 1] >> (16 * (e & 1))),
                                                    half_bits_to_float(gs[e >> 1] >> (16 * (e & 1))));
                    mx = fmaxf(mx, fabsf(pr[i][8 * part + e]));
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) pr[i][e] = 0.f;
        }
    }
    const float amax = __uint_as_float(block_max_u32_n<NW>(__float_as_uint(mx), redu));
    const float inv = amax > 0.f ? __fdiv_rn(kImgMaxF, amax) : 0.f;

    int sum = 0;
    int8_t* hi_row = planes + (size_t)m * 3 * K;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = threadIdx.x + i * kRegThreads;
        if (c >= ng) break;
        int X[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) X[e] = rne_bits(__fmul_rn(pr[i][e], inv)) - kRneBias;
        sum += store_limbs_group(X, hi_row + 32 * c, K);
    }
    const long long tot = block_sum_i64_n<NW>((long long)sum, redl);
    if (threadIdx.x == 0) {
        tsum[m] = tot;
        step[m] = amax > 0.f ? __fdiv_rn(amax, kImgMaxF) : 0.f;
    }
}

template <auto KERN, int THREADS = kThreads, typename... Args>
cudaError_t launch_pdl(int blocks, cudaStream_t s, Args... args) {
    static KernelAttrs kattrs;  // one per kernel
    if (cudaError_t e = kattrs.ensure(KERN, 0)) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(THREADS);
    cfg.stream = s;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, KERN, args...);
}

// chunks of 16 elements per thread for the register-resident kernel, 0 = too long
inline int reg_chunks(int K) {
    const int need = (K / 16 + kRegThreads - 1) / kRegThreads;
    for (int c = 1; c <= kRegMaxChunks; c *= 2)
        if (need <= c) return c;
    return 0;
}

template <int LAYOUT>
cudaError_t launch_quant(const uint16_t* x, int M, int K, int8_t* q, float* scale,
                         int32_t* qsum, unsigned int* zero, int n_zero, cudaStream_t s) {
    switch (reg_chunks(K)) {
        case 1: return launch_pdl<quant_act_reg_kernel<LAYOUT, 1>, kRegThreads>(M, s, x, K, q, scale, qsum, zero, n_zero);
        case 2: return launch_pdl<quant_act_reg_kernel<LAYOUT, 2>, kRegThreads>(M, s, x, K, q, scale, qsum, zero, n_zero);
        case 4: return launch_pdl<quant_act_reg_kernel<LAYOUT, 4>, kRegThreads>(M, s, x, K, q, scale, qsum, zero, n_zero);
        case 8: return launch_pdl<quant_act_reg_kernel<LAYOUT, 8>, kRegThreads>(M, s, x, K, q, scale, qsum, zero, n_zero);
        default: return launch_pdl<quant_act_kernel<LAYOUT>>(M, s, x, K, q, scale, qsum, zero, n_zero);
    }
}

}  // namespace

cudaError_t launch_quant_plain(const uint16_t* x, int M, int K, int8_t* q, float* scale,
                               cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    return launch_quant<0>(x, M, K, q, scale, (int32_t*)nullptr, (unsigned int*)nullptr, 0, s);
}

cudaError_t launch_quant_ternary_perm(const uint16_t* x, int M, int K, int8_t* qp,
                                      float* scale, int32_t* qsum, cudaStream_t s,
                                      unsigned int* zero, int n_zero) {
    if (M == 0) return cudaSuccess;
    return launch_quant<1>(x, M, K, qp, scale, qsum, zero, n_zero, s);
}

cudaError_t launch_prep_onebit(const uint16_t* x, const uint16_t* g, int M, int K,
                               int8_t* planes, float* step, long long* tsum, cudaStream_t s,
                               unsigned int* zero, int n_zero) {
    if (M == 0) return cudaSuccess;
    const int groups = K / 32;
    if (groups <= kRegThreads)
        return launch_pdl<prep_onebit_reg_kernel<1>, kRegThreads>(M, s, x, g, K, planes, step, tsum, zero, n_zero);
    if (groups <= 2 * kRegThreads)
        return launch_pdl<prep_onebit_reg_kernel<2>, kRegThreads>(M, s, x, g, K, planes, step, tsum, zero, n_zero);
    return launch_pdl<prep_onebit_kernel>(M, s, x, g, K, planes, step, tsum, zero, n_zero);
}

}  // namespace bl
