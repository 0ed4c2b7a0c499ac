// billm.cu -- the two-plane binary layer of BiLLM's residual approximation.
//
// BiLLM page ("BiLLM: Pushing the Limit of Post-Training Quantization for
// LLMs"), section "方法细节：残差近似与最优断点拆分", step 2: W is binarised
// once (alpha_o B_o) and its residual once more (alpha_r B_r), so
//     y = x (alpha_o (.) B_o + alpha_r (.) B_r)^T
//       = alpha_o (.) (x B_o^T) + alpha_r (.) (x B_r^T)
// with one scale per output row (the reading taken here) and fp16
// activations that are not quantised.  The layer is stored as the two sign
// planes stacked into one s1 matrix [2N, K/32] (B_o rows, then B_r rows) and
// the scales as one fp16 vector [2N] (alpha_o, then alpha_r): exactly a OneBit
// layer of 2N rows with g = 1 and h = alpha.  So the contraction runs on the
// OneBit kernels (exact integer contraction of a 23-bit image of x), which
// also write the fp32 products z (.) h; this file adds
//   billm_combine_kernel   y[m][n] = fp16(zf[m][n] + zf[m][N + n])
//   billm_binarize_kernel  the residual binarisation of a weight on the device
#include "common.cuh"
#include "kernels.h"

namespace bl {
namespace {

constexpr int kBinThreads = 256;

// y = fp16(zf[:, :N] + zf[:, N:]), four outputs per thread (N % 16 == 0)
__global__ void __launch_bounds__(256) billm_combine_kernel(const float* __restrict__ zf, int M, int N,
                                                            uint16_t* __restrict__ y) {
    const int q = N / 4;                 // float4 groups per output row
    const size_t total = (size_t)M * q;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t m = i / q, c = i - m * q;
        const float4 a = __ldcs(reinterpret_cast<const float4*>(zf + m * 2 * N) + c);
        const float4 b = __ldcs(reinterpret_cast<const float4*>(zf + m * 2 * N + N) + c);
        const uint32_t lo = (uint32_t)__half_as_ushort(__float2half_rn(__fadd_rn(a.x, b.x))) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(__fadd_rn(a.y, b.y))) << 16);
        const uint32_t hi = (uint32_t)__half_as_ushort(__float2half_rn(__fadd_rn(a.z, b.z))) |
                            ((uint32_t)__half_as_ushort(__float2half_rn(__fadd_rn(a.w, b.w))) << 16);
        reinterpret_cast<uint2*>(y + m * N)[c] = make_uint2(lo, hi);
    }
}

// fixed-order CTA sum of one double per thread (result valid in every thread)
__device__ double block_sum_f64(double v, double* sm) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();                      // sm may still be read from a previous call
    if (lane == 0) sm[warp] = v;
    __syncthreads();
    double s = 0.0;
    for (int w = 0; w < kBinThreads / 32; ++w) s += sm[w];
    return s;
}

// One CTA per row n: alpha_o = mean |W[n]|, B_o = sign(W[n]); residual
// R = W[n] - alpha_o B_o, alpha_r = mean |R|, B_r = sign(R)  (sign(0) = +1),
// all in fp64.  Each thread packs whole 32-element words.
__global__ void __launch_bounds__(kBinThreads) billm_binarize_kernel(const float* __restrict__ W, int N,
                                                                     int K, uint32_t* __restrict__ b2,
                                                                     uint16_t* __restrict__ alpha,
                                                                     double* ao_out, double* ar_out,
                                                                     unsigned int* bad_flag) {
    __shared__ double sm[kBinThreads / 32];
    const int n = blockIdx.x;
    const float* row = W + (size_t)n * K;
    const int words = K / 32;
    double sa = 0.0;
    bool bad = false;
    for (int w = threadIdx.x; w < words; w += kBinThreads) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 v = *reinterpret_cast<const float4*>(row + 32 * w + 4 * c);
            const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                bad |= !isfinite(e[j]);
                sa += fabs((double)e[j]);
            }
        }
    }
    if (bad) atomicOr(bad_flag, 1u);
    const double ao = block_sum_f64(sa, sm) / (double)K;
    double sr = 0.0;
    for (int w = threadIdx.x; w < words; w += kBinThreads) {
        uint32_t wo = 0, wr = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 v = *reinterpret_cast<const float4*>(row + 32 * w + 4 * c);
            const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const double b = e[j] < 0.0f ? -1.0 : 1.0;
                const double r = (double)e[j] - ao * b;
                sr += fabs(r);
                wo |= (e[j] < 0.0f ? 0u : 1u) << (4 * c + j);
                wr |= (r < 0.0 ? 0u : 1u) << (4 * c + j);
            }
        }
        b2[(size_t)n * words + w] = wo;
        b2[((size_t)N + n) * words + w] = wr;
    }
    const double ar = block_sum_f64(sr, sm) / (double)K;
    if (threadIdx.x == 0) {
        alpha[n] = __half_as_ushort(__double2half(ao));
        alpha[N + n] = __half_as_ushort(__double2half(ar));
        if (ao_out) ao_out[n] = ao;
        if (ar_out) ar_out[n] = ar;
    }
}

}  // namespace

cudaError_t launch_billm_combine(const float* zf, int M, int N, uint16_t* y, cudaStream_t s) {
    const size_t groups = (size_t)M * (N / 4);
    if (groups == 0) return cudaSuccess;
    const int sms = device_sm_count();
    size_t blocks = (groups + 255) / 256;
    const size_t cap = (size_t)(sms > 0 ? sms : 148) * 8;
    if (blocks > cap) blocks = cap;
    billm_combine_kernel<<<(unsigned)blocks, 256, 0, s>>>(zf, M, N, y);
    return cudaGetLastError();
}

cudaError_t launch_billm_binarize(const float* W, int N, int K, uint32_t* b2, uint16_t* alpha,
                                  double* ao, double* ar, unsigned int* bad_flag, cudaStream_t s) {
    if (N == 0) return cudaSuccess;
    billm_binarize_kernel<<<N, kBinThreads, 0, s>>>(W, N, K, b2, alpha, ao, ar, bad_flag);
    return cudaGetLastError();
}

}  // namespace bl
