// skinny.cu -- decode-shaped (small M) packed-weight contraction on the
// warp-level int8 tensor-core MMA (m16n8k32, u8 x s8 -> s32).
//
// BitLinear (BitNet b1.58 page, "BitNet b1.58 介绍" / "能耗"): the ternary
// weight t = code - 1 with code in {0,1,2} stored in 2 bits, so
//     sum_k q*t = sum_k q*code - sum_k q,
// and the codes are fed to the MMA as unsigned bytes straight from a
// byte-SIMD unpack, (w >> 2j) & 0x03030303 -- four weights per two integer ops,
// no multiplies by weights anywhere.
// OneBit (OneBit page, "1. 新的 1bit 结构" and "讨论与分析 / 1. 效率": matrix
// products become bit assignment and addition): with b = (S+1)/2 in {0,1},
//     sum_k X*S = 2 sum_k X*b - sum_k X,
// where X is the 23-bit fixed-point image of x*g split into three int8 limbs
// (each limb contracted exactly in int32), and the bits are unpacked as
// (w >> j) & 0x01010101.
//
// Because integer sums are exact in any order, the k order inside the MMA is
// free: the activation preparation kernels store each 16-byte (ternary) or
// 32-byte (sign) group already transposed to match the unpacked byte order,
// so every operand register comes from one aligned load.
//
// Work split: a CTA owns 16 weight rows (one m16 tile) and a group of tokens;
// its 8 warps split K in steps (256 k ternary, 512 k sign, 16 words per row
// per step, one 16-byte load per lane per row), then reduce through shared
// memory.  The kernel is HBM-bound on the packed weights for M up to 8
// (ternary) / 2 (OneBit) tokens per MMA column tile.
#include "common.cuh"
#include "kernels.h"

namespace bl {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

template <int FORM>
struct Form;

template <>
struct Form<0> {                         // ternary, 2-bit codes
    static constexpr int kPerWord = 16;  // weights per 32-bit word
    static constexpr int kRegs = 4;      // int8x4 registers unpacked per word
    static constexpr int kShift = 2;
    static constexpr uint32_t kMask = 0x03030303u;
    static constexpr int kStepK = 256;   // k per warp step (16 words per row)
    static constexpr int kChunkK = 64;   // k per lane per row per step (4 words)
    static constexpr int kColsPerToken = 1;
};

template <>
struct Form<1> {                         // sign, 1 bit
    static constexpr int kPerWord = 32;
    static constexpr int kRegs = 8;
    static constexpr int kShift = 1;
    static constexpr uint32_t kMask = 0x01010101u;
    static constexpr int kStepK = 512;
    static constexpr int kChunkK = 128;
    static constexpr int kColsPerToken = 3;  // hi, mid and lo limb of the fixed-point image
};

struct SkinnyParams {
    const uint32_t* w;      // packed weights [N][K / kPerWord]
    const int8_t* act;      // prepared activations [M][kColsPerToken][K] (permuted)
    const float* scale;     // ternary: token scale; onebit: fixed-point step
    const int32_t* rsum;    // ternary: sum_k q
    const long long* xsum;  // onebit: sum_k X
    const uint16_t* h;      // onebit output value vector [N]
    float w_scale;          // ternary per-tensor weight scale
    int M, K, N;
    uint16_t* y;            // fp16 [M][N]
    int32_t* acc_out;       // ternary optional int32 [M][N]
    float* zf;              // onebit optional fp32 [M][N] copy of y before fp16 rounding
};

template <int FORM, int NT>
__global__ void __launch_bounds__(kThreads) skinny_kernel(const SkinnyParams p) {
    using F = Form<FORM>;
    constexpr int kTokPerCta = NT * 8 / F::kColsPerToken;
    __shared__ int red[kWarps][NT][16][8];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int row0 = blockIdx.x * 16 + g;
    const int tok_base = blockIdx.y * kTokPerCta;
    const int K = p.K;
    const size_t wpr = (size_t)(K / F::kPerWord);
    const uint32_t* w0 = p.w + (size_t)row0 * wpr + 4 * t;
    const uint32_t* w1 = w0 + 8 * wpr;

    // B operand source for this lane's column in each n8 tile
    const int8_t* bsrc[NT];
    bool bvalid[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + g;
        const int tok = tok_base + col / F::kColsPerToken;
        const int plane = col % F::kColsPerToken;
        // (OneBit: the columns past the last whole token of the tile stay unused)
        bvalid[nt] = tok < p.M && col < kTokPerCta * F::kColsPerToken;
        bsrc[nt] = p.act + ((size_t)(bvalid[nt] ? tok : 0) * F::kColsPerToken + plane) * K +
                   t * F::kChunkK;
    }

    int acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;

    const int nsteps = (K + F::kStepK - 1) / F::kStepK;
    for (int s = warp; s < nsteps; s += kWarps) {
        const bool lane_ok = s * F::kStepK + t * F::kChunkK < K;
        uint4 a0 = make_uint4(0, 0, 0, 0), a1 = make_uint4(0, 0, 0, 0);
        if (lane_ok) {
            a0 = ld_stream_v4(w0 + 16 * s);
            a1 = ld_stream_v4(w1 + 16 * s);
        }
        const uint32_t r0[4] = {a0.x, a0.y, a0.z, a0.w};
        const uint32_t r1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int om = 0; om < 4; ++om) {
            uint32_t u0[F::kRegs], u1[F::kRegs];
#pragma unroll
            for (int j = 0; j < F::kRegs; ++j) {
                u0[j] = (r0[om] >> (F::kShift * j)) & F::kMask;
                u1[j] = (r1[om] >> (F::kShift * j)) & F::kMask;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                uint32_t b[F::kRegs];
                if (lane_ok && bvalid[nt]) {
                    const int8_t* src = bsrc[nt] + (size_t)s * F::kStepK + om * (4 * F::kRegs);
#pragma unroll
                    for (int v = 0; v < F::kRegs / 4; ++v) {
                        uint4 bv = ld_ro_v4(src + 16 * v);
                        b[4 * v + 0] = bv.x;
                        b[4 * v + 1] = bv.y;
                        b[4 * v + 2] = bv.z;
                        b[4 * v + 3] = bv.w;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < F::kRegs; ++j) b[j] = 0;
                }
#pragma unroll
                for (int j = 0; j < F::kRegs; j += 2)
                    mma_u8s8_16832(acc[nt], u0[j], u1[j], u0[j + 1], u1[j + 1], b[j], b[j + 1]);
            }
        }
    }

#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        red[warp][nt][g][2 * t] = acc[nt][0];
        red[warp][nt][g][2 * t + 1] = acc[nt][1];
        red[warp][nt][g + 8][2 * t] = acc[nt][2];
        red[warp][nt][g + 8][2 * t + 1] = acc[nt][3];
    }
    __syncthreads();

    if (FORM == 0) {
        // one output per (token column, row); consecutive threads -> consecutive rows
        for (int o = threadIdx.x; o < NT * 8 * 16; o += kThreads) {
            const int col = o >> 4, r = o & 15;
            const int tok = tok_base + col;
            if (tok >= p.M) continue;
            int sum = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) sum += red[w][col >> 3][r][col & 7];
            const int accv = sum - p.rsum[tok];
            const int n = blockIdx.x * 16 + r;
            const float v = __fmul_rn(__fmul_rn((float)accv, p.scale[tok]), p.w_scale);
            p.y[(size_t)tok * p.N + n] = __half_as_ushort(__float2half_rn(v));
            if (p.acc_out) p.acc_out[(size_t)tok * p.N + n] = accv;
        }
    } else {
        for (int o = threadIdx.x; o < kTokPerCta * 16; o += kThreads) {
            const int u = o >> 4, r = o & 15;
            const int tok = tok_base + u;
            if (tok >= p.M) continue;
            int d[3];
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                const int c = 3 * u + l;
                int v = 0;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) v += red[w][c >> 3][r][c & 7];
                d[l] = v;
            }
            const long long Z = limb_combine(d[0], d[1], d[2], p.xsum[tok]);  // sum_k X * S
            const int n = blockIdx.x * 16 + r;
            const float z = __fmul_rn(p.scale[tok], (float)Z);
            const float hv = __half2float(__ushort_as_half(p.h[n]));
            const float zh = __fmul_rn(z, hv);
            p.y[(size_t)tok * p.N + n] = __half_as_ushort(__float2half_rn(zh));
            if (p.zf) p.zf[(size_t)tok * p.N + n] = zh;
        }
    }
}

template <int FORM, int NT>
cudaError_t launch(const SkinnyParams& p, cudaStream_t s) {
    constexpr int kTokPerCta = NT * 8 / Form<FORM>::kColsPerToken;
    dim3 grid(p.N / 16, (p.M + kTokPerCta - 1) / kTokPerCta);
    static KernelAttrs kattrs;
    if (cudaError_t e = kattrs.ensure(skinny_kernel<FORM, NT>, 0)) return e;
    skinny_kernel<FORM, NT><<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ternary_skinny(const uint32_t* w2, const int8_t* qp, const float* scale,
                                  const int32_t* qsum, int M, int K, int N, float w_scale,
                                  uint16_t* y, int32_t* acc_out, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    SkinnyParams p{w2, qp, scale, qsum, nullptr, nullptr, w_scale, M, K, N, y, acc_out, nullptr};
    if (M <= 8) return launch<0, 1>(p, s);
    if (M <= 16) return launch<0, 2>(p, s);
    return launch<0, 4>(p, s);
}

cudaError_t launch_onebit_skinny(const uint32_t* s1, const int8_t* planes, const float* step,
                                 const long long* tsum, const uint16_t* h, int M, int K, int N,
                                 uint16_t* y, cudaStream_t s, float* zf) {
    if (M == 0 || N == 0) return cudaSuccess;
    SkinnyParams p{s1, planes, step, nullptr, tsum, h, 0.f, M, K, N, y, nullptr, zf};
    if (M <= 2) return launch<1, 1>(p, s);
    if (M <= 5) return launch<1, 2>(p, s);
    return launch<1, 4>(p, s);
}

}  // namespace bl
