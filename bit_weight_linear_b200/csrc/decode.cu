// decode.cu -- fused decode-shaped (small M) forward of both layer forms:
// activation preparation + packed-weight contraction + epilogue in ONE kernel.
//
// Arithmetic is the same as the two-kernel path (quant.cu + skinny.cu):
//   BitLinear (BitNet b1.58 page, "BitNet b1.58 介绍"): per-token absmax int8
//     q = rne(x * (127/amax)), acc = sum q*code - sum q, y = fp16((acc*s)*w_scale);
//   OneBit (OneBit page, "1. 新的 1bit 结构"): 16-bit fixed-point image X of
//     x*g in two int8 limbs, sum X*S = 2 sum X*b - sum X, y = fp16(step*Z*h).
//
// B200 structure (one CTA = 16 weight rows x all of K, 8 warps):
//   1. At launch, one thread issues bulk async copies (cp.async.bulk) of the
//      CTA's whole 16-row packed-weight slab into shared memory, then the grid
//      releases its dependents (programmatic dependent launch), so the next
//      call's weights start streaming while this call computes.
//   2. griddepcontrol.wait -- only now is x (the previous call's output, in a
//      model) read.
//   3. Activation preparation is split over an 8-CTA thread-block cluster:
//      CTA r handles every 8th group of 16 (ternary) / 32 (sign) inputs.  The
//      per-token absmax and the per-token row sums are exchanged through
//      distributed shared memory, and each quantised, permuted group is stored
//      into all eight CTAs' activation tiles (st.shared::cluster), so x is read
//      once per cluster instead of once per CTA.
//   4. The contraction runs from shared memory on the warp-level u8 x s8 MMA
//      (byte-SIMD unpack as in skinny.cu), warps split K, and reduce through
//      shared memory for the epilogue.
// Shared-memory rows are padded by 16 bytes so that the 8 row groups a warp
// reads land on different banks.
#include "common.cuh"
#include "kernels.h"
#include "tc_prims.cuh"

namespace bl {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kCluster = 8;
constexpr int kMaxTok = 32;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

template <int FORM>
struct DF;
template <>
struct DF<0> {
    static constexpr int kPerWord = 16, kRegs = 4, kShift = 2, kStepK = 256, kChunkK = 64;
    static constexpr int kCPT = 1, kGroup = 16;
    static constexpr uint32_t kMask = 0x03030303u;
};
template <>
struct DF<1> {
    static constexpr int kPerWord = 32, kRegs = 8, kShift = 1, kStepK = 512, kChunkK = 128;
    static constexpr int kCPT = 2, kGroup = 32;
    static constexpr uint32_t kMask = 0x01010101u;
};

struct DecodeParams {
    const uint16_t* x;
    const uint16_t* g;      // OneBit input value vector
    const uint16_t* h;      // OneBit output value vector
    const uint32_t* w;      // packed weights
    float w_scale;
    int M, K, N;
    uint16_t* y;
    int32_t* acc_out;
    unsigned int* flags;
};

struct DecodeLayout {
    int wstride, astride, off_a, off_red, off_tok, off_bar, total;
};

template <int FORM, int NT>
__host__ __device__ inline DecodeLayout decode_layout(int M, int K) {
    DecodeLayout l;
    l.wstride = K / DF<FORM>::kPerWord * 4 + 16;
    l.astride = K + 16;
    l.off_a = 16 * l.wstride;
    l.off_red = l.off_a + M * DF<FORM>::kCPT * l.astride;
    l.off_tok = l.off_red + kWarps * NT * 16 * 8 * 4;       // contraction partials
    // token scratch: warp partials (2 x kWarps x kMaxTok) + cluster partials
    // (2 x kCluster x kMaxTok), 4 bytes each
    l.off_bar = l.off_tok + 4 * (2 * kWarps * kMaxTok + 2 * kCluster * kMaxTok);
    l.total = l.off_bar + 16;
    return l;
}

__device__ __forceinline__ float hbits(uint32_t v) {
    return __half2float(__ushort_as_half((unsigned short)(v & 0xffffu)));
}

template <int FORM, int NT>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
    using F = DF<FORM>;
    extern __shared__ __align__(16) uint8_t smem[];
    const DecodeLayout L = decode_layout<FORM, NT>(p.M, p.K);
    const int K = p.K, M = p.M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sb = tc::smem_u32(smem);
    const uint32_t bar = sb + L.off_bar;
    float* red_max = reinterpret_cast<float*>(smem + L.off_tok);             // [kWarps][kMaxTok]
    int* red_sum = reinterpret_cast<int*>(red_max + kWarps * kMaxTok);       // [kWarps][kMaxTok]
    float* cl_max = reinterpret_cast<float*>(red_sum + kWarps * kMaxTok);    // [kCluster][kMaxTok]
    int* cl_sum = reinterpret_cast<int*>(cl_max + kCluster * kMaxTok);       // [kCluster][kMaxTok]
    const int rg = blockIdx.x;                 // 16-row group
    const bool has_rows = rg * 16 < p.N;       // trailing CTAs of the last cluster may be idle
    const int wbytes = K / F::kPerWord * 4;    // packed bytes per weight row

    // 1. stream this CTA's weight slab into shared memory (independent of x)
    if (threadIdx.x == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_fence_init();
        if (has_rows) {
            tc::mbar_arrive_expect_tx(bar, (uint32_t)(16 * wbytes));
            const uint8_t* src = reinterpret_cast<const uint8_t*>(p.w) + (size_t)rg * 16 * wbytes;
            for (int r = 0; r < 16; ++r)
                tc::bulk_g2s(sb + r * L.wstride, src + (size_t)r * wbytes, (uint32_t)wbytes, bar);
        }
    }
    // every CTA of the cluster must be running before any distributed
    // shared-memory store; the matching wait comes just before the first one
    tc::cluster_arrive_relaxed();
    tc::pdl_trigger();
    tc::pdl_wait();

    // 2-3. cluster-split activation preparation
    const uint32_t rank = tc::cluster_ctarank();
    const int ngroups = K / F::kGroup;
    constexpr int G = F::kGroup;
    // pass A: per-token max |x| (ternary) or |x*g| (OneBit) over this CTA's groups
    for (int m = 0; m < M; ++m) {
        float mx = 0.f;
        for (int i = (int)rank + kCluster * threadIdx.x; i < ngroups; i += kCluster * kThreads) {
            const uint16_t* xs = p.x + (size_t)m * K + (size_t)i * G;
#pragma unroll
            for (int v = 0; v < G / 8; ++v) {
                uint4 a = tc::ld_v4(xs + 8 * v);
                const uint32_t av[4] = {a.x, a.y, a.z, a.w};
                if (FORM == 0) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(hbits(av[e >> 1] >> (16 * (e & 1)))));
                } else {
                    uint4 gg = tc::ld_v4(p.g + (size_t)i * G + 8 * v);
                    const uint32_t gv[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        mx = fmaxf(mx, fabsf(__fmul_rn(hbits(av[e >> 1] >> (16 * (e & 1))),
                                                       hbits(gv[e >> 1] >> (16 * (e & 1))))));
                }
            }
        }
        mx = warp_max(mx);
        if (lane == 0) red_max[warp * kMaxTok + m] = mx;
    }
    __syncthreads();
    tc::cluster_wait();
    if (threadIdx.x < M) {
        float mx = 0.f;
        for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, red_max[w * kMaxTok + threadIdx.x]);
        const uint32_t off = tc::smem_u32(cl_max + rank * kMaxTok + threadIdx.x);
        for (int d = 0; d < kCluster; ++d) tc::st_cluster_u32(tc::mapa(off, d), __float_as_uint(mx));
    }
    tc::cluster_sync();

    // pass B: quantise this CTA's groups into every CTA's activation tile
    for (int m = 0; m < M; ++m) {
        float amax = 0.f;
        for (int r = 0; r < kCluster; ++r) amax = fmaxf(amax, cl_max[r * kMaxTok + m]);
        int sum = 0;
        for (int i = (int)rank + kCluster * threadIdx.x; i < ngroups; i += kCluster * kThreads) {
            const uint16_t* xs = p.x + (size_t)m * K + (size_t)i * G;
            if (FORM == 0) {
                const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
                int qv[16];
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    uint4 a = tc::ld_v4(xs + 8 * v);
                    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        int r = __float2int_rn(__fmul_rn(hbits(av[e >> 1] >> (16 * (e & 1))), inv));
                        r = min(127, max(-127, r));
                        qv[8 * v + e] = r;
                        sum += r;
                    }
                }
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t wv = 0;
#pragma unroll
                    for (int bb = 0; bb < 4; ++bb) wv |= ((uint32_t)qv[4 * bb + j] & 0xffu) << (8 * bb);
                    o[j] = wv;
                }
                const uint32_t off = sb + L.off_a + m * L.astride + i * G;
                const uint4 val = make_uint4(o[0], o[1], o[2], o[3]);
                for (int d = 0; d < kCluster; ++d) tc::st_cluster_v4(tc::mapa(off, d), val);
            } else {
                constexpr int kFix = 32639;
                const float inv = amax > 0.f ? __fdiv_rn((float)kFix, amax) : 0.f;
                int hv[32], lv[32];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 a = tc::ld_v4(xs + 8 * v);
                    uint4 gg = tc::ld_v4(p.g + (size_t)i * G + 8 * v);
                    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float pr = __fmul_rn(hbits(av[e >> 1] >> (16 * (e & 1))),
                                                   hbits(gv[e >> 1] >> (16 * (e & 1))));
                        int X = __float2int_rn(__fmul_rn(pr, inv));
                        X = min(kFix, max(-kFix, X));
                        const int hi = (X + 128) >> 8;
                        hv[8 * v + e] = hi;
                        lv[8 * v + e] = X - 256 * hi;
                        sum += X;
                    }
                }
                uint32_t ho[8], lo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t a = 0, b = 0;
#pragma unroll
                    for (int bb = 0; bb < 4; ++bb) {
                        a |= ((uint32_t)hv[8 * bb + j] & 0xffu) << (8 * bb);
                        b |= ((uint32_t)lv[8 * bb + j] & 0xffu) << (8 * bb);
                    }
                    ho[j] = a;
                    lo[j] = b;
                }
                const uint32_t offh = sb + L.off_a + (2 * m) * L.astride + i * G;
                const uint32_t offl = offh + L.astride;
                for (int d = 0; d < kCluster; ++d) {
                    tc::st_cluster_v4(tc::mapa(offh, d), make_uint4(ho[0], ho[1], ho[2], ho[3]));
                    tc::st_cluster_v4(tc::mapa(offh + 16, d), make_uint4(ho[4], ho[5], ho[6], ho[7]));
                    tc::st_cluster_v4(tc::mapa(offl, d), make_uint4(lo[0], lo[1], lo[2], lo[3]));
                    tc::st_cluster_v4(tc::mapa(offl + 16, d), make_uint4(lo[4], lo[5], lo[6], lo[7]));
                }
            }
        }
        sum = warp_sum(sum);
        if (lane == 0) red_sum[warp * kMaxTok + m] = sum;
    }
    __syncthreads();
    if (threadIdx.x < M) {
        int s = 0;
        for (int w = 0; w < kWarps; ++w) s += red_sum[w * kMaxTok + threadIdx.x];
        const uint32_t off = tc::smem_u32(cl_sum + rank * kMaxTok + threadIdx.x);
        for (int d = 0; d < kCluster; ++d) tc::st_cluster_u32(tc::mapa(off, d), (uint32_t)s);
    }
    tc::cluster_sync();
    // From here on no CTA touches another CTA's shared memory.
    if (!has_rows) return;

    const bool w_ok = __syncthreads_and(tc::mbar_wait(bar, 0, p.flags, kWaitLimitNs));
    if (!w_ok) return;

    // 4. contraction from shared memory
    const int g = lane >> 2, t = lane & 3;
    const uint8_t* w0 = smem + g * L.wstride + 16 * t;
    const uint8_t* w1 = w0 + 8 * L.wstride;
    const int ncols = M * F::kCPT;
    const uint8_t* bsrc[NT];
    bool bvalid[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + g;
        bvalid[nt] = col < ncols;
        bsrc[nt] = smem + L.off_a + (bvalid[nt] ? col : 0) * L.astride + t * F::kChunkK;
    }
    int acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;
    const int nsteps = (K + F::kStepK - 1) / F::kStepK;
    for (int s = warp; s < nsteps; s += kWarps) {
        const bool lane_ok = s * F::kStepK + t * F::kChunkK < K;
        uint4 a0 = make_uint4(0, 0, 0, 0), a1 = make_uint4(0, 0, 0, 0);
        if (lane_ok) {
            a0 = *reinterpret_cast<const uint4*>(w0 + 64 * s);
            a1 = *reinterpret_cast<const uint4*>(w1 + 64 * s);
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
                    const uint8_t* src = bsrc[nt] + s * F::kStepK + om * (4 * F::kRegs);
#pragma unroll
                    for (int v = 0; v < F::kRegs / 4; ++v) {
                        const uint4 bv = *reinterpret_cast<const uint4*>(src + 16 * v);
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

    int* red = reinterpret_cast<int*>(smem + L.off_red);  // [kWarps][NT][16][8]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        int* rb = red + ((warp * NT + nt) * 16) * 8;
        rb[g * 8 + 2 * t] = acc[nt][0];
        rb[g * 8 + 2 * t + 1] = acc[nt][1];
        rb[(g + 8) * 8 + 2 * t] = acc[nt][2];
        rb[(g + 8) * 8 + 2 * t + 1] = acc[nt][3];
    }
    __syncthreads();
    auto part = [&](int col, int r) {
        int s = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[((w * NT + (col >> 3)) * 16 + r) * 8 + (col & 7)];
        return s;
    };
    if (FORM == 0) {
        for (int o = threadIdx.x; o < M * 16; o += kThreads) {
            const int m = o >> 4, r = o & 15;
            float amax = 0.f;
            int qs = 0;
            for (int c = 0; c < kCluster; ++c) {
                amax = fmaxf(amax, cl_max[c * kMaxTok + m]);
                qs += cl_sum[c * kMaxTok + m];
            }
            const float sc = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
            const int accv = part(m, r) - qs;
            const int n = rg * 16 + r;
            const float v = __fmul_rn(__fmul_rn((float)accv, sc), p.w_scale);
            p.y[(size_t)m * p.N + n] = __half_as_ushort(__float2half_rn(v));
            if (p.acc_out) p.acc_out[(size_t)m * p.N + n] = accv;
        }
    } else {
        for (int o = threadIdx.x; o < M * 16; o += kThreads) {
            const int m = o >> 4, r = o & 15;
            float amax = 0.f;
            long long ts = 0;
            for (int c = 0; c < kCluster; ++c) {
                amax = fmaxf(amax, cl_max[c * kMaxTok + m]);
                ts += cl_sum[c * kMaxTok + m];
            }
            const float st = amax > 0.f ? __fdiv_rn(amax, 32639.0f) : 0.f;
            const long long P = 256ll * part(2 * m, r) + part(2 * m + 1, r);
            const int n = rg * 16 + r;
            const float z = __fmul_rn(st, (float)(2 * P - ts));
            const float hv = __half2float(__ushort_as_half(p.h[n]));
            p.y[(size_t)m * p.N + n] = __half_as_ushort(__float2half_rn(__fmul_rn(z, hv)));
        }
    }
}

template <int FORM, int NT>
cudaError_t launch_decode(const DecodeParams& p, int smem, cudaStream_t s) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<FORM, NT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kDecodeMaxSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int groups = p.N / 16;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((groups + kCluster - 1) / kCluster * kCluster);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = kCluster;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, decode_kernel<FORM, NT>, p);
}

template <int FORM>
int pick_nt(int M) {
    const int cols = M * DF<FORM>::kCPT;
    return cols <= 8 ? 1 : cols <= 16 ? 2 : cols <= 32 ? 4 : 0;
}

template <int FORM>
int decode_smem(int M, int K) {
    const int nt = pick_nt<FORM>(M);
    if (nt == 0) return -1;
    if (nt == 1) return decode_layout<FORM, 1>(M, K).total;
    if (nt == 2) return decode_layout<FORM, 2>(M, K).total;
    return decode_layout<FORM, 4>(M, K).total;
}

template <int FORM>
cudaError_t launch_decode_form(const DecodeParams& p, cudaStream_t s) {
    const int smem = decode_smem<FORM>(p.M, p.K);
    switch (pick_nt<FORM>(p.M)) {
        case 1: return launch_decode<FORM, 1>(p, smem, s);
        case 2: return launch_decode<FORM, 2>(p, smem, s);
        default: return launch_decode<FORM, 4>(p, smem, s);
    }
}

}  // namespace

bool decode_fused_fits(int form, int M, int K) {
    if (M < 1 || M > kMaxTok) return false;
    const int smem = form == 0 ? decode_smem<0>(M, K) : decode_smem<1>(M, K);
    return smem > 0 && smem <= kDecodeMaxSmem;
}

cudaError_t launch_ternary_decode(const uint16_t* x, const uint32_t* w2, int M, int K, int N,
                                  float w_scale, uint16_t* y, int32_t* acc_out,
                                  unsigned int* flags, cudaStream_t s) {
    DecodeParams p{x, nullptr, nullptr, w2, w_scale, M, K, N, y, acc_out, flags};
    return launch_decode_form<0>(p, s);
}

cudaError_t launch_onebit_decode(const uint16_t* x, const uint16_t* g, const uint16_t* h,
                                 const uint32_t* s1, int M, int K, int N, uint16_t* y,
                                 unsigned int* flags, cudaStream_t s) {
    DecodeParams p{x, g, h, s1, 0.f, M, K, N, y, nullptr, flags};
    return launch_decode_form<1>(p, s);
}

}  // namespace bl
