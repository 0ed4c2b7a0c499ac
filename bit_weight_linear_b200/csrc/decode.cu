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
//   3. Activation preparation in the CTA: per-token absmax (warp shuffles +
//      one CTA barrier), then every thread quantises its 16- (ternary) or
//      32-element (sign) groups straight into the permuted shared-memory tile.
//      x is small at decode sizes and L2-resident, so each CTA reading it is
//      cheaper than any cross-CTA exchange.
//   4. The contraction runs from shared memory on the warp-level u8 x s8 MMA
//      (byte-SIMD unpack as in skinny.cu), warps split K, and reduce through
//      shared memory for the epilogue.
// Weight rows in shared memory are padded to a stride of 64 (mod 128) bytes so
// that every quarter-warp's 16-byte loads hit 8 distinct bank groups.
#include "common.cuh"
#include "decode_forms.cuh"
#include "kernels.h"
#include "tc_prims.cuh"

namespace bl {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxTok = 32;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct DecodeParams {
    int stage_x;            // 1: x (and g) are staged in shared memory between the two passes
    const int8_t* prep;     // prepared activations [cols][K] (PREP kernels only)
    const float* pscale;    // per token: scale (ternary) / fixed-point step (OneBit)
    const int32_t* prsum;   // per token: row sum of the prepared activations
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
    int wstride, astride, off_a, off_x, off_red, off_tok, off_bar, total;
};

// Shared memory: weight slab [16][wstride] | prepared activations [cols][astride] |
// staged x [M][K] (+ g [K]) fp16 when stage_x | partial sums | token scratch | mbarrier
template <int FORM, int NT>
__host__ __device__ inline DecodeLayout decode_layout(int M, int K, int stage_x) {
    DecodeLayout l;
    // row stride = 64 (mod 128) bytes: the 8 lanes of a quarter-warp (rows 2q,
    // 2q+1; chunks t = 0..3) then read 8 disjoint 16-byte bank groups
    const int rowbytes = K / DF<FORM>::kPerWord * 4;
    l.wstride = rowbytes + ((64 - rowbytes % 128) + 128) % 128;
    l.astride = K + 16;
    l.off_a = 16 * l.wstride;
    l.off_x = l.off_a + M * DF<FORM>::kCPT * l.astride;
    l.off_red = l.off_x + (stage_x ? 2 * K * (M + (FORM == 1 ? 1 : 0)) : 0);
    l.off_tok = l.off_red + kWarps * NT * 16 * 8 * 4;       // contraction partials
    // token scratch: warp partials of the max and of the row sums (2 x kWarps x kMaxTok)
    l.off_bar = l.off_tok + 4 * (2 * kWarps * kMaxTok);
    l.total = l.off_bar + 16;
    return l;
}

// 16-byte read of x or g in pass B: from the shared-memory copy when staged,
// else (coherently) from global memory.
__device__ __forceinline__ uint4 ld_act(const uint16_t* p, int staged) {
    return staged ? *reinterpret_cast<const uint4*>(p) : tc::ld_v4(p);
}

// PREP = 0: the kernel prepares the activations from x itself (decode sizes).
// PREP = 1: they were prepared by the activation kernel launched just before
// (quant.cu); the kernel only copies them into shared memory.
template <int FORM, int NT, int PREP>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
    using F = DF<FORM>;
    extern __shared__ __align__(16) uint8_t smem[];
    const DecodeLayout L = decode_layout<FORM, NT>(p.M, p.K, p.stage_x);
    const int K = p.K, M = p.M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sb = tc::smem_u32(smem);
    const uint32_t bar = sb + L.off_bar;
    float* red_max = reinterpret_cast<float*>(smem + L.off_tok);        // [kWarps][kMaxTok]
    int* red_sum = reinterpret_cast<int*>(red_max + kWarps * kMaxTok);  // [kWarps][kMaxTok]
    const int rg = blockIdx.x;                 // 16-row group
    const int wbytes = K / F::kPerWord * 4;    // packed bytes per weight row

    // 1. stream this CTA's weight slab into shared memory (independent of x)
    if (threadIdx.x == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_fence_init();
        tc::mbar_arrive_expect_tx(bar, (uint32_t)(16 * wbytes));
        const uint8_t* src = reinterpret_cast<const uint8_t*>(p.w) + (size_t)rg * 16 * wbytes;
        for (int r = 0; r < 16; ++r)
            tc::bulk_g2s(sb + r * L.wstride, src + (size_t)r * wbytes, (uint32_t)wbytes, bar);
    }
    __syncthreads();  // the mbarrier is initialised before any thread waits on it
    tc::pdl_trigger();
    tc::pdl_wait();

    if (PREP) {
        // prepared activations -> shared memory as 16-byte asynchronous copies
        const int cols = M * F::kCPT, per_row = K / 16;
        for (int c = threadIdx.x; c < cols * per_row; c += kThreads) {
            const int row = c / per_row, off = c - row * per_row;
            tc::cp_async16(sb + L.off_a + row * L.astride + 16 * off,
                           p.prep + (size_t)row * K + 16 * off);
        }
        tc::cp_async_wait_all();
        __syncthreads();
    } else {
    // 2-3. activation preparation
    constexpr int G = F::kGroup;
    const int ngroups = K / G;
    // pass A: per-token max |x| (ternary) or |x*g| (OneBit); x (and g) are copied
    // into shared memory on the way, so pass B does not go back to L2
    uint16_t* xs_s = reinterpret_cast<uint16_t*>(smem + L.off_x);
    uint16_t* gs_s = xs_s + (size_t)M * K;
    if (FORM == 1 && p.stage_x) {
        for (int c = threadIdx.x; c < K / 8; c += kThreads)
            reinterpret_cast<uint4*>(gs_s)[c] = tc::ld_v4(p.g + 8 * c);
    }
    for (int m = 0; m < M; ++m) {
        float mx = 0.f;
        for (int i = threadIdx.x; i < ngroups; i += kThreads) {
            const uint16_t* xs = p.x + (size_t)m * K + (size_t)i * G;
#pragma unroll
            for (int v = 0; v < G / 8; ++v) {
                uint4 a = tc::ld_v4(xs + 8 * v);
                if (p.stage_x)
                    *reinterpret_cast<uint4*>(xs_s + (size_t)m * K + (size_t)i * G + 8 * v) = a;
                const uint32_t av[4] = {a.x, a.y, a.z, a.w};
                if (FORM == 0) {
                    // max of |fp16| bit patterns, two lanes per word (monotone for finite values)
                    uint32_t mb = __vmaxu2(__vmaxu2(av[0] & 0x7fff7fffu, av[1] & 0x7fff7fffu),
                                           __vmaxu2(av[2] & 0x7fff7fffu, av[3] & 0x7fff7fffu));
                    mx = fmaxf(mx, hbits(max(mb & 0xffffu, mb >> 16)));
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
    const uint16_t* xsrc = p.stage_x ? xs_s : p.x;
    const uint16_t* gsrc = p.stage_x ? gs_s : p.g;

    // pass B: quantise into the permuted shared-memory activation tile
    for (int m = 0; m < M; ++m) {
        float amax = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) amax = fmaxf(amax, red_max[w * kMaxTok + m]);
        int sum = 0;
        for (int i = threadIdx.x; i < ngroups; i += kThreads) {
            const uint16_t* xs = xsrc + (size_t)m * K + (size_t)i * G;
            if (FORM == 0) {
                // |x * inv| <= 127 (1 + 2^-24) for inv = rn(127/amax): the rounded
                // value never leaves [-127, 127], so no clamp is needed
                const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
                int qv[16];
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    uint4 a = ld_act(xs + 8 * v, p.stage_x);
                    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        qv[8 * v + e] = __float2int_rn(__fmul_rn(hbits(av[e >> 1] >> (16 * (e & 1))), inv));
                }
                // byte 4j+b of the group holds element 4b+j
                uint4 o;
                o.x = pack4(qv[0], qv[4], qv[8], qv[12]);
                o.y = pack4(qv[1], qv[5], qv[9], qv[13]);
                o.z = pack4(qv[2], qv[6], qv[10], qv[14]);
                o.w = pack4(qv[3], qv[7], qv[11], qv[15]);
                *reinterpret_cast<uint4*>(smem + L.off_a + m * L.astride + i * G) = o;
                sum = __dp4a((int)o.x, 0x01010101, sum);
                sum = __dp4a((int)o.y, 0x01010101, sum);
                sum = __dp4a((int)o.z, 0x01010101, sum);
                sum = __dp4a((int)o.w, 0x01010101, sum);
            } else {
                constexpr int kFix = 32639;
                const float inv = amax > 0.f ? __fdiv_rn((float)kFix, amax) : 0.f;
                int hv[32], lv[32];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 a = ld_act(xs + 8 * v, p.stage_x);
                    uint4 gg = ld_act(gsrc + (size_t)i * G + 8 * v, p.stage_x);
                    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float pr = __fmul_rn(hbits(av[e >> 1] >> (16 * (e & 1))),
                                                   hbits(gv[e >> 1] >> (16 * (e & 1))));
                        // |pr * inv| <= 32639 (1 + 2^-24): no clamp needed
                        const int X = __float2int_rn(__fmul_rn(pr, inv));
                        const int hi = (X + 128) >> 8;
                        hv[8 * v + e] = hi;
                        lv[8 * v + e] = X - 256 * hi;
                    }
                }
                // byte 4j+b of the 32-byte group holds element 8b+j
                uint32_t ho[8], lo[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    ho[j] = pack4(hv[j], hv[8 + j], hv[16 + j], hv[24 + j]);
                    lo[j] = pack4(lv[j], lv[8 + j], lv[16 + j], lv[24 + j]);
                }
                int shi = 0, slo = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    shi = __dp4a((int)ho[j], 0x01010101, shi);
                    slo = __dp4a((int)lo[j], 0x01010101, slo);
                }
                sum += 256 * shi + slo;  // sum of X over the group
                uint4* dh = reinterpret_cast<uint4*>(smem + L.off_a + (2 * m) * L.astride + i * G);
                uint4* dl = reinterpret_cast<uint4*>(smem + L.off_a + (2 * m + 1) * L.astride + i * G);
                dh[0] = make_uint4(ho[0], ho[1], ho[2], ho[3]);
                dh[1] = make_uint4(ho[4], ho[5], ho[6], ho[7]);
                dl[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                dl[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
            }
        }
        sum = warp_sum(sum);
        if (lane == 0) red_sum[warp * kMaxTok + m] = sum;
    }
    __syncthreads();

    }

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
    // four independent accumulator chains (one per word of the lane's 4-word
    // chunk) cut the dependent MMA latency per step
    int acc[NT][4][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[nt][c][0] = acc[nt][c][1] = acc[nt][c][2] = acc[nt][c][3] = 0;
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
                    mma_u8s8_16832(acc[nt][om], u0[j], u1[j], u0[j + 1], u1[j + 1], b[j], b[j + 1]);
            }
        }
    }

    int* red = reinterpret_cast<int*>(smem + L.off_red);  // [kWarps][NT][16][8]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        int* rb = red + ((warp * NT + nt) * 16) * 8;
        int v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = acc[nt][0][e] + acc[nt][1][e] + acc[nt][2][e] + acc[nt][3][e];
        rb[g * 8 + 2 * t] = v[0];
        rb[g * 8 + 2 * t + 1] = v[1];
        rb[(g + 8) * 8 + 2 * t] = v[2];
        rb[(g + 8) * 8 + 2 * t + 1] = v[3];
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
            float sc;
            int qs = 0;
            if (PREP) {
                sc = p.pscale[m];
                qs = p.prsum[m];
            } else {
                float amax = 0.f;
                for (int w = 0; w < kWarps; ++w) {
                    amax = fmaxf(amax, red_max[w * kMaxTok + m]);
                    qs += red_sum[w * kMaxTok + m];
                }
                sc = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
            }
            const int accv = part(m, r) - qs;
            const int n = rg * 16 + r;
            const float v = __fmul_rn(__fmul_rn((float)accv, sc), p.w_scale);
            p.y[(size_t)m * p.N + n] = __half_as_ushort(__float2half_rn(v));
            if (p.acc_out) p.acc_out[(size_t)m * p.N + n] = accv;
        }
    } else {
        for (int o = threadIdx.x; o < M * 16; o += kThreads) {
            const int m = o >> 4, r = o & 15;
            float st;
            long long ts = 0;
            if (PREP) {
                st = p.pscale[m];
                ts = p.prsum[m];
            } else {
                float amax = 0.f;
                for (int w = 0; w < kWarps; ++w) {
                    amax = fmaxf(amax, red_max[w * kMaxTok + m]);
                    ts += red_sum[w * kMaxTok + m];
                }
                st = amax > 0.f ? __fdiv_rn(amax, 32639.0f) : 0.f;
            }
            const long long P = 256ll * part(2 * m, r) + part(2 * m + 1, r);
            const int n = rg * 16 + r;
            const float z = __fmul_rn(st, (float)(2 * P - ts));
            const float hv = __half2float(__ushort_as_half(p.h[n]));
            p.y[(size_t)m * p.N + n] = __half_as_ushort(__float2half_rn(__fmul_rn(z, hv)));
        }
    }
}

template <int FORM, int NT, int PREP>
cudaError_t launch_decode(const DecodeParams& p, int smem, cudaStream_t s) {
    static_assert(NT >= 1, "");
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<FORM, NT, PREP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kDecodeMaxSmem);
        if (e != cudaSuccess) return e;
        e = use_max_shared_carveout(decode_kernel<FORM, NT, PREP>);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.N / 16);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<FORM, NT, PREP>, p);
}

template <int FORM>
int pick_nt(int M) {
    const int cols = M * DF<FORM>::kCPT;
    return cols <= 8 ? 1 : cols <= 16 ? 2 : cols <= 32 ? 4 : 0;
}

template <int FORM>
int decode_smem(int M, int K, int stage_x) {
    const int nt = pick_nt<FORM>(M);
    if (nt == 0) return -1;
    if (nt == 1) return decode_layout<FORM, 1>(M, K, stage_x).total;
    if (nt == 2) return decode_layout<FORM, 2>(M, K, stage_x).total;
    return decode_layout<FORM, 4>(M, K, stage_x).total;
}

// Stage x in shared memory whenever that still fits next to the weight slab.
template <int FORM>
int decode_stage_x(int M, int K) {
    const int s = decode_smem<FORM>(M, K, 1);
    return (s > 0 && s <= kDecodeMaxSmem) ? 1 : 0;
}

template <int FORM, int PREP>
cudaError_t launch_decode_form(DecodeParams p, cudaStream_t s) {
    p.stage_x = PREP ? 0 : decode_stage_x<FORM>(p.M, p.K);
    const int smem = decode_smem<FORM>(p.M, p.K, p.stage_x);
    switch (pick_nt<FORM>(p.M)) {
        case 1: return launch_decode<FORM, 1, PREP>(p, smem, s);
        case 2: return launch_decode<FORM, 2, PREP>(p, smem, s);
        default: return launch_decode<FORM, 4, PREP>(p, smem, s);
    }
}

}  // namespace

bool decode_fused_fits(int form, int M, int K) {
    if (M < 1 || M > kMaxTok) return false;
    const int smem = form == 0 ? decode_smem<0>(M, K, 0) : decode_smem<1>(M, K, 0);
    return smem > 0 && smem <= kDecodeMaxSmem;
}

cudaError_t launch_ternary_decode(const uint16_t* x, const uint32_t* w2, int M, int K, int N,
                                  float w_scale, uint16_t* y, int32_t* acc_out,
                                  unsigned int* flags, cudaStream_t s) {
    DecodeParams p{0, nullptr, nullptr, nullptr, x, nullptr, nullptr, w2, w_scale, M, K, N, y,
                   acc_out, flags};
    return launch_decode_form<0, 0>(p, s);
}

cudaError_t launch_onebit_decode(const uint16_t* x, const uint16_t* g, const uint16_t* h,
                                 const uint32_t* s1, int M, int K, int N, uint16_t* y,
                                 unsigned int* flags, cudaStream_t s) {
    DecodeParams p{0, nullptr, nullptr, nullptr, x, g, h, s1, 0.f, M, K, N, y, nullptr, flags};
    return launch_decode_form<1, 0>(p, s);
}

cudaError_t launch_ternary_decode_prepared(const int8_t* qp, const float* scale, const int32_t* qsum,
                                           const uint32_t* w2, int M, int K, int N, float w_scale,
                                           uint16_t* y, int32_t* acc_out, unsigned int* flags,
                                           cudaStream_t s) {
    DecodeParams p{0, qp, scale, qsum, nullptr, nullptr, nullptr, w2, w_scale, M, K, N, y,
                   acc_out, flags};
    return launch_decode_form<0, 1>(p, s);
}

cudaError_t launch_onebit_decode_prepared(const int8_t* planes, const float* step,
                                          const int32_t* tsum, const uint16_t* h,
                                          const uint32_t* s1, int M, int K, int N, uint16_t* y,
                                          unsigned int* flags, cudaStream_t s) {
    DecodeParams p{0, planes, step, tsum, nullptr, nullptr, h, s1, 0.f, M, K, N, y, nullptr, flags};
    return launch_decode_form<1, 1>(p, s);
}

bool decode_prepared_fits(int form, int M, int K) {
    if (M < 1 || M > kMaxTok) return false;
    const int smem = form == 0 ? decode_smem<0>(M, K, 0) : decode_smem<1>(M, K, 0);
    return smem > 0 && smem <= kDecodeMaxSmem;
}

}  // namespace bl
