// prefill.cu -- prefill-shaped (large M) packed-weight GEMM on the 5th-generation
// tensor cores (tcgen05.mma kind::i8, accumulator in TMEM).
//
// At prefill sizes the layer really is a dense contraction (BitNet b1.58 page,
// "BitNet b1.58 介绍": 8-bit activations against ternary weights; OneBit page,
// "1. 新的 1bit 结构": the +-1 matrix between x*g and h), so the weights are
// expanded on chip to int8 and run through the int8 tensor cores:
//   ternary: B = code in {0,1,2} (= t + 1), D = q . code^T, acc = D - sum_k q
//   OneBit : B = bit in {0,1}, A rows = the two int8 limbs (hi, lo) of each
//            token's 16-bit fixed-point image X of x*g, so
//            sum X*S = 2 (256 D_hi + D_lo) - sum X
// Both are exact in int32.
//
// CTA tile: 128 A rows (tokens, or token limbs) x 256 weight rows, K in
// 128-byte stages.  Warp roles (192 threads):
//   warp 0     TMA producer: A tile (128x128 B, 128-byte swizzle) and the packed
//              weight tile (256 rows x 32 B or 16 B) into a 3-stage ring;
//   warp 1     TMEM allocator + single-thread MMA issuer (4 x K=32 per stage);
//   warps 2-5  unpack the packed tile into the UMMA K-major 128-byte-swizzled
//              int8 layout, then run the epilogue (tcgen05.ld -> scale -> fp16).
// The unpacked byte order inside each 16-byte (ternary) / 32-byte (sign) group
// is the order the byte-SIMD unpack produces; the activation preparation
// kernels store A in the same order, so no shuffle is needed anywhere.
// Every mbarrier wait is bounded (a timeout sets the device condition word).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_prims.cuh"

namespace bl {

namespace {

constexpr int BM = 128;          // A rows per tile (MMA M)
constexpr int BN = 256;          // weight rows per tile (MMA N)
constexpr int BK = 128;          // k per stage (bytes of int8 A per row)
constexpr int STAGES = 3;
constexpr int kThreads = 192;
constexpr int A_STAGE = BM * BK;        // 16 KB
constexpr int BU_STAGE = BN * BK;       // 32 KB
constexpr int BP_STAGE_MAX = BN * BK / 4;  // 8 KB (ternary); sign uses half
constexpr int OFF_A = 0;
constexpr int OFF_BU = OFF_A + STAGES * A_STAGE;
constexpr int OFF_BP = OFF_BU + STAGES * BU_STAGE;
constexpr int OFF_BAR = OFF_BP + STAGES * BP_STAGE_MAX;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // barriers + alignment slack
constexpr uint32_t TMEM_COLS = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

template <int FORM>
struct PF;
template <>
struct PF<0> {  // ternary
    static constexpr int kPackedRowBytes = BK / 4;  // 32
};
template <>
struct PF<1> {  // sign
    static constexpr int kPackedRowBytes = BK / 8;  // 16
};

struct PrefillParams {
    int rows_a;        // M (ternary) or 2M (OneBit limb rows)
    int M, K, N;
    const float* scale;   // per token: ternary scale / OneBit fixed-point step
    const int32_t* rsum;  // per token: sum q / sum X
    const uint16_t* h;    // OneBit output value vector
    float w_scale;
    uint16_t* y;
    int32_t* acc_out;
    unsigned int* flags;
};

template <int FORM>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b, const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(smem);
    const uint32_t bar_full = sbase + OFF_BAR;             // TMA landed   [STAGES]
    const uint32_t bar_unp = bar_full + 8 * STAGES;        // unpacked     [STAGES]
    const uint32_t bar_empty = bar_unp + 8 * STAGES;       // MMA consumed [STAGES]
    const uint32_t bar_acc = bar_empty + 8 * STAGES;       // accumulator complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * (3 * STAGES + 1));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN;
    const int m0 = blockIdx.y * BM;
    const int nk = p.K / BK;
    constexpr int kBp = PF<FORM>::kPackedRowBytes * BN;
    constexpr uint32_t kTx = A_STAGE + kBp;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(bar_full + 8 * s, 1);
            tc::mbar_init(bar_unp + 8 * s, 128);
            tc::mbar_init(bar_empty + 8 * s, 1);
        }
        tc::mbar_init(bar_acc, 1);
        tc::mbar_fence_init();
        tc::prefetch_tmap(&tmap_a);
        tc::prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % STAGES;
                if (kb >= STAGES)
                    ok = tc::mbar_wait(bar_empty + 8 * s, ((kb / STAGES) - 1) & 1, p.flags,
                                       kWaitLimitNs);
                if (!ok) break;
                tc::mbar_arrive_expect_tx(bar_full + 8 * s, kTx);
                tc::tma_load_2d(sbase + OFF_A + s * A_STAGE, &tmap_a, kb * BK, m0, bar_full + 8 * s);
                tc::tma_load_2d(sbase + OFF_BP + s * BP_STAGE_MAX, &tmap_b,
                                kb * PF<FORM>::kPackedRowBytes, n0, bar_full + 8 * s);
                ++issued;
            }
            if (!ok) {
                // drain copies still in flight before the CTA's shared memory goes away
                for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb)
                    tc::mbar_wait(bar_full + 8 * (kb % STAGES), (kb / STAGES) & 1, p.flags,
                                  kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_i8(BM, BN);
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % STAGES;
                const uint32_t par = (kb / STAGES) & 1;
                ok = tc::mbar_wait(bar_full + 8 * s, par, p.flags, kWaitLimitNs) &&
                     tc::mbar_wait(bar_unp + 8 * s, par, p.flags, kWaitLimitNs);
                if (!ok) break;
                tc::tc_fence_after();
                const uint32_t a_s = sbase + OFF_A + s * A_STAGE;
                const uint32_t b_s = sbase + OFF_BU + s * BU_STAGE;
#pragma unroll
                for (int j = 0; j < BK / 32; ++j)
                    tc::mma_i8(tmem_d, tc::desc_kmajor_sw128(a_s + 32 * j),
                               tc::desc_kmajor_sw128(b_s + 32 * j), idesc, kb > 0 || j > 0);
                tc::mma_commit(bar_empty + 8 * s);
            }
            // completion of everything issued (also on the abort path)
            tc::mma_commit(bar_acc);
            tc::mbar_wait(bar_acc, 0, p.flags, kWaitLimitNs);
        }
    } else {
        // ---------------- unpack (warps 2-5, 128 threads) -------------------
        const int ut = threadIdx.x - 64;  // 0..127
        bool ok = true;
        for (int kb = 0; kb < nk && ok; ++kb) {
            const int s = kb % STAGES;
            ok = tc::mbar_wait(bar_full + 8 * s, (kb / STAGES) & 1, p.flags, kWaitLimitNs);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const uint8_t* bp = smem + OFF_BP + s * BP_STAGE_MAX;
            uint8_t* bu = smem + OFF_BU + s * BU_STAGE;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = ut + 128 * half;   // weight row within the tile
                uint8_t* rowp = bu + r * BK;
                const int sw = r & 7;
                if (FORM == 0) {
                    const uint4* src = reinterpret_cast<const uint4*>(bp + r * 32);
#pragma unroll
                    for (int v = 0; v < 2; ++v) {
                        const uint4 w = src[v];
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t x = ws[e];
                            const int c = 4 * v + e;  // 16-byte chunk = packed word
                            *reinterpret_cast<uint4*>(rowp + ((c ^ sw) << 4)) =
                                make_uint4(x & 0x03030303u, (x >> 2) & 0x03030303u,
                                           (x >> 4) & 0x03030303u, (x >> 6) & 0x03030303u);
                        }
                    }
                } else {
                    const uint4 w = *reinterpret_cast<const uint4*>(bp + r * 16);
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t x = ws[e];
                        const int c0 = 2 * e, c1 = 2 * e + 1;
                        *reinterpret_cast<uint4*>(rowp + ((c0 ^ sw) << 4)) =
                            make_uint4(x & 0x01010101u, (x >> 1) & 0x01010101u,
                                       (x >> 2) & 0x01010101u, (x >> 3) & 0x01010101u);
                        *reinterpret_cast<uint4*>(rowp + ((c1 ^ sw) << 4)) =
                            make_uint4((x >> 4) & 0x01010101u, (x >> 5) & 0x01010101u,
                                       (x >> 6) & 0x01010101u, (x >> 7) & 0x01010101u);
                    }
                }
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(bar_unp + 8 * s);
        }

        // ---------------- epilogue ----------------------------------------
        const bool acc_ok =
            __all_sync(0xffffffffu, tc::mbar_wait(bar_acc, 0, p.flags, kWaitLimitNs));
        tc::tc_fence_after();
        if (ok && acc_ok) {
            const int q = warp & 3;             // TMEM lane quarter this warp may read
            const int arow = m0 + 32 * q + lane;  // A row held by this thread
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t r[32];
                tc::tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(32 * q) << 16) + 32 * cc, r);
                tc::tmem_ld_wait();
                const int nb = n0 + 32 * cc;
                if (FORM == 0) {
                    if (arow < p.M && nb < p.N) {
                        const float sc = p.scale[arow];
                        const int rs = p.rsum[arow];
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int a0 = (int)r[2 * i] - rs, a1 = (int)r[2 * i + 1] - rs;
                            const float v0 = __fmul_rn(__fmul_rn((float)a0, sc), p.w_scale);
                            const float v1 = __fmul_rn(__fmul_rn((float)a1, sc), p.w_scale);
                            packed[i] = (uint32_t)__half_as_ushort(__float2half_rn(v0)) |
                                        ((uint32_t)__half_as_ushort(__float2half_rn(v1)) << 16);
                            r[2 * i] = (uint32_t)a0;
                            r[2 * i + 1] = (uint32_t)a1;
                        }
                        uint16_t* yrow = p.y + (size_t)arow * p.N + nb;
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8)
                            if (nb + 8 * g8 < p.N)
                                reinterpret_cast<uint4*>(yrow)[g8] =
                                    make_uint4(packed[4 * g8], packed[4 * g8 + 1],
                                               packed[4 * g8 + 2], packed[4 * g8 + 3]);
                        if (p.acc_out) {
                            int32_t* arw = p.acc_out + (size_t)arow * p.N + nb;
#pragma unroll
                            for (int g4 = 0; g4 < 8; ++g4)
                                if (nb + 4 * g4 < p.N)
                                    reinterpret_cast<uint4*>(arw)[g4] =
                                        make_uint4(r[4 * g4], r[4 * g4 + 1], r[4 * g4 + 2],
                                                   r[4 * g4 + 3]);
                        }
                    }
                } else {
                    // lanes (2i, 2i+1) hold the hi and lo limb rows of one token
                    uint32_t lo[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) lo[i] = __shfl_down_sync(0xffffffffu, r[i], 1);
                    const int tok = arow >> 1;
                    if ((lane & 1) == 0 && tok < p.M && nb < p.N) {
                        const float st = p.scale[tok];
                        const long long ts = p.rsum[tok];
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float v[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int c = 2 * i + e;
                                const long long P = 256ll * (int)r[c] + (int)lo[c];
                                const float z = __fmul_rn(st, (float)(2 * P - ts));
                                const int n = min(nb + c, p.N - 1);
                                v[e] = __fmul_rn(z, __half2float(__ushort_as_half(p.h[n])));
                            }
                            packed[i] = (uint32_t)__half_as_ushort(__float2half_rn(v[0])) |
                                        ((uint32_t)__half_as_ushort(__float2half_rn(v[1])) << 16);
                        }
                        uint16_t* yrow = p.y + (size_t)tok * p.N + nb;
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8)
                            if (nb + 8 * g8 < p.N)
                                reinterpret_cast<uint4*>(yrow)[g8] =
                                    make_uint4(packed[4 * g8], packed[4 * g8 + 1],
                                               packed[4 * g8 + 2], packed[4 * g8 + 3]);
                    }
                }
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_d, TMEM_COLS);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D uint8 tensor map: rows x cols bytes (row stride = cols), box box_cols x box_rows.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
               uint32_t box_rows, CUtensorMapSwizzle swz) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int FORM>
cudaError_t launch_prefill(const int8_t* act, const uint32_t* w, const PrefillParams& p,
                           cudaStream_t s) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(prefill_kernel<FORM>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap ta, tb;
    if (!make_tmap(&ta, act, (uint64_t)p.rows_a, (uint64_t)p.K, BK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const uint64_t prow = (uint64_t)p.K / (FORM == 0 ? 4 : 8);
    if (!make_tmap(&tb, w, (uint64_t)p.N, prow, PF<FORM>::kPackedRowBytes, BN,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    dim3 grid((p.N + BN - 1) / BN, (p.rows_a + BM - 1) / BM);
    prefill_kernel<FORM><<<grid, kThreads, SMEM_BYTES, s>>>(ta, tb, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ternary_prefill(const uint32_t* w2, const int8_t* qp, const float* scale,
                                   const int32_t* qsum, int M, int K, int N, float w_scale,
                                   uint16_t* y, int32_t* acc_out, unsigned int* flags,
                                   cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    PrefillParams p{M, M, K, N, scale, qsum, nullptr, w_scale, y, acc_out, flags};
    return launch_prefill<0>(qp, w2, p, s);
}

cudaError_t launch_onebit_prefill(const uint32_t* s1, const int8_t* planes, const float* step,
                                  const int32_t* tsum, const uint16_t* h, int M, int K, int N,
                                  uint16_t* y, unsigned int* flags, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    PrefillParams p{2 * M, M, K, N, step, tsum, h, 0.f, y, nullptr, flags};
    return launch_prefill<1>(planes, s1, p, s);
}

}  // namespace bl
