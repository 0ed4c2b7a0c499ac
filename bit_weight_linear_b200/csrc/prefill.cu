// prefill.cu -- prefill-shaped (large M) packed-weight GEMM on the 5th-generation
// tensor cores (tcgen05.mma kind::i8, accumulator in TMEM).
//
// At prefill sizes the layer really is a dense contraction (BitNet b1.58 page,
// "BitNet b1.58 介绍": 8-bit activations against ternary weights; OneBit page,
// "1. 新的 1bit 结构": the +-1 matrix between x*g and h), so the weights are
// expanded on chip to int8 and run through the int8 tensor cores:
//   ternary: code in {0,1,2} (= t + 1), D = code . q^T, acc = D - sum_k q
//   OneBit : bit in {0,1}, activation rows = the three int8 limbs (hi, mid, lo)
//            of each token's 23-bit fixed-point image X of x*g, so
//            sum X*S = 2 (65536 D_hi + 256 D_mid + D_lo) - sum X
// Both are exact in int32.
//
// The expanded weights never touch shared memory: they are the MMA's A
// operand and live in TENSOR memory.  Each unpack thread owns one weight row
// (one TMEM lane), expands that row's 128 k of a stage to 128 bytes and writes
// them with one tcgen05.st; the MMA reads A from TMEM and only the activations
// (B operand, TMA-loaded, 128-byte swizzle) come from shared memory.  That
// keeps shared-memory traffic per MMA at the activation tile alone.
//
// CTA tile: 128 weight rows (MMA M, TMEM lanes) x bt activation rows (MMA N:
// tokens, or token limb rows; bt = the smallest multiple of 32 covering them,
// at most 256), K in 128-byte stages; tiles ordered
// activation-tile-fastest so CTAs sharing a weight tile run together.  A
// OneBit tile holds tpt <= bt/3 whole tokens (3 tpt limb rows; the rows past
// them are loaded but unused), so a token's limbs never straddle two tiles.
// Warp roles (320 threads):
//   warp 0     TMA producer: activation tile (256 x 128 B) and packed weight tile
//              (128 rows x 32 B or 16 B) into a 5-stage shared-memory ring; the
//              weight tiles have their own full barriers and the first ring of
//              them is requested before the wait on the previous kernel
//              (programmatic dependent launch), the activations after it;
//   warp 1     TMEM allocator + single-thread MMA issuer (4 x K=32 per stage);
//   warps 2-5  one thread per weight row: unpack into a 4-slot TMEM ring;
//   warps 2-9  the epilogue (tcgen05.ld -> correction and scale -> fp16), two
//              warps per TMEM lane quarter taking alternate 32-column chunks; a
//              warp's lanes are 32 consecutive output columns.  The fp16 tile
//              is staged in the idle activation ring and leaves by one TMA
//              tensor store.
// The expanded byte order inside each 16-byte (ternary) / 32-byte (sign) group
// is the order the byte-SIMD unpack produces; the activation preparation
// kernels store the activations in the same order.
// Every mbarrier wait is bounded (a timeout sets the device condition word).
#include "common.cuh"
#include "kernels.h"
#include "tc_prims.cuh"
#include "tmap.cuh"

namespace bl {

namespace {

constexpr int BW = 128;          // weight rows per tile (MMA M)
constexpr int BT = 256;          // max activation rows per tile (MMA N); per call bt <= BT
constexpr int BK = 128;          // k per block (bytes of int8 per activation row)
constexpr int kThreads = 320;
constexpr int kEpiThreads = kThreads - 64;   // warps 2-9: the epilogue (2-5 also expand)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t kAccCol = 0;          // accumulator: columns [0, 256)
constexpr uint32_t kWCol = 256;          // expanded-weight slots: columns [256, 512)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

// A ring stage carries KB consecutive 128-k blocks: KB = 1 for 256-row activation
// tiles, 2 for <= 128 rows, 4 for <= 64 rows.  The activation part of a stage
// stays 32 KB, so small token counts still move enough bytes per stage to keep
// the SM's copy pipeline full.
template <int KB>
struct PS {
    static constexpr int SS = KB == 1 ? 5 : 4;             // shared-memory ring stages
    static constexpr int SU = KB == 1 ? 4 : 8 / KB;        // TMEM weight slots (32*KB columns each)
    static constexpr int ACT_STAGE = BT * BK;              // 32 KB: KB blocks of bt <= BT/KB rows
    static constexpr int BP_STAGE = BW * BK / 4 * KB;      // packed weights (ternary; sign uses half)
    static constexpr int OFF_ACT = 0;
    static constexpr int OFF_BP = OFF_ACT + SS * ACT_STAGE;
    static constexpr int OFF_TOK = OFF_BP + SS * BP_STAGE;  // per-token scale / row sum [BT]
    static constexpr int OFF_BAR = OFF_TOK + 2 * BT * 4;
    static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // barriers + alignment slack
};

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
    int rows_a;        // activation rows: M (ternary) or 3M (OneBit limb rows)
    int bt;            // activation rows per tile: multiple of 32, <= BT
    int tpt;           // tokens per tile: bt (ternary), <= bt / 3 (OneBit)
    int rpt;           // first activation row of token tile i is i * rpt (bt; 3 tpt)
    int M, K, N;
    const float* scale;   // per token: ternary scale / OneBit fixed-point step
    const int32_t* rsum;  // ternary, per token: sum q
    const long long* xsum;  // OneBit, per token: sum X
    const uint16_t* h;    // OneBit output value vector
    float w_scale;
    uint16_t* y;
    int32_t* acc_out;
    unsigned int* flags;
    float* zf;            // OneBit: optional fp32 [M][N] copy of y before fp16 rounding
    // Work split.  CTAs [0, dp_tiles) each compute one whole tile.  The
    // remaining sk_tiles tiles form one balanced round: CTA dp_tiles + c
    // (c < sk_ctas) takes the (tile, k-stage) units [c U / G, (c+1) U / G) of
    // them (U = sk_tiles * stages, G = sk_ctas), tile by tile.  A tile split
    // between CTAs is finished by whichever of them arrives last.
    int dp_tiles, sk_tiles, sk_ctas;
    unsigned int* sk_ctr;  // [sk_tiles] arrival counts, zero when the kernel starts
    int32_t* sk_slots;     // [2 * sk_ctas][bt * BW] partial accumulators
    // Whole-tile kernel: the limit of a pipeline wait (2 s).  Test hook
    // (bl_debug_stall_next_launch): stall = 1 leaves CTA 0's first activation
    // stage unrequested, so the MMA's wait for it runs out after wait_ns.
    uint64_t wait_ns;
    int stall;
};

// Expand one weight row's 128 k of packed codes (32 B ternary / 16 B sign at
// bp) to 128 int8 bytes and store them as 32 TMEM columns of this thread's
// lane.  The byte order inside each 16-k (32-k) group is the order the byte
// SIMD unpack produces: byte 4j+b holds element 4b+j (8b+j for sign).
template <int FORM>
__device__ __forceinline__ void expand_row_block(const uint8_t* bp, uint32_t taddr) {
    uint32_t e[32];
    if (FORM == 0) {
        const uint4 w0 = *reinterpret_cast<const uint4*>(bp);
        const uint4 w1 = *reinterpret_cast<const uint4*>(bp + 16);
        const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int o = 0; o < 8; ++o)
#pragma unroll
            for (int j = 0; j < 4; ++j) e[4 * o + j] = (ws[o] >> (2 * j)) & 0x03030303u;
    } else {
        const uint4 w0 = *reinterpret_cast<const uint4*>(bp);
        const uint32_t ws[4] = {w0.x, w0.y, w0.z, w0.w};
#pragma unroll
        for (int o = 0; o < 4; ++o)
#pragma unroll
            for (int j = 0; j < 8; ++j) e[8 * o + j] = (ws[o] >> j) & 0x01010101u;
    }
    tc::tmem_st_32x32b_x32(taddr, e);
}

// Per-token scale and row sum of the tile's tokens [tok0, tok0 + tpt), zero
// past M; filled by the epilogue threads et = 0 .. kEpiThreads-1.  The row
// sums are int32 (ternary, tok_rsum) or int64 (OneBit, tok_xsum; the same
// shared-memory bytes).
template <int FORM>
__device__ __forceinline__ void fill_token_table(const PrefillParams& p, int tok0, int et,
                                                 float* tok_scale, int* tok_rsum) {
    long long* tok_xsum = reinterpret_cast<long long*>(tok_rsum);
    for (int i = et; i < p.tpt; i += kEpiThreads) {
        const int tok = tok0 + i;
        const bool in = tok < p.M;
        tok_scale[i] = in ? p.scale[tok] : 0.f;
        if (FORM == 0) tok_rsum[i] = in ? p.rsum[tok] : 0;
        else tok_xsum[i] = in ? p.xsum[tok] : 0ll;
    }
}

// Ternary epilogue of one 32-token chunk of accumulators d (TMEM lane = weight
// row r, output column n): bias by the token row sums, scale, round to fp16
// and stage as [token][128 columns]; optionally also store the int32
// accumulators.
__device__ __forceinline__ void convert_chunk(const uint32_t (&d)[32], int cc, uint16_t* stage,
                                              const float* tok_scale, const int* tok_rsum,
                                              const PrefillParams& p, int r, int n, int t0) {
#pragma unroll
    for (int i4 = 0; i4 < 32; i4 += 4) {
        const int tb = 32 * cc + i4;
        const float4 sc = *reinterpret_cast<const float4*>(tok_scale + tb);
        const int4 rs = *reinterpret_cast<const int4*>(tok_rsum + tb);
        const float scs[4] = {sc.x, sc.y, sc.z, sc.w};
        const int rss[4] = {rs.x, rs.y, rs.z, rs.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int a = (int)d[i4 + j] - rss[j];
            const float v = __fmul_rn(__fmul_rn((float)a, scs[j]), p.w_scale);
            stage[(tb + j) * BW + r] = __half_as_ushort(__float2half_rn(v));
            const int m = t0 + tb + j;
            if (p.acc_out && m < p.M && n < p.N) p.acc_out[(size_t)m * p.N + n] = a;
        }
    }
}

// OneBit epilogue of token group gi (tokens 32 gi .. 32 gi + 31 of the tile,
// accumulator columns 96 gi .. 96 gi + 95 in d): combine each token's three
// limb columns, scale by its step and h[n], round to fp16 and stage as
// [token][128 columns].  Tokens past the tile's tpt are skipped.
__device__ __forceinline__ void convert_onebit_group(const uint32_t (&d)[96], int gi,
                                                     uint16_t* stage, const float* tok_scale,
                                                     const long long* tok_xsum, int tpt, int r,
                                                     float hn, const PrefillParams& p, int n, int t0) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int t = 32 * gi + i;
        if (t < tpt) {
            const long long Z = limb_combine((int)d[3 * i], (int)d[3 * i + 1], (int)d[3 * i + 2],
                                             tok_xsum[t]);
            const float z = __fmul_rn(tok_scale[t], (float)Z);
            const float zh = __fmul_rn(z, hn);
            stage[t * BW + r] = __half_as_ushort(__float2half_rn(zh));
            if (p.zf && t0 + t < p.M && n < p.N) p.zf[(size_t)(t0 + t) * p.N + n] = zh;
        }
    }
}

// One whole tile per CTA (launches without a balanced round).
template <int FORM, int KB>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_act,
                   const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_y, const PrefillParams p) {
    using L = PS<KB>;
    constexpr int SS = L::SS, SU = L::SU, ACT_STAGE = L::ACT_STAGE, BP_STAGE = L::BP_STAGE;
    constexpr int OFF_ACT = L::OFF_ACT, OFF_BP = L::OFF_BP, OFF_TOK = L::OFF_TOK, OFF_BAR = L::OFF_BAR;
    constexpr int kRowBytes = PF<FORM>::kPackedRowBytes * KB;  // packed bytes of a row per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(smem);
    const uint32_t bar_full = sbase + OFF_BAR;        // activation tile landed         [SS]
    const uint32_t bar_wfull = bar_full + 8 * SS;     // packed weight tile landed      [SS]
    const uint32_t bar_empty = bar_wfull + 8 * SS;    // MMA done with the stage        [SS]
    const uint32_t bar_ufull = bar_empty + 8 * SS;    // expanded weights in TMEM      [SU]
    const uint32_t bar_uempty = bar_ufull + 8 * SU;   // MMA done with a TMEM slot     [SU]
    const uint32_t bar_acc = bar_uempty + 8 * SU;     // accumulator complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * (3 * SS + 2 * SU + 1));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bt = p.bt;
    const int ttiles = (p.M + p.tpt - 1) / p.tpt;
    const int a0 = (blockIdx.x % ttiles) * p.rpt;  // first activation row of the tile
    const int t0 = (blockIdx.x % ttiles) * p.tpt;  // first token of the tile
    const int n0 = (blockIdx.x / ttiles) * BW;     // first weight row of the tile
    const int nblk = p.K / BK;                 // 128-k blocks
    const int nk = (nblk + KB - 1) / KB;       // stages; the last may hold fewer blocks
    // blocks in stage kb; the weight box of a short last stage runs past the row
    // end and is zero-filled (codes 0 expand to 0, so those products vanish)
    auto blocks = [&](int kb) { return KB == 1 ? 1 : min(KB, nblk - kb * KB); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < SS; ++s) {
            tc::mbar_init(bar_full + 8 * s, 1);
            tc::mbar_init(bar_wfull + 8 * s, 1);
            tc::mbar_init(bar_empty + 8 * s, 1);
        }
        for (int u = 0; u < SU; ++u) {
            tc::mbar_init(bar_ufull + 8 * u, 128);
            tc::mbar_init(bar_uempty + 8 * u, 1);
        }
        tc::mbar_init(bar_acc, 1);
        tc::mbar_fence_init();
        tc::prefetch_tmap(&tmap_act);
        tc::prefetch_tmap(&tmap_w);
        tc::prefetch_tmap(&tmap_y);
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // The packed weights are call parameters, not written by the kernel
            // this launch may overlap (programmatic dependent launch): the first
            // ring of weight tiles is requested before waiting for the producer
            // of the activations, so the expansion warps can start early.
            const int pre = nk < SS ? nk : SS;
            int wissued = 0, issued = 0;
            for (; wissued < pre; ++wissued) {
                tc::mbar_arrive_expect_tx(bar_wfull + 8 * wissued, (uint32_t)(kRowBytes * BW));
                tc::tma_load_2d(sbase + OFF_BP + wissued * BP_STAGE, &tmap_w,
                                wissued * kRowBytes, n0, bar_wfull + 8 * wissued);
            }
            tc::pdl_wait();
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % SS;
                if (kb >= SS) {
                    ok = tc::mbar_wait(bar_empty + 8 * s, ((kb / SS) - 1) & 1, p.flags, p.wait_ns);
                    if (!ok) break;
                    tc::mbar_arrive_expect_tx(bar_wfull + 8 * s, (uint32_t)(kRowBytes * BW));
                    tc::tma_load_2d(sbase + OFF_BP + s * BP_STAGE, &tmap_w, kb * kRowBytes, n0,
                                    bar_wfull + 8 * s);
                    ++wissued;
                }
                const int nb = blocks(kb);
                ++issued;
                if (p.stall && blockIdx.x == 0 && kb == 0) continue;   // test hook
                tc::mbar_arrive_expect_tx(bar_full + 8 * s, (uint32_t)(nb * bt * BK));
                for (int b = 0; b < nb; ++b)
                    tc::tma_load_2d(sbase + OFF_ACT + s * ACT_STAGE + b * bt * BK, &tmap_act,
                                    (kb * KB + b) * BK, a0, bar_full + 8 * s);
            }
            // Every copy requested here lands before the CTA can exit: on the
            // normal path the MMA has consumed them (these waits return at
            // once); after a timeout some may still be in flight.
            for (int kb = (issued > SS ? issued - SS : 0); kb < issued; ++kb)
                if (!(p.stall && blockIdx.x == 0 && kb == 0))   // never requested
                    tc::mbar_wait(bar_full + 8 * (kb % SS), (kb / SS) & 1, p.flags, kWaitLimitNs);
            for (int kb = (wissued > SS ? wissued - SS : 0); kb < wissued; ++kb)
                tc::mbar_wait(bar_wfull + 8 * (kb % SS), (kb / SS) & 1, p.flags, kWaitLimitNs);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_i8(BW, bt);
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % SS, u = kb % SU;
                ok = tc::mbar_wait(bar_full + 8 * s, (kb / SS) & 1, p.flags, p.wait_ns) &&
                     tc::mbar_wait(bar_ufull + 8 * u, (kb / SU) & 1, p.flags, p.wait_ns);
                if (!ok) break;
                tc::tc_fence_after();
                const uint32_t act_s = sbase + OFF_ACT + s * ACT_STAGE;
                const int nj = 4 * blocks(kb);
#pragma unroll
                for (int j = 0; j < KB * BK / 32; ++j)
                    if (j < nj)
                    tc::mma_i8_ts(tmem + kAccCol, tmem + kWCol + 32 * KB * u + 8 * j,
                                  tc::desc_kmajor_sw128(act_s + (j >> 2) * bt * BK + 32 * (j & 3)),
                                  idesc, kb > 0 || j > 0);
                tc::mma_commit(bar_empty + 8 * s);
                tc::mma_commit(bar_uempty + 8 * u);
            }
            // the next kernel on the stream may start launching now; it waits for
            // this grid's completion before touching anything this grid writes
            tc::pdl_trigger();
            // completion of everything issued (also on the abort path)
            tc::mma_commit(bar_acc);
            tc::mbar_wait(bar_acc, 0, p.flags, kWaitLimitNs);
        }
    } else {
        // ------- expand (warps 2-5): thread = weight row = TMEM lane -------
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int hsel = (warp - 2) >> 2;       // 0: warps 2-5, 1: warps 6-9 (epilogue only)
        const int r = 32 * q + lane;            // weight row within the tile
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        bool ok = true;
        for (int kb = 0; hsel == 0 && kb < nk && ok; ++kb) {
            const int s = kb % SS, u = kb % SU;
            ok = tc::mbar_wait(bar_wfull + 8 * s, (kb / SS) & 1, p.flags, p.wait_ns);
            if (ok && kb >= SU)
                ok = tc::mbar_wait(bar_uempty + 8 * u, ((kb / SU) - 1) & 1, p.flags, p.wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
#pragma unroll
            for (int b = 0; b < KB; ++b) {
                const uint8_t* bp = smem + OFF_BP + s * BP_STAGE + r * kRowBytes +
                                    b * PF<FORM>::kPackedRowBytes;
                expand_row_block<FORM>(bp, lane_base + kWCol + 32 * KB * u + 32 * b);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(bar_ufull + 8 * u);
        }

        // ---------------- epilogue ----------------------------------------
        // per-token scale and row sum of this activation tile, staged once
        float* tok_scale = reinterpret_cast<float*>(smem + OFF_TOK);
        int* tok_rsum = reinterpret_cast<int*>(tok_scale + BT);
        const int et = threadIdx.x - 64;        // 0..kEpiThreads-1
        tc::pdl_wait();                          // scale / row sums come from the previous kernel
        fill_token_table<FORM>(p, t0, et, tok_scale, tok_rsum);
        const bool acc_ok = tc::mbar_wait(bar_acc, 0, p.flags, p.wait_ns);
        // one decision for the eight epilogue warps; also publishes the token table
        const bool good = tc::bar_and(1, kEpiThreads, ok && acc_ok);
        tc::tc_fence_after();
        if (good) {
            // The fp16 tile is staged in the (now idle) activation ring as
            // [token][128 columns] and leaves with one tensor store, which also
            // drops the rows past M and the columns past N.
            uint16_t* stage = reinterpret_cast<uint16_t*>(smem + OFF_ACT);
            const int n = n0 + r;                // output column held by this thread
            const float hn = (FORM == 1 && n < p.N) ? __half2float(__ushort_as_half(p.h[n])) : 0.f;
            const int nch = bt / 32;
            if constexpr (FORM == 0) {
                // chunks cc = hsel, hsel+2, ...; the TMEM load of the next chunk is
                // in flight while this one is converted
                uint32_t da[32], db[32];
                if (hsel < nch) tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * hsel, da);
                tc::tmem_ld_wait();
#pragma unroll 1
                for (int cc = hsel; cc < nch; cc += 4) {
                    if (cc + 2 < nch) tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * (cc + 2), db);
                    convert_chunk(da, cc, stage, tok_scale, tok_rsum, p, r, n, t0);
                    tc::tmem_ld_wait();
                    if (cc + 2 >= nch) break;
                    if (cc + 4 < nch) tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * (cc + 4), da);
                    convert_chunk(db, cc + 2, stage, tok_scale, tok_rsum, p, r, n, t0);
                    tc::tmem_ld_wait();
                }
            } else {
                // token groups gi = hsel, hsel+2, ...: 32 tokens = 96 columns = 3 chunks
                const long long* tok_xsum = reinterpret_cast<const long long*>(tok_rsum);
#pragma unroll 1
                for (int gi = hsel; gi < (p.tpt + 31) / 32; gi += 2) {
                    uint32_t d[96];
#pragma unroll
                    for (int c = 0; c < 3; ++c)
                        if (3 * gi + c < nch)
                            tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * (3 * gi + c),
                                                   *reinterpret_cast<uint32_t(*)[32]>(d + 32 * c));
                    tc::tmem_ld_wait();
                    convert_onebit_group(d, gi, stage, tok_scale, tok_xsum, p.tpt, r, hn, p, n, t0);
                }
            }
            tc::fence_proxy_async_smem();
            asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
            if (et == 0) {
                tc::tma_store_2d(&tmap_y, sbase + OFF_ACT, n0 * 2, t0);
                tc::bulk_commit_group();
                tc::bulk_wait_group_read0();
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// The same tile pipeline over a CTA's run of (tile, k-stage) units, used for
// launches with a balanced round: pieces of tiles, int32 partial slots and
// per-tile arrival counts (see PrefillParams).  Ring and TMEM-slot phases run
// on across the pieces of a CTA; the accumulator and the staging area are
// handed back by two more barriers before the next piece starts.
template <int FORM, int KB>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_split_kernel(const __grid_constant__ CUtensorMap tmap_act,
                   const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_y, const PrefillParams p) {
    using L = PS<KB>;
    constexpr int SS = L::SS, SU = L::SU, ACT_STAGE = L::ACT_STAGE, BP_STAGE = L::BP_STAGE;
    constexpr int OFF_ACT = L::OFF_ACT, OFF_BP = L::OFF_BP, OFF_TOK = L::OFF_TOK, OFF_BAR = L::OFF_BAR;
    constexpr int kRowBytes = PF<FORM>::kPackedRowBytes * KB;  // packed bytes of a row per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(smem);
    const uint32_t bar_full = sbase + OFF_BAR;        // activation tile landed         [SS]
    const uint32_t bar_wfull = bar_full + 8 * SS;     // packed weight tile landed      [SS]
    const uint32_t bar_empty = bar_wfull + 8 * SS;    // MMA done with the stage        [SS]
    const uint32_t bar_ufull = bar_empty + 8 * SS;    // expanded weights in TMEM      [SU]
    const uint32_t bar_uempty = bar_ufull + 8 * SU;   // MMA done with a TMEM slot     [SU]
    const uint32_t bar_acc = bar_uempty + 8 * SU;     // accumulator of a piece complete
    const uint32_t bar_accfree = bar_acc + 8;         // epilogue done reading it
    const uint32_t bar_stfree = bar_accfree + 8;      // epilogue done with the staging area
    const uint32_t bar_part = bar_stfree + 8;         // another piece's partial slot landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * (3 * SS + 2 * SU + 4));
    unsigned int* arrivals = reinterpret_cast<unsigned int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bt = p.bt;
    const int ttiles = (p.M + p.tpt - 1) / p.tpt;
    const int nblk = p.K / BK;                 // 128-k blocks
    const int nk = (nblk + KB - 1) / KB;       // stages; the last may hold fewer blocks
    // blocks in stage kb; the weight box of a short last stage runs past the row
    // end and is zero-filled (codes 0 expand to 0, so those products vanish)
    auto blocks = [&](int kb) { return KB == 1 ? 1 : min(KB, nblk - kb * KB); };

    // This CTA's (tile, stage) units [ua, ub), walked in pieces of one tile each.
    const long long U = (long long)p.sk_tiles * nk;
    const int G = p.sk_ctas > 0 ? p.sk_ctas : 1;
    const int cme = (int)blockIdx.x - p.dp_tiles;       // >= 0: a CTA of the balanced round
    auto sk_start = [&](int c) { return (long long)c * U / G; };   // relative to the round
    long long ua, ub;
    if (cme < 0) {
        ua = (long long)blockIdx.x * nk;
        ub = ua + nk;
    } else {
        const long long base = (long long)p.dp_tiles * nk;
        ua = base + sk_start(cme);
        ub = base + sk_start(cme + 1);
    }
    auto piece = [&](long long u, int& tile, int& kb0, int& kb1) {
        tile = (int)(u / nk);
        kb0 = (int)(u - (long long)tile * nk);
        kb1 = (int)min((long long)nk, kb0 + (ub - u));
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < SS; ++s) {
            tc::mbar_init(bar_full + 8 * s, 1);
            tc::mbar_init(bar_wfull + 8 * s, 1);
            tc::mbar_init(bar_empty + 8 * s, 1);
        }
        for (int u = 0; u < SU; ++u) {
            tc::mbar_init(bar_ufull + 8 * u, 128);
            tc::mbar_init(bar_uempty + 8 * u, 1);
        }
        tc::mbar_init(bar_acc, 1);
        tc::mbar_init(bar_accfree, kEpiThreads);
        tc::mbar_init(bar_stfree, 1);
        tc::mbar_init(bar_part, 1);
        tc::mbar_fence_init();
        tc::prefetch_tmap(&tmap_act);
        tc::prefetch_tmap(&tmap_w);
        tc::prefetch_tmap(&tmap_y);
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Ring and TMEM-slot positions run on across pieces: g counts this CTA's stages.
    if (warp == 0) {
        if (lane == 0) {
            int tile, kb0, kb1;
            piece(ua, tile, kb0, kb1);
            // The packed weights are call parameters, not written by the kernel
            // this launch may overlap (programmatic dependent launch): the first
            // ring of weight tiles is requested before waiting for the producer
            // of the activations, so the expansion warps can start early.
            const int pre = min(SS, kb1 - kb0);
            int ag = 0, wg = 0;                  // activation / weight stages issued
            for (; wg < pre; ++wg) {
                tc::mbar_arrive_expect_tx(bar_wfull + 8 * wg, (uint32_t)(kRowBytes * BW));
                tc::tma_load_2d(sbase + OFF_BP + wg * BP_STAGE, &tmap_w, (kb0 + wg) * kRowBytes,
                                (tile / ttiles) * BW, bar_wfull + 8 * wg);
            }
            tc::pdl_wait();
            bool ok = true;
            int item = 0;
            for (long long u = ua; u < ub && ok; ++item) {
                piece(u, tile, kb0, kb1);
                u += kb1 - kb0;
                const int a0 = (tile % ttiles) * p.rpt, n0 = (tile / ttiles) * BW;
                // the previous piece's epilogue stages its output in the ring
                if (item > 0) ok = tc::mbar_wait(bar_stfree, (item - 1) & 1, p.flags, kWaitLimitNs);
                for (int kb = kb0; kb < kb1 && ok; ++kb) {
                    const int g = ag, s = g % SS;
                    if (g >= SS) {
                        ok = tc::mbar_wait(bar_empty + 8 * s, ((g / SS) - 1) & 1, p.flags, kWaitLimitNs);
                        if (!ok) break;
                    }
                    if (g >= wg) {
                        tc::mbar_arrive_expect_tx(bar_wfull + 8 * s, (uint32_t)(kRowBytes * BW));
                        tc::tma_load_2d(sbase + OFF_BP + s * BP_STAGE, &tmap_w, kb * kRowBytes, n0,
                                        bar_wfull + 8 * s);
                        ++wg;
                    }
                    const int nb = blocks(kb);
                    tc::mbar_arrive_expect_tx(bar_full + 8 * s, (uint32_t)(nb * bt * BK));
                    for (int b = 0; b < nb; ++b)
                        tc::tma_load_2d(sbase + OFF_ACT + s * ACT_STAGE + b * bt * BK, &tmap_act,
                                        (kb * KB + b) * BK, a0, bar_full + 8 * s);
                    ++ag;
                }
            }
            // Every copy requested here lands before the CTA can exit (see
            // prefill_kernel).
            for (int g = (ag > SS ? ag - SS : 0); g < ag; ++g)
                tc::mbar_wait(bar_full + 8 * (g % SS), (g / SS) & 1, p.flags, kWaitLimitNs);
            for (int g = (wg > SS ? wg - SS : 0); g < wg; ++g)
                tc::mbar_wait(bar_wfull + 8 * (g % SS), (g / SS) & 1, p.flags, kWaitLimitNs);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_i8(BW, bt);
            bool ok = true;
            int g = 0, item = 0;
            for (long long u = ua; u < ub && ok; ++item) {
                int tile, kb0, kb1;
                piece(u, tile, kb0, kb1);
                u += kb1 - kb0;
                if (item > 0) {
                    // the accumulator is reused: the previous piece's epilogue must have read it
                    ok = tc::mbar_wait(bar_accfree, (item - 1) & 1, p.flags, kWaitLimitNs);
                    if (!ok) break;
                    tc::tc_fence_after();
                }
                for (int kb = kb0; kb < kb1; ++kb, ++g) {
                    const int s = g % SS, uu = g % SU;
                    ok = tc::mbar_wait(bar_full + 8 * s, (g / SS) & 1, p.flags, kWaitLimitNs) &&
                         tc::mbar_wait(bar_ufull + 8 * uu, (g / SU) & 1, p.flags, kWaitLimitNs);
                    if (!ok) break;
                    tc::tc_fence_after();
                    const uint32_t act_s = sbase + OFF_ACT + s * ACT_STAGE;
                    const int nj = 4 * blocks(kb);
#pragma unroll
                    for (int j = 0; j < KB * BK / 32; ++j)
                        if (j < nj)
                        tc::mma_i8_ts(tmem + kAccCol, tmem + kWCol + 32 * KB * uu + 8 * j,
                                      tc::desc_kmajor_sw128(act_s + (j >> 2) * bt * BK + 32 * (j & 3)),
                                      idesc, kb > kb0 || j > 0);
                    tc::mma_commit(bar_empty + 8 * s);
                    tc::mma_commit(bar_uempty + 8 * uu);
                }
                // completion of this piece's MMAs (also on the abort path)
                tc::mma_commit(bar_acc);
            }
            // the next kernel on the stream may start launching now; it waits for
            // this grid's completion before touching anything this grid writes
            tc::pdl_trigger();
            // everything issued has completed before the accumulator is freed
            if (item > 0) tc::mbar_wait(bar_acc, (item - 1) & 1, p.flags, kWaitLimitNs);
        }
    } else {
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int hsel = (warp - 2) >> 2;       // 0: warps 2-5 (expand + epilogue), 1: warps 6-9
        const int r = 32 * q + lane;            // weight row within the tile = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        float* tok_scale = reinterpret_cast<float*>(smem + OFF_TOK);
        int* tok_rsum = reinterpret_cast<int*>(tok_scale + BT);
        const int et = threadIdx.x - 64;        // 0..kEpiThreads-1
        const size_t slot_elems = (size_t)bt * BW;
        // a finisher brings the other piece's slot into the idle activation
        // ring, behind the fp16 staging area (at most 64 KB)
        constexpr int kPartOff = 32 * 1024;
        bool ok = true;
        int g = 0, item = 0, nfin = 0;
        for (long long u = ua; u < ub; ++item) {
            const long long upiece = u;
            int tile, kb0, kb1;
            piece(u, tile, kb0, kb1);
            u += kb1 - kb0;
            const int t0 = (tile % ttiles) * p.tpt, n0 = (tile / ttiles) * BW;

            // ------- expand (warps 2-5): one thread per weight row -------
            for (int kb = kb0; hsel == 0 && kb < kb1 && ok; ++kb, ++g) {
                const int s = g % SS, uu = g % SU;
                ok = tc::mbar_wait(bar_wfull + 8 * s, (g / SS) & 1, p.flags, kWaitLimitNs);
                if (ok && g >= SU)
                    ok = tc::mbar_wait(bar_uempty + 8 * uu, ((g / SU) - 1) & 1, p.flags, kWaitLimitNs);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    const uint8_t* bp = smem + OFF_BP + s * BP_STAGE + r * kRowBytes +
                                        b * PF<FORM>::kPackedRowBytes;
                    expand_row_block<FORM>(bp, lane_base + kWCol + 32 * KB * uu + 32 * b);
                }
                tc::tmem_st_wait();
                tc::tc_fence_before();
                tc::mbar_arrive(bar_ufull + 8 * uu);
            }

            // ---------------- epilogue (warps 2-9) ----------------------------
            if (item == 0) tc::pdl_wait();       // scale / row sums come from the previous kernel
            // per-token scale and row sum of this activation tile
            fill_token_table<FORM>(p, t0, et, tok_scale, tok_rsum);
            const bool acc_ok = tc::mbar_wait(bar_acc, item & 1, p.flags, kWaitLimitNs);
            // one decision for the eight epilogue warps; also publishes the token table
            const bool good = tc::bar_and(1, kEpiThreads, ok && acc_ok);
            if (!good) break;
            tc::tc_fence_after();

            // A piece that is not a whole tile: store its int32 accumulator in
            // this CTA's slot (0: its first piece, 1: its last), then count the
            // arrival; the last of the tile's pieces to arrive finishes the tile.
            const bool whole = kb0 == 0 && kb1 == nk;
            int ts = 0, c_first = 0, c_last = 0;
            if (!whole) {
                ts = tile - p.dp_tiles;
                const long long t_lo = (long long)ts * nk, t_hi = t_lo + nk - 1;
                c_first = (int)(((t_lo + 1) * G - 1) / U);   // CTA holding the tile's first unit
                c_last = (int)(((t_hi + 1) * G - 1) / U);    // ... and its last unit
                int32_t* slot = p.sk_slots + (size_t)(2 * cme + (upiece == ua ? 0 : 1)) * slot_elems;
#pragma unroll 1
                for (int cc = hsel; cc < bt / 32; cc += 2) {
                    uint32_t d[32];
                    tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * cc, d);
                    tc::tmem_ld_wait();
                    int4* dst = reinterpret_cast<int4*>(slot) + (size_t)cc * 8 * BW + r;
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4)
                        dst[i4 * BW] = make_int4((int)d[4 * i4], (int)d[4 * i4 + 1],
                                                 (int)d[4 * i4 + 2], (int)d[4 * i4 + 3]);
                }
                __threadfence();
                asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
                if (et == 0) *arrivals = atomicAdd(p.sk_ctr + ts, 1u);
                asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
                if (*arrivals != (unsigned int)(c_last - c_first)) {
                    // another piece of this tile is still running; it finishes the tile
                    tc::tc_fence_before();
                    tc::mbar_arrive(bar_accfree);
                    if (et == 0) tc::mbar_arrive(bar_stfree);
                    continue;
                }
                __threadfence();
                if (c_last - c_first == 1) {
                    // one other piece: one bulk copy of its slot into shared memory
                    const int c = c_first == cme ? c_last : c_first;
                    const int which = (c == c_first && sk_start(c) < (long long)ts * nk) ? 1 : 0;
                    const int32_t* src = p.sk_slots + (size_t)(2 * c + which) * slot_elems;
                    const uint32_t bytes = (uint32_t)(slot_elems * 4), quarter = bytes / 4;
                    if (et == 0) {
                        tc::fence_proxy_async_global();
                        tc::mbar_arrive_expect_tx(bar_part, bytes);
                        for (int i = 0; i < 4; ++i)
                            tc::bulk_g2s(sbase + OFF_ACT + kPartOff + i * quarter,
                                         reinterpret_cast<const uint8_t*>(src) + (size_t)i * quarter,
                                         quarter, bar_part);
                    }
                    const bool landed = tc::bar_and(
                        1, kEpiThreads, tc::mbar_wait(bar_part, nfin & 1, p.flags, kWaitLimitNs));
                    if (!landed) {
                        // the flag is set; let the copy land before shared memory goes away
                        if (et == 0) tc::mbar_wait(bar_part, nfin & 1, p.flags, kWaitLimitNs);
                        break;
                    }
                    ++nfin;
                }
            }

            // The fp16 tile is staged in the activation ring as [token][128
            // columns] and leaves with one tensor store, which also drops the
            // rows past M and the columns past N.
            uint16_t* stage = reinterpret_cast<uint16_t*>(smem + OFF_ACT);
            const int n = n0 + r;                // output column held by this thread
            const float hn = (FORM == 1 && n < p.N) ? __half2float(__ushort_as_half(p.h[n])) : 0.f;
            // add the other pieces' partial accumulators of chunk cc (exact in int32)
            auto add_parts = [&](uint32_t (&d)[32], int cc) {
                if (whole) return;
                if (c_last - c_first == 1) {
                    const int4* src = reinterpret_cast<const int4*>(smem + OFF_ACT + kPartOff) +
                                      (size_t)cc * 8 * BW + r;
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const int4 v = src[i4 * BW];
                        d[4 * i4] += (uint32_t)v.x;
                        d[4 * i4 + 1] += (uint32_t)v.y;
                        d[4 * i4 + 2] += (uint32_t)v.z;
                        d[4 * i4 + 3] += (uint32_t)v.w;
                    }
                    return;
                }
                for (int c = c_first; c <= c_last; ++c) {
                    if (c == cme) continue;
                    const int which = (c == c_first && sk_start(c) < (long long)ts * nk) ? 1 : 0;
                    const int4* src = reinterpret_cast<const int4*>(
                                          p.sk_slots + (size_t)(2 * c + which) * slot_elems) +
                                      (size_t)cc * 8 * BW + r;
                    int4 v[8];
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) v[i4] = __ldcg(src + i4 * BW);   // another CTA's
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        d[4 * i4] += (uint32_t)v[i4].x;
                        d[4 * i4 + 1] += (uint32_t)v[i4].y;
                        d[4 * i4 + 2] += (uint32_t)v[i4].z;
                        d[4 * i4 + 3] += (uint32_t)v[i4].w;
                    }
                }
            };
            const int nch = bt / 32;
            if constexpr (FORM == 0) {
                // chunks cc = hsel, hsel+2, ...; the TMEM load of the next chunk is
                // in flight while this one is finished
                uint32_t da[32], db[32];
                if (hsel < nch) tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * hsel, da);
                tc::tmem_ld_wait();
#pragma unroll 1
                for (int cc = hsel; cc < nch; cc += 4) {
                    // 256-row tiles: the staging of chunks 4-7 reuses the space of
                    // the partial's chunks 0-1, read in the first round
                    if (cc >= 4 && nch == 8 && !whole && c_last - c_first == 1)
                        asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
                    if (cc + 2 < nch) tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * (cc + 2), db);
                    add_parts(da, cc);
                    convert_chunk(da, cc, stage, tok_scale, tok_rsum, p, r, n, t0);
                    tc::tmem_ld_wait();
                    if (cc + 2 >= nch) break;
                    if (cc + 4 < nch) tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * (cc + 4), da);
                    add_parts(db, cc + 2);
                    convert_chunk(db, cc + 2, stage, tok_scale, tok_rsum, p, r, n, t0);
                    tc::tmem_ld_wait();
                }
            } else {
                // token groups gi = hsel, hsel+2, ...: 32 tokens = 96 columns = 3
                // chunks (the fp16 staging of at most 85 tokens stays below the
                // partial slot's copy at kPartOff)
                const long long* tok_xsum = reinterpret_cast<const long long*>(tok_rsum);
#pragma unroll 1
                for (int gi = hsel; gi < (p.tpt + 31) / 32; gi += 2) {
                    uint32_t d[96];
#pragma unroll
                    for (int c = 0; c < 3; ++c)
                        if (3 * gi + c < nch)
                            tc::tmem_ld_32x32b_x32(lane_base + kAccCol + 32 * (3 * gi + c),
                                                   *reinterpret_cast<uint32_t(*)[32]>(d + 32 * c));
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 3; ++c)
                        if (3 * gi + c < nch)
                            add_parts(*reinterpret_cast<uint32_t(*)[32]>(d + 32 * c), 3 * gi + c);
                    convert_onebit_group(d, gi, stage, tok_scale, tok_xsum, p.tpt, r, hn, p, n, t0);
                }
            }
            tc::tc_fence_before();
            tc::mbar_arrive(bar_accfree);
            tc::fence_proxy_async_smem();
            asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
            if (et == 0) {
                tc::tma_store_2d(&tmap_y, sbase + OFF_ACT, n0 * 2, t0);
                tc::bulk_commit_group();
                tc::bulk_wait_group_read0();
                tc::mbar_arrive(bar_stfree);
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// 2-D uint8 tensor map: rows x cols bytes (row stride = cols), box box_cols x box_rows.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
               uint32_t box_rows, CUtensorMapSwizzle swz) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {box_cols, box_rows};
    return encode_u8_map(m, base, 2, dims, strides, box, swz);
}

// Activation rows per tile: the smallest multiple of 32 that covers them, at most BT.
inline int choose_bt(int rows) {
    const int r = (rows + 31) / 32 * 32;
    return r < BT ? r : BT;
}

// Tile geometry of a call: activation rows per tile, tokens per tile, k-blocks
// per stage, stages per tile and the number of (weight-row, token) tiles.
// The tokens are cut into the fewest tiles of at most BT activation rows (BT
// tokens, or BT/3 OneBit tokens of three limb rows), of balanced size: 300
// ternary tokens run as two 160-row tiles rather than 256 + 44.  A OneBit tile
// loads bt >= 3 tpt rows; the rows past its tokens are computed but unused.
struct Geometry {
    int bt, tpt, kb, nk, tiles;
};

Geometry geometry(int form, int M, int K, int N) {
    Geometry g;
    const int cpt = form == 0 ? 1 : 3;           // activation rows per token
    const int max_tpt = BT / cpt;
    const int ttiles = (M + max_tpt - 1) / max_tpt;
    const int tpt = (M + ttiles - 1) / ttiles;
    g.bt = choose_bt(cpt * tpt);
    g.tpt = form == 0 ? g.bt : tpt;
    g.kb = g.bt <= BT / 4 ? 4 : g.bt <= BT / 2 ? 2 : 1;
    g.nk = (K / BK + g.kb - 1) / g.kb;
    g.tiles = ((N + BW - 1) / BW) * ((M + g.tpt - 1) / g.tpt);
    return g;
}

// One CTA per SM at a time (the ring takes most of shared memory), so the
// tiles run in rounds of G.  When the last round would leave SMs idle, the
// last one or two rounds' tiles are instead shared out evenly in k-stages over
// G CTAs.  The cost model, in stage-times (measured on the 70B-shaped layers):
// a whole tile's epilogue is worth about 10 stages; a CTA of the balanced
// round pays about 36 more (writing a partial slot, the refill before its
// next piece, and finishing a split tile from another CTA's slot).  The
// balanced round must win by 5 % to be used.
struct SplitPlan {
    int dp_tiles, sk_tiles, sk_ctas;
};

SplitPlan plan_split(const Geometry& g, int G) {
    SplitPlan pl{g.tiles, 0, 0};
    if (G <= 0 || g.tiles % G == 0) return pl;
    const int rounds = g.tiles / G;
    const int dp = rounds >= 1 ? (rounds - 1) * G : 0;
    const int skt = g.tiles - dp;
    if ((long long)skt * g.nk < 4ll * G) return pl;   // too little work to share out
    // both overheads scale with the activation rows of a tile (bt) on top of a
    // fixed part: at bt = 256 they are the measured 10 and 36 stages
    const double r = g.bt / 256.0;
    const double kEpi = 2.0 + 8.0 * r, kSplit = 8.0 + 28.0 * r;
    const double dp_cost = (double)((g.tiles + G - 1) / G) * (g.nk + kEpi);
    const double sk_cost = (double)(dp / G) * (g.nk + kEpi) + (double)skt * g.nk / G + kSplit;
    if (sk_cost >= 0.95 * dp_cost) return pl;
    pl.dp_tiles = dp;
    pl.sk_tiles = skt;
    pl.sk_ctas = G;
    return pl;
}

inline size_t round256(size_t v) { return (v + 255) / 256 * 256; }

// Scratch of a balanced round: arrival counters, then two partial-accumulator
// slots per CTA.
size_t split_bytes(const Geometry& g, const SplitPlan& pl) {
    if (pl.sk_ctas == 0) return 0;
    return round256((size_t)pl.sk_tiles * 4) + (size_t)2 * pl.sk_ctas * g.bt * BW * 4;
}

template <int FORM, int KB, bool SPLIT>
cudaError_t launch_prefill_kb(const int8_t* act, const uint32_t* w, PrefillParams p,
                              cudaStream_t s) {
    constexpr int smem = PS<KB>::SMEM_BYTES;
    constexpr auto kern = SPLIT ? prefill_split_kernel<FORM, KB> : prefill_kernel<FORM, KB>;
    static KernelAttrs kattrs;
    if (cudaError_t e = kattrs.ensure(kern, smem)) return e;
    CUtensorMap ta, tw;
    if (!make_tmap(&ta, act, (uint64_t)p.rows_a, (uint64_t)p.K, BK, (uint32_t)p.bt,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const uint64_t prow = (uint64_t)p.K / (FORM == 0 ? 4 : 8);
    if (!make_tmap(&tw, w, (uint64_t)p.N, prow, PF<FORM>::kPackedRowBytes * KB, BW,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    // y as bytes: N * 2 per row; one box = 128 columns x the tile's tokens
    CUtensorMap ty;
    if (!make_tmap(&ty, p.y, (uint64_t)p.M, (uint64_t)p.N * 2, BW * 2, (uint32_t)p.tpt,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    p.wait_ns = kWaitLimitNs;
    p.stall = 0;
    if (!SPLIT) {
        const unsigned long long stall = take_stall();
        if (stall) {
            p.wait_ns = stall;
            p.stall = 1;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.dp_tiles + p.sk_ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, ta, tw, ty, p);
}

template <int FORM>
cudaError_t launch_prefill(const int8_t* act, const uint32_t* w, PrefillParams p, void* split_ws,
                           size_t split_ws_bytes, cudaStream_t s) {
    const Geometry g = geometry(FORM, p.M, p.K, p.N);
    p.bt = g.bt;
    p.tpt = g.tpt;
    p.rpt = FORM == 0 ? g.bt : 3 * g.tpt;   // a token tile's first activation row
    SplitPlan pl = plan_split(g, device_sm_count());
    const size_t need = split_bytes(g, pl);
    if (need == 0 || split_ws == nullptr || split_ws_bytes < need) pl = SplitPlan{g.tiles, 0, 0};
    p.dp_tiles = pl.dp_tiles;
    p.sk_tiles = pl.sk_tiles;
    p.sk_ctas = pl.sk_ctas;
    p.sk_ctr = pl.sk_ctas ? static_cast<unsigned int*>(split_ws) : nullptr;
    p.sk_slots = pl.sk_ctas ? reinterpret_cast<int32_t*>(static_cast<char*>(split_ws) +
                                                         round256((size_t)pl.sk_tiles * 4))
                            : nullptr;
    if (pl.sk_ctas > 0) {
        if (g.kb == 4) return launch_prefill_kb<FORM, 4, true>(act, w, p, s);
        if (g.kb == 2) return launch_prefill_kb<FORM, 2, true>(act, w, p, s);
        return launch_prefill_kb<FORM, 1, true>(act, w, p, s);
    }
    if (g.kb == 4) return launch_prefill_kb<FORM, 4, false>(act, w, p, s);
    if (g.kb == 2) return launch_prefill_kb<FORM, 2, false>(act, w, p, s);
    return launch_prefill_kb<FORM, 1, false>(act, w, p, s);
}

}  // namespace

void prefill_plan_info(int form, int M, int K, int N, int sm_count, int plan[5]) {
    const Geometry g = geometry(form, M, K, N);
    const SplitPlan pl = plan_split(g, sm_count);
    plan[0] = g.bt;
    plan[1] = g.nk;
    plan[2] = g.tiles;
    plan[3] = pl.dp_tiles;
    plan[4] = pl.sk_tiles;
}

size_t prefill_split_bytes(int form, int M, int K, int N, int* n_counters) {
    *n_counters = 0;
    if (M <= 0 || N <= 0) return 0;
    const Geometry g = geometry(form, M, K, N);
    const SplitPlan pl = plan_split(g, device_sm_count());
    *n_counters = pl.sk_tiles;
    return split_bytes(g, pl);
}

cudaError_t launch_ternary_prefill(const uint32_t* w2, const int8_t* qp, const float* scale,
                                   const int32_t* qsum, int M, int K, int N, float w_scale,
                                   uint16_t* y, int32_t* acc_out, unsigned int* flags,
                                   cudaStream_t s, void* split_ws, size_t split_ws_bytes) {
    if (M == 0 || N == 0) return cudaSuccess;
    PrefillParams p{M, 0, 0, 0, M, K, N, scale, qsum, nullptr, nullptr, w_scale, y, acc_out,
                    flags, nullptr, 0, 0, 0, nullptr, nullptr, 0, 0};
    return launch_prefill<0>(qp, w2, p, split_ws, split_ws_bytes, s);
}

cudaError_t launch_onebit_prefill(const uint32_t* s1, const int8_t* planes, const float* step,
                                  const long long* tsum, const uint16_t* h, int M, int K, int N,
                                  uint16_t* y, unsigned int* flags, cudaStream_t s,
                                  void* split_ws, size_t split_ws_bytes, float* zf) {
    if (M == 0 || N == 0) return cudaSuccess;
    PrefillParams p{3 * M, 0, 0, 0, M, K, N, step, nullptr, tsum, h, 0.f, y, nullptr, flags, zf,
                    0, 0, 0, nullptr, nullptr, 0, 0};
    return launch_prefill<1>(planes, s1, p, split_ws, split_ws_bytes, s);
}

}  // namespace bl
