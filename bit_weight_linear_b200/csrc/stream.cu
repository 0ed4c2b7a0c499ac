// stream.cu -- streamed decode-shaped (small M) forward of both layer forms:
// one 512-thread CTA per SM owns a contiguous range of 16-row weight tiles and
// streams them through a shared-memory ring.
//
// Arithmetic is that of the other decode kernels:
//   BitLinear (BitNet b1.58 page, "BitNet b1.58 介绍"): per-token absmax int8
//     q = rne(x * rn(127/amax)), acc = sum q*code - sum q, y = fp16((acc*s)*w_scale);
//   OneBit (OneBit page, "1. 新的 1bit 结构"): 23-bit fixed-point image X of
//     x*g in three int8 limbs, sum X*S = 2 sum X*b - sum X, y = fp16(step*Z*h).
//
// Why this shape on B200.  At M = 1 a call is a chain: wait for the previous
// grid, read x, reduce its absmax, quantise, contract, write y.  The weights
// do not depend on that chain, so they are read before it:
//   * The grid has at most one CTA per SM, and a CTA fits twice per SM
//     (512 threads x 64 registers, <= 112 KB shared memory), so the CTA of the
//     NEXT call becomes resident beside the running one and streams its tiles
//     while this call finishes (programmatic dependent launch).
//   * At launch, one thread fills the ring: ONE 3-D TMA load per stage
//     (16 rows x up to 32 k-steps, laid out [step][row][64 B], so the MMA
//     fragment loads are bank-conflict free).  Large copies matter: per-row
//     1 KB bulk copies stream at under half of HBM bandwidth per SM, 8 KB and
//     larger ones at full rate.  x is prefetched into L2.  Only then does the
//     CTA wait for the preceding grid.
//   * x is quantised once per SM (not once per 16 rows), by all 16 warps.
//   * Warps split each ring stage's 256-k (ternary) / 512-k (sign) steps and
//     run the u8 x s8 warp MMA; the last warp to finish a stage refills its
//     slot.  Per-tile partial sums meet in shared memory through integer
//     atomics (exact in any order).
#include "common.cuh"
#include "act_groups.cuh"
#include "decode_forms.cuh"
#include "kernels.h"
#include "tc_prims.cuh"
#include "tmap.cuh"

#include <mutex>

namespace bl {

namespace {

constexpr int kSWarps = 16;
constexpr int kSThreads = kSWarps * 32;
constexpr int kMaxSlots = 16;
constexpr int kMaxTokS = 32;
constexpr uint64_t kSWaitLimitNs = 2000000000ull;
constexpr uint64_t kSDrainLimitNs = 100000000ull;
// two CTAs per SM: (228 KB - 2 x 1 KB reserved) / 2, rounded down
constexpr int kStreamSmemPair = 112 * 1024;

struct StreamParams {
    const int8_t* prep;     // prepared activations [cols][K] (PREP kernels only)
    const float* pscale;    // per token: scale (ternary) / fixed-point step (OneBit)
    const int32_t* prsum;   // ternary, per token: row sum of the prepared activations
    const long long* prsum64;  // OneBit, per token: sum of the fixed-point image
    const uint16_t* x;
    const uint16_t* g;      // OneBit input value vector
    const uint16_t* h;      // OneBit output value vector
    const uint32_t* w;      // packed weights
    float w_scale;
    int M, K, N;
    uint16_t* y;
    int32_t* acc_out;
    float* zf;              // OneBit: optional fp32 [M][N] copy of the output before fp16 rounding
    unsigned int* flags;
    // plan (host-computed)
    int t_lo, t_rem, t_max;  // tiles per CTA: t_lo + (cta < t_rem)
    int steps, nch, S;       // k-steps per row, ring stages per tile, ring slots
    int nfull, bsteps;       // whole 64-byte steps per row; steps per stage (box depth)
    int ragged;              // 1: the last step is partial: `tail` bytes per row (tail map)
    int tail;                // 16, 32 or 48 bytes (sign); 32 (ternary)
    int slot_bytes;
    int compact;             // 1: per-tile reduction through one [16 warps][16][cols] scratch
    int off_act, astride, off_red, off_tok, off_h, off_bar, off_cnt;
    // Bounded waits: the limit of a ring-stage wait (2 s).  Test hook
    // (bl_debug_stall_next_launch): stall = 1 leaves CTA 0's first stage
    // unrequested, so its wait runs out after wait_ns.
    uint64_t wait_ns;
    int stall;
};

// Steps [s0, s1) of chunk c of a tile: chunks of bsteps steps, the last one
// shorter (its box runs past the row end and is zero-filled without reading).
struct Chunk {
    int s0, s1;
};
__host__ __device__ __forceinline__ Chunk chunk_of(int c, int steps, int bsteps) {
    Chunk ch;
    ch.s0 = c * bsteps;
    ch.s1 = min(ch.s0 + bsteps, steps);
    return ch;
}

// sum of one partial over the NW warps' copies (warp stride `stride` ints)
template <int NW>
__device__ __forceinline__ int warp_rows_sum(const int* red, int idx, int stride) {
    int v = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += red[w * stride + idx];
    return v;
}

// partial sum idx ([row][col] over the CTA's tiles): the NW warps' copies, or
// the compact mode's reduced result rows
template <int NW>
__device__ __forceinline__ int tile_sum(const int* red, const StreamParams& p, int idx, int ncols) {
    return p.compact ? red[NW * 16 * ncols + idx] : warp_rows_sum<NW>(red, idx, p.t_max * 16 * ncols);
}

// Ring stage u = (tile u / nch, chunk u % nch): one box of bsteps whole steps
// ([step][row][64 B]) and, for the chunk holding a partial last step, the tail
// box ([row][tail B]) behind it.  The caller arms the barrier with stage_bytes.
__device__ __forceinline__ uint32_t stage_bytes(const StreamParams& p, int u) {
    const Chunk ch = chunk_of(u % p.nch, p.steps, p.bsteps);
    uint32_t b = ch.s0 < p.nfull ? (uint32_t)p.bsteps * 1024u : 0u;
    if (p.ragged && ch.s1 == p.steps) b += 16u * (uint32_t)p.tail;
    return b;
}

__device__ __forceinline__ void issue_stage(const StreamParams& p, const CUtensorMap* tm_main,
                                            const CUtensorMap* tm_tail, uint32_t sb, int tile0,
                                            int u) {
    const int lt = u / p.nch;
    const Chunk ch = chunk_of(u - lt * p.nch, p.steps, p.bsteps);
    const int slot = u % p.S;
    const uint32_t dst = sb + slot * p.slot_bytes;
    const uint32_t bar = sb + p.off_bar + 8 * slot;
    const int row0 = (tile0 + lt) * 16;
    if (ch.s0 < p.nfull) tc::tma_load_3d(dst, tm_main, 0, row0, ch.s0, bar);
    if (p.ragged && ch.s1 == p.steps) tc::tma_load_2d(dst + p.bsteps * 1024, tm_tail, 0, row0, bar);
}

// PREP = 0: the CTA prepares the activations from x.
//   XREG != 0: warp-local preparation with x in registers; 1, 2: M == 1
//   (2 when K is a whole number of steps, so the contraction has no partial
//   step to guard); 3: M > 1 (up to 2 units per lane, 1 for sign); 4: M > 1,
//   4 units per lane, whole steps (ternary).
//   XREG = 0: general M, x read twice (second pass from L1/L2).
// PREP = 1: the activation kernel prepared them; they are copied in.
// NW: warps per CTA (16; 8 for single-token launches with a register
// preparation, where each warp takes more steps of a stage and the per-stage
// warp overhead -- waits, releases, folds -- is paid half as often).
template <int FORM, int NT, int PREP, int XREG, int NW = kSWarps>
__global__ void __launch_bounds__(NW * 32, 2)
    stream_kernel(const __grid_constant__ CUtensorMap tm_main,
                  const __grid_constant__ CUtensorMap tm_tail, const StreamParams p) {
    using F = DF<FORM>;
    constexpr int CH = 4 / NT;  // independent accumulator chains per column tile
    // ternary with one column tile: in-place masked unpack (one AND per register)
    constexpr bool kMasked = FORM == 0 && NT == 1;
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int kW = NW, kT = NW * 32;
    const int K = p.K, M = p.M;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sb = tc::smem_u32(smem);
    const int cta = blockIdx.x;
    const int T = p.t_lo + (cta < p.t_rem ? 1 : 0);
    const int tile0 = cta * p.t_lo + min(cta, p.t_rem);
    const int nstages = T * p.nch;
    const int S = p.S;
    const int ncols = M * F::kCPT;
    uint8_t* act = smem + p.off_act;
    int* racc = reinterpret_cast<int*>(smem + p.off_red);             // [NW warps][t_max*16][ncols]
    float* red_max = reinterpret_cast<float*>(smem + p.off_tok);      // [NW][M]
    constexpr int LS = FORM == 1 ? 3 : 1;                             // row sums per token
    int* red_sum = reinterpret_cast<int*>(red_max + kW * M);          // [NW][M][LS]
    uint16_t* hs = reinterpret_cast<uint16_t*>(smem + p.off_h);       // [t_max*16]
    uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + p.off_cnt);    // [S] releases, [S] rounds issued
    const uint32_t cnt_sb = sb + p.off_cnt;

    // 1. weights and parameters: independent of the preceding grid
    if (tid == 0) {
        for (int i = 0; i < S; ++i) tc::mbar_init(sb + p.off_bar + 8 * i, 1);
        tc::mbar_fence_init();
        if (p.nfull > 0) tc::prefetch_tmap(&tm_main);
        if (p.ragged) tc::prefetch_tmap(&tm_tail);
    }
    for (int i = tid; i < 2 * S; i += kT) cnt[i] = 0;
    if (FORM == 1)
        for (int i = tid; i < T * 16; i += kT) hs[i] = p.h[tile0 * 16 + i];
    // Warp-local activation preparation (XREG): warp w owns the k-steps
    // s = w, w + 16, ... (the steps it contracts).  Its work is the units
    // (token m, group q of its owned steps), token-major; lane l takes units
    // l, l + 32, ... (at most U).  OneBit's g is a parameter, read before the wait.
    constexpr int G = F::kGroup;
    constexpr bool kOne = XREG == 1 || XREG == 2;            // M == 1 variants
    // units per lane: OneBit's 32-element units also hold their g, so two of
    // them only for one token on 8 warps (16 would spill at 64 registers)
    constexpr int U = XREG == 4 ? 4 : (FORM == 0 || (kOne && NW == 8) ? 2 : 1);
    const int Mx = kOne ? 1 : M;                             // compile-time 1 for M == 1
    int um[U], uk[U];
    bool has[U];
    if constexpr (XREG != 0) {
        const int own = warp < p.steps ? (p.steps - 1 - warp) / kW + 1 : 0;
        const int gw = own * 16;  // groups per token owned by this warp
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int v = lane + 32 * i;
            int m, q;
            if constexpr (kOne) {
                m = v < gw ? 0 : 1;
                q = v;
            } else {
                m = gw > 0 ? v / gw : M;
                q = gw > 0 ? v - m * gw : 0;
            }
            um[i] = m;
            uk[i] = (warp + kW * (q >> 4)) * F::kStepK + (q & 15) * G;
            has[i] = m < Mx && uk[i] < K;
        }
    }
    // OneBit: each unit's g (with several tokens, a lane's units share one group)
    constexpr int UG = FORM == 1 && kOne ? U : 1;
    uint4 ga[UG][4];
    if constexpr (FORM == 1 && XREG != 0) {
#pragma unroll
        for (int i = 0; i < UG; ++i) {
            if (has[i]) {
#pragma unroll
                for (int v = 0; v < 4; ++v) ga[i][v] = ld_gvec(p.g, uk[i] + 8 * v);
            }
        }
    }
    __syncthreads();  // barriers initialised, counters zeroed
    tc::pdl_trigger();
    if (tid == 0) {
        const int nfill = min(S, nstages);
        for (int u = 0; u < nfill; ++u) {
            if (p.stall && cta == 0 && u == 0) continue;   // test hook: a stage that never comes
            tc::mbar_arrive_expect_tx(sb + p.off_bar + 8 * u, stage_bytes(p, u));
            issue_stage(p, &tm_main, &tm_tail, sb, tile0, u);
        }
    } else if (!PREP && cta == 0 && tid == 32) {
        tc::bulk_prefetch_l2(p.x, (uint32_t)(2 * (size_t)M * K));
    }
    tc::pdl_wait();

    // 2. activations
    float tok_amax = 0.f;  // XREG: the token's absmax, kept for the epilogue
    if (PREP) {
        const int per_row = K / 16;
        for (int c = tid; c < ncols * per_row; c += kT) {
            const int row = c / per_row, off = c - row * per_row;
            tc::cp_async16(sb + p.off_act + row * p.astride + 16 * off,
                           p.prep + (size_t)row * K + 16 * off);
        }
        tc::cp_async_wait_all();
        __syncthreads();
    } else if (XREG) {
        // M <= 8 (ternary) / 2 (sign): x stays in registers; one CTA barrier
        // (the per-token absmax); each warp then quantises exactly the steps it
        // contracts, so the contraction needs only the warp's own writes
        uint4 xa[U][G / 8];
        float umx[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            if (has[i]) {
#pragma unroll
                for (int v = 0; v < G / 8; ++v) xa[i][v] = tc::ld_v4(p.x + (size_t)um[i] * K + uk[i] + 8 * v);
            }
        }
#pragma unroll
        for (int i = 0; i < U; ++i) {
            umx[i] = 0.f;
            if (!has[i]) continue;
            if constexpr (FORM == 0) {
                umx[i] = hbits(max(absmax_bits_t(xa[i][0]), absmax_bits_t(xa[i][1])));
            } else {
#pragma unroll
                for (int v = 0; v < G / 8; ++v)
                    umx[i] = fmaxf(umx[i], absmax_prod(xa[i][v], ga[UG > 1 ? i : 0][v]));
            }
        }
        // non-negative floats order like their bit patterns: one redux.sync max per token
        for (int m = 0; m < Mx; ++m) {
            float v = 0.f;
#pragma unroll
            for (int i = 0; i < U; ++i)
                if (has[i] && um[i] == m) v = fmaxf(v, umx[i]);
            v = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
            if (lane == 0) red_max[warp * Mx + m] = v;
        }
        __syncthreads();
        // lane m < M reduces token m's absmax and inverse step; units fetch theirs by shuffle
        float amax_l = 0.f;
        if (Mx == 1) {
#pragma unroll
            for (int w = 0; w < kW; w += 4) {
                const float4 r4 = *reinterpret_cast<const float4*>(red_max + w);
                amax_l = fmaxf(fmaxf(amax_l, r4.x), fmaxf(r4.y, fmaxf(r4.z, r4.w)));
            }
        } else if (lane < Mx) {
#pragma unroll
            for (int w = 0; w < kW; ++w) amax_l = fmaxf(amax_l, red_max[w * Mx + lane]);
        }
        tok_amax = amax_l;
        const float qmax = FORM == 0 ? 127.0f : kImgMaxF;
        const float inv_l = amax_l > 0.f ? __fdiv_rn(qmax, amax_l) : 0.f;
        int usum[U][LS];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const float inv = Mx == 1 ? inv_l : __shfl_sync(0xffffffffu, inv_l, um[i] < Mx ? um[i] : 0);
#pragma unroll
            for (int l = 0; l < LS; ++l) usum[i][l] = 0;
            if (!has[i]) continue;
            uint8_t* dst = act + (kOne ? 0 : um[i]) * F::kCPT * p.astride + uk[i];
            if constexpr (FORM == 0) {
                usum[i][0] = quant_group_t(xa[i][0], xa[i][1], inv, dst);
            } else {
                quant_group_s(xa[i], ga[UG > 1 ? i : 0], inv, dst, p.astride, usum[i]);
            }
        }
        for (int m = 0; m < Mx; ++m) {
#pragma unroll
            for (int l = 0; l < LS; ++l) {
                int v = 0;
#pragma unroll
                for (int i = 0; i < U; ++i)
                    if (has[i] && um[i] == m) v += usum[i][l];
                v = __reduce_add_sync(0xffffffffu, v);
                if (lane == 0) red_sum[(warp * Mx + m) * LS + l] = v;
            }
        }
        __syncwarp();
    } else {
        // general M: x is read twice (the second pass hits L1/L2)
        constexpr int G = F::kGroup;
        const int ngroups = K / G;
        for (int m = 0; m < M; ++m) {
            const uint16_t* xr = p.x + (size_t)m * K;
            float mx = 0.f;
            for (int i = tid; i < ngroups; i += kT) {
                if (FORM == 0) {
                    const uint32_t mb = max(absmax_bits_t(tc::ld_v4(xr + 16 * i)),
                                            absmax_bits_t(tc::ld_v4(xr + 16 * i + 8)));
                    mx = fmaxf(mx, hbits(mb));
                } else {
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        mx = fmaxf(mx, absmax_prod(tc::ld_v4(xr + 32 * i + 8 * v),
                                                   ld_gvec(p.g, 32 * i + 8 * v)));
                }
            }
            mx = warp_max(mx);
            if (lane == 0) red_max[warp * M + m] = mx;
        }
        __syncthreads();
        for (int m = 0; m < M; ++m) {
            const uint16_t* xr = p.x + (size_t)m * K;
            float amax = 0.f;
#pragma unroll
            for (int w = 0; w < kW; ++w) amax = fmaxf(amax, red_max[w * M + m]);
            int sum = 0;
            if (FORM == 0) {
                const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
                for (int i = tid; i < ngroups; i += kT)
                    sum += quant_group_t(tc::ld_v4(xr + 16 * i), tc::ld_v4(xr + 16 * i + 8), inv,
                                         act + m * p.astride + 16 * i);
            } else {
                const float inv = amax > 0.f ? __fdiv_rn(kImgMaxF, amax) : 0.f;
                int ls3[3] = {0, 0, 0};
                for (int i = tid; i < ngroups; i += kT) {
                    uint4 xa[4], gg[4];
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        xa[v] = tc::ld_v4(xr + 32 * i + 8 * v);
                        gg[v] = ld_gvec(p.g, 32 * i + 8 * v);
                    }
                    int gs[3];
                    quant_group_s(xa, gg, inv, act + (3 * m) * p.astride + 32 * i, p.astride, gs);
                    ls3[0] += gs[0];
                    ls3[1] += gs[1];
                    ls3[2] += gs[2];
                }
#pragma unroll
                for (int l = 0; l < 3; ++l) {
                    const int v = warp_sum(ls3[l]);
                    if (lane == 0) red_sum[(warp * M + m) * LS + l] = v;
                }
            }
            if (FORM == 0) {
                sum = warp_sum(sum);
                if (lane == 0) red_sum[warp * M + m] = sum;
            }
        }
        __syncthreads();
    }

    // 3. contraction, one ring stage at a time (tile-major).  The warps split a
    // stage's steps; a warp accumulates a tile in registers (CH independent
    // chains) and adds it into its own rows of wred, which the epilogue sums
    // over the 16 warps (no atomics).
    const int g8 = lane >> 2, t = lane & 3;
    const uint8_t* bsrc[NT];
    bool bvalid[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + g8;
        bvalid[nt] = col < ncols;
        bsrc[nt] = act + (bvalid[nt] ? col : 0) * p.astride + t * F::kChunkK;
    }
    // this warp's partial sums: [t_max*16][ncols], or (compact) [16][ncols] for the current tile
    // (M = 1 kernels never use the compact layout: its code is compiled out there)
    const bool compact = XREG == 0 && p.compact;
    int* wred_w = racc + warp * (compact ? 16 : p.t_max * 16) * ncols;
    int acc[NT][CH][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < CH; ++c) acc[nt][c][0] = acc[nt][c][1] = acc[nt][c][2] = acc[nt][c][3] = 0;
    bool ok = true;
    int slot = 0, phase = 0, chunk = 0, lt = 0;  // stage u = lt * nch + chunk, in slot u % S
    for (int u = 0; u < nstages; ++u) {
        // compact mode has CTA barriers inside the loop: a failed wait skips
        // the work but keeps the warp in step until the tile's barrier, where
        // the CTA agrees to stop
        if (!compact) {
            ok = __all_sync(0xffffffffu, tc::mbar_wait(sb + p.off_bar + 8 * slot, (uint32_t)phase,
                                                       p.flags, p.wait_ns));
            if (!ok) break;
        } else if (ok) {
            ok = __all_sync(0xffffffffu, tc::mbar_wait(sb + p.off_bar + 8 * slot, (uint32_t)phase,
                                                       p.flags, p.wait_ns));
        }
        const int s0 = chunk * p.bsteps, s1 = ok ? min(s0 + p.bsteps, p.steps) : s0;
        const uint8_t* slot_p = smem + slot * p.slot_bytes;
        for (int s = s0 + warp; s < s1; s += kW) {
            // whole step: [step][row][64 B]; partial last step: tail box [row][tail B]
            const bool part = (XREG == 2 || XREG == 4) ? false : s >= p.nfull;
            const uint8_t* w0 = part ? slot_p + p.bsteps * 1024 + p.tail * g8 + 16 * t
                                     : slot_p + (s - s0) * 1024 + 64 * g8 + 16 * t;
            const int rs8 = part ? 8 * p.tail : 512;  // 8 rows further down
            const bool lane_ok = XREG == 2 || XREG == 4 || s * F::kStepK + t * F::kChunkK < K;
            uint4 a0 = make_uint4(0, 0, 0, 0), a1 = make_uint4(0, 0, 0, 0);
            if (lane_ok) {
                a0 = *reinterpret_cast<const uint4*>(w0);
                a1 = *reinterpret_cast<const uint4*>(w0 + rs8);
            }
            const uint32_t r0[4] = {a0.x, a0.y, a0.z, a0.w};
            const uint32_t r1[4] = {a1.x, a1.y, a1.z, a1.w};
            if constexpr (kMasked) {
                // ternary, one column tile: field j of every byte is masked in
                // place (value code * 4^j) and multiplies activation word j; the
                // two words of a pair share j, so each MMA has one scale 4^j and
                // accumulates into chain j
                uint32_t b[4][4];
#pragma unroll
                for (int om = 0; om < 4; ++om) {
                    if (lane_ok && bvalid[0]) {
                        const uint4 bv = *reinterpret_cast<const uint4*>(bsrc[0] + s * F::kStepK + 16 * om);
                        b[om][0] = bv.x;
                        b[om][1] = bv.y;
                        b[om][2] = bv.z;
                        b[om][3] = bv.w;
                    } else {
                        b[om][0] = b[om][1] = b[om][2] = b[om][3] = 0;
                    }
                }
#pragma unroll
                for (int op = 0; op < 4; op += 2)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t m = 0x03030303u << (2 * j);
                        mma_u8s8_16832(acc[0][j], r0[op] & m, r1[op] & m, r0[op + 1] & m,
                                       r1[op + 1] & m, b[op][j], b[op + 1][j]);
                    }
            } else {
#pragma unroll
            for (int om = 0; om < 4; ++om) {
                uint32_t u0r[F::kRegs], u1r[F::kRegs];
#pragma unroll
                for (int j = 0; j < F::kRegs; ++j) {
                    u0r[j] = (r0[om] >> (F::kShift * j)) & F::kMask;
                    u1r[j] = (r1[om] >> (F::kShift * j)) & F::kMask;
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint32_t b[F::kRegs];
                    if (lane_ok && bvalid[nt]) {
                        const uint8_t* src = bsrc[nt] + s * F::kStepK + om * (4 * F::kRegs);
#pragma unroll
                        for (int q = 0; q < F::kRegs / 4; ++q) {
                            const uint4 bv = *reinterpret_cast<const uint4*>(src + 16 * q);
                            b[4 * q + 0] = bv.x;
                            b[4 * q + 1] = bv.y;
                            b[4 * q + 2] = bv.z;
                            b[4 * q + 3] = bv.w;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < F::kRegs; ++j) b[j] = 0;
                    }
#pragma unroll
                    for (int j = 0; j < F::kRegs; j += 2)
                        mma_u8s8_16832(acc[nt][om % CH], u0r[j], u1r[j], u0r[j + 1], u1r[j + 1],
                                       b[j], b[j + 1]);
                }
            }
            }
        }
        // release the slot (only when it is to be refilled); the warp that
        // releases it last refills it
        if (ok && u + S < nstages) {
            __syncwarp();
            if (lane == 0) {
                const uint32_t old = tc::atom_add_acq_rel_smem(cnt_sb + 4 * slot, 1u);
                if ((old + 1) % kW == 0) {
                    tc::fence_proxy_async_smem();
                    const int un = u + S;
                    tc::mbar_arrive_expect_tx(sb + p.off_bar + 8 * slot, stage_bytes(p, un));
                    issue_stage(p, &tm_main, &tm_tail, sb, tile0, un);
                    cnt[S + slot] = (uint32_t)(un / S);  // newest round issued into the slot
                }
            }
            __syncwarp();
        }
        if (chunk == p.nch - 1) {
            // tile finished: fold the chains into the warp's partial sums
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int v = 0;
#pragma unroll
                    for (int cc = 0; cc < CH; ++cc) {
                        // masked chains hold 4^cc times their sums (exact shifts)
                        v += kMasked ? (acc[nt][cc][e] >> (2 * cc)) : acc[nt][cc][e];
                        acc[nt][cc][e] = 0;
                    }
                    const int row = g8 + 8 * (e >> 1), col = nt * 8 + 2 * t + (e & 1);
                    // compact: wred_w is this warp's [16][ncols] scratch for the tile
                    if (col < ncols) wred_w[((compact ? 0 : lt) * 16 + row) * ncols + col] = v;
                }
            }
            if (compact) {
                // add the 16 warps' partials of this tile into its result rows
                if (!__syncthreads_and(ok)) {
                    ok = false;
                    break;
                }
                int* res = racc + kW * 16 * ncols;  // [t_max*16][ncols]
                for (int i = tid; i < 16 * ncols; i += kT)
                    res[lt * 16 * ncols + i] = warp_rows_sum<kW>(racc, i, 16 * ncols);
                __syncthreads();
            }
        }
        if (++slot == S) {
            slot = 0;
            phase ^= 1;
        }
        if (++chunk == p.nch) {
            chunk = 0;
            ++lt;
        }
    }
    if (!__syncthreads_and(ok)) {
        // a stage never arrived: let the copies still in flight land before the
        // CTA's shared memory is released, then leave (the flag is set)
        if (tid == 0) {
            for (int sl = 0; sl < min(S, nstages); ++sl) {
                if (p.stall && cta == 0 && sl == 0) continue;   // nothing was ever requested there
                tc::mbar_wait(sb + p.off_bar + 8 * sl, cnt[S + sl] & 1u, p.flags, kSDrainLimitNs);
            }
        }
        __syncthreads();
        return;
    }

    // 4. epilogue: one output per thread and step, consecutive threads on consecutive n
    const int rows = T * 16;
    if (FORM == 0) {
        for (int o = tid; o < M * rows; o += kT) {
            const int m = o / rows, r = o - m * rows;
            float sc;
            int qs = 0;
            if (PREP) {
                sc = p.pscale[m];
                qs = p.prsum[m];
            } else {
                float amax = tok_amax;
                if (kOne) {  // M == 1: the 16 warp sums are contiguous
#pragma unroll
                    for (int w = 0; w < kW; w += 4) {
                        const int4 r4 = *reinterpret_cast<const int4*>(red_sum + w);
                        qs += (r4.x + r4.y) + (r4.z + r4.w);
                    }
                } else {
                    amax = 0.f;
#pragma unroll
                    for (int w = 0; w < kW; ++w) {
                        amax = fmaxf(amax, red_max[w * M + m]);
                        qs += red_sum[w * M + m];
                    }
                }
                sc = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
            }
            const int accv = tile_sum<kW>(racc, p, r * ncols + m, ncols) - qs;
            const int n = tile0 * 16 + r;
            const float v = __fmul_rn(__fmul_rn((float)accv, sc), p.w_scale);
            p.y[(size_t)m * p.N + n] = __half_as_ushort(__float2half_rn(v));
            if (p.acc_out) p.acc_out[(size_t)m * p.N + n] = accv;
        }
    } else {
        for (int o = tid; o < M * rows; o += kT) {
            const int m = o / rows, r = o - m * rows;
            float st;
            long long ts = 0;
            if (PREP) {
                st = p.pscale[m];
                ts = p.prsum64[m];
            } else {
                float amax = kOne ? tok_amax : 0.f;
#pragma unroll
                for (int w = 0; w < kW; ++w) {
                    if (!kOne) amax = fmaxf(amax, red_max[w * M + m]);
                    const int* rs = red_sum + (w * M + m) * LS;
                    ts += 65536ll * rs[0] + 256ll * rs[1] + (long long)rs[2];
                }
                st = amax > 0.f ? __fdiv_rn(amax, kImgMaxF) : 0.f;
            }
            const int c0 = r * ncols + 3 * m;
            const long long Z = limb_combine(tile_sum<kW>(racc, p, c0, ncols),
                                             tile_sum<kW>(racc, p, c0 + 1, ncols),
                                             tile_sum<kW>(racc, p, c0 + 2, ncols), ts);
            const int n = tile0 * 16 + r;
            const float z = __fmul_rn(st, (float)Z);
            const float hv = __half2float(__ushort_as_half(hs[r]));
            const float zh = __fmul_rn(z, hv);
            p.y[(size_t)m * p.N + n] = __half_as_ushort(__float2half_rn(zh));
            if (p.zf) p.zf[(size_t)m * p.N + n] = zh;
        }
    }
}

// ------------------------------------------------------------------ host --

int sm_count() { return device_sm_count(); }

struct StreamPlan {
    int grid, nt, xreg, smem, nw;
};

// Fill the plan fields of p and choose the launch.  Shared memory is laid out
// as: ring slots [S][bsteps][16][64 B] (+ [16][32 B] ragged tail) | activation tile [cols][K+16] | per-tile
// partial sums [t_max*16][cols] int32 | token scratch [2][16][M] | h [t_max*16]
// fp16 | full barriers [S] | release counters [S] + rounds issued [S].
template <int FORM>
bool stream_plan(StreamParams& p, int prep, StreamPlan& pl, int nw = kSWarps) {
    using F = DF<FORM>;
    const int M = p.M, K = p.K, N = p.N;
    const int cols = M * F::kCPT;
    if (M < 1 || M > kMaxTokS || cols > 32 || N % 16 != 0 || K % 128 != 0 || K <= 0) return false;
    // int32 partial sums: the masked ternary chain 3 reaches K/4 * 128 * 127
    if (K > 262144) return false;
    pl.nt = cols <= 8 ? 1 : cols <= 16 ? 2 : 4;
    const int sms = sm_count();
    if (sms <= 0) return false;
    const int tiles = N / 16;
    pl.grid = tiles < sms ? tiles : sms;
    p.t_lo = tiles / pl.grid;
    p.t_rem = tiles % pl.grid;
    p.t_max = p.t_lo + (p.t_rem > 0 ? 1 : 0);
    const int wbytes = K / (F::kPerWord / 4);  // packed bytes per row, a multiple of 16
    p.nfull = wbytes / 64;
    p.tail = wbytes % 64;                      // a partial last step of 16/32/48 bytes
    p.ragged = p.tail != 0 ? 1 : 0;
    p.steps = p.nfull + p.ragged;
    // stage depth: a row's steps in one box when they fit (<= 48 steps), else
    // boxes of a multiple of 16 steps, so every chunk starts at a step that is
    // 0 mod 16 (a warp owns the same steps in every chunk)
    auto set_depth = [&](int max_steps) {
        p.nch = (p.steps + max_steps - 1) / max_steps;
        p.bsteps = (p.steps + p.nch - 1) / p.nch;
        if (p.nch > 1) p.bsteps = (p.bsteps + 15) / 16 * 16;
        p.slot_bytes = (p.bsteps * 1024 + 16 * p.tail + 127) / 128 * 128;
    };
    p.astride = K + 16;
    const int act = cols * p.astride;
    // per-warp partial sums for every tile, or (compact) one tile's worth plus
    // the reduced rows, when the first does not fit beside the activations
    const int red_full = nw * p.t_max * 16 * cols * 4;
    const int red_compact = (nw * 16 + p.t_max * 16) * cols * 4;
    p.compact = act + red_full > kStreamSmemPair / 2 ? 1 : 0;
    // A CTA that would need the compact reduction to fit beside a second CTA
    // takes the SM alone instead, with the full per-warp reduction: the
    // compact mode's two CTA barriers per tile cost more than the lost overlap
    // with the next call (M = 4 on 13824-long rows: 17.8 -> 13.7 us).
    const bool alone = p.compact && act + red_full <= kDecodeMaxSmem / 2;
    if (alone) p.compact = 0;
    const int red = p.compact ? red_compact : red_full;
    const int tok = prep ? 0 : (FORM == 1 ? 4 : 2) * nw * M * 4;  // [NW][M] max + [NW][M][LS] sums
    const int hbytes = FORM == 1 ? p.t_max * 16 * 2 : 0;
    auto up16 = [](int v) { return (v + 15) & ~15; };
    const int fixed = up16(act) + up16(red) + up16(tok) + up16(hbytes) + 16 * kMaxSlots + 8 * kMaxSlots;
    for (int cand = 0; cand < 4; ++cand) {
        // (depth, budget): two CTAs per SM with 48-, 32- then 16-step boxes, else
        // one (from the start for a CTA that takes the SM alone)
        const int depth = cand == 0 ? 48 : cand == 1 ? 32 : 16;
        const int budget = alone || cand == 3 ? kDecodeMaxSmem : kStreamSmemPair;
        set_depth(depth);
        const int nst = p.t_max * p.nch;
        int S = (budget - fixed) / p.slot_bytes;
        if (S > kMaxSlots) S = kMaxSlots;
        if (S > nst) S = nst;
        if (S < 1 || (S < 2 && nst > 1)) continue;
        p.S = S;
        int off = S * p.slot_bytes;
        p.off_act = off;
        off += up16(act);
        p.off_red = off;
        off += up16(red);
        p.off_tok = off;
        off += up16(tok);
        p.off_h = off;
        off += up16(hbytes);
        p.off_bar = off;
        off += 8 * S;
        p.off_cnt = off;
        off += 8 * S;
        pl.smem = off;
        // warp-local preparation: a warp's units (tokens x owned groups) spread
        // over its 32 lanes, at most 2 (4 when K has whole steps) per lane for
        // ternary, for sign 2 at M == 1 on 8 warps and 1 otherwise; M > 1
        // without it is prepared by the activation kernel
        // (xreg 1, 2: M == 1; 3: M > 1; 4: M > 1 with 4 units per lane, whole steps)
        const int units = (p.steps + nw - 1) / nw * 16 * M;
        pl.xreg = 0;
        if (!prep && cols <= 8) {
            if (units <= 32 * (FORM == 0 || (M == 1 && nw == 8) ? 2 : 1))
                pl.xreg = M == 1 ? (p.ragged ? 1 : 2) : 3;
            else if (FORM == 0 && !p.ragged && units <= 128) pl.xreg = 4;
        }
        if (!prep && M > 1 && pl.xreg == 0) return false;
        pl.nw = nw;
        return true;
    }
    return false;
}

template <int FORM, int NT, int PREP, int XREG, int NW = kSWarps>
cudaError_t launch_stream(const CUtensorMap& tm_main, const CUtensorMap& tm_tail,
                          const StreamParams& p, const StreamPlan& pl, cudaStream_t s) {
    constexpr auto kern = stream_kernel<FORM, NT, PREP, XREG, NW>;
    static KernelAttrs kattrs;
    if (cudaError_t e = kattrs.ensure(kern, kDecodeMaxSmem)) return e;
    StreamParams q = p;
    const unsigned long long stall = take_stall();
    q.wait_ns = stall ? stall : kSWaitLimitNs;
    q.stall = stall ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(NW * 32);
    cfg.dynamicSmemBytes = (size_t)pl.smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tm_main, tm_tail, q);
}

template <int FORM, int PREP>
cudaError_t launch_stream_form(StreamParams p, cudaStream_t s) {
    StreamPlan pl;
    // One token: 8 warps whenever the activations still take a register
    // preparation.  A chain of dependent calls runs much slower when its
    // kernels alternate between 8- and 16-warp CTAs (measured: a 7B-shaped
    // stack of single-token calls lost 20 %), so every single-token call of a
    // given form makes the same choice unless K is too long for it.
    bool planned = false;
    if (!PREP && p.M == 1) planned = stream_plan<FORM>(p, PREP, pl, 8) && pl.xreg != 0;
    if (!planned && !stream_plan<FORM>(p, PREP, pl)) return cudaErrorInvalidConfiguration;
    // weights as [step][row][64 B] boxes: dim 0 = the 64 bytes of a step,
    // dim 1 = rows (stride = packed row bytes), dim 2 = steps (stride 64)
    const uint64_t wbytes = (uint64_t)p.K / (DF<FORM>::kPerWord / 4);
    CUtensorMap tm_main = {}, tm_tail = {};
    if (p.nfull > 0) {
        const cuuint64_t dims[3] = {64, (cuuint64_t)p.N, (cuuint64_t)p.nfull};
        const cuuint64_t strides[2] = {wbytes, 64};
        const cuuint32_t box[3] = {64, 16, (cuuint32_t)p.bsteps};
        if (!encode_u8_map(&tm_main, p.w, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidConfiguration;
    }
    if (p.ragged) {
        const cuuint64_t dims[2] = {(cuuint64_t)p.tail, (cuuint64_t)p.N};
        const cuuint64_t strides[1] = {wbytes};
        const cuuint32_t box[2] = {(cuuint32_t)p.tail, 16};
        const uint8_t* tail = reinterpret_cast<const uint8_t*>(p.w) + 64 * (size_t)p.nfull;
        if (!encode_u8_map(&tm_tail, tail, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidConfiguration;
    }
    if constexpr (!PREP) {
        if (pl.xreg) {
            if (pl.nt == 1) {
                if constexpr (FORM == 0)
                    if (pl.xreg == 4)
                        return pl.nw == 8 ? launch_stream<FORM, 1, 0, 4, 8>(tm_main, tm_tail, p, pl, s)
                                          : launch_stream<FORM, 1, 0, 4>(tm_main, tm_tail, p, pl, s);
                if (pl.xreg == 3) return launch_stream<FORM, 1, 0, 3>(tm_main, tm_tail, p, pl, s);
                if (pl.nw == 8)
                    return pl.xreg == 2 ? launch_stream<FORM, 1, 0, 2, 8>(tm_main, tm_tail, p, pl, s)
                                        : launch_stream<FORM, 1, 0, 1, 8>(tm_main, tm_tail, p, pl, s);
                return pl.xreg == 2 ? launch_stream<FORM, 1, 0, 2>(tm_main, tm_tail, p, pl, s)
                                    : launch_stream<FORM, 1, 0, 1>(tm_main, tm_tail, p, pl, s);
            }
            return cudaErrorInvalidConfiguration;  // M == 1 always has one column tile
        }
    }
    switch (pl.nt) {
        case 1: return launch_stream<FORM, 1, PREP, 0>(tm_main, tm_tail, p, pl, s);
        case 2: return launch_stream<FORM, 2, PREP, 0>(tm_main, tm_tail, p, pl, s);
        default: return launch_stream<FORM, 4, PREP, 0>(tm_main, tm_tail, p, pl, s);
    }
}

}  // namespace

bool stream_fits(int form, int M, int K, int N, int prep) {
    StreamParams p = {};
    p.M = M;
    p.K = K;
    p.N = N;
    StreamPlan pl;
    return form == 0 ? stream_plan<0>(p, prep, pl) : stream_plan<1>(p, prep, pl);
}

cudaError_t launch_ternary_stream(const uint16_t* x, const uint32_t* w2, int M, int K, int N,
                                  float w_scale, uint16_t* y, int32_t* acc_out, unsigned int* flags,
                                  cudaStream_t s) {
    StreamParams p = {};
    p.x = x;
    p.w = w2;
    p.w_scale = w_scale;
    p.M = M;
    p.K = K;
    p.N = N;
    p.y = y;
    p.acc_out = acc_out;
    p.flags = flags;
    return launch_stream_form<0, 0>(p, s);
}

cudaError_t launch_onebit_stream(const uint16_t* x, const uint16_t* g, const uint16_t* h,
                                 const uint32_t* s1, int M, int K, int N, uint16_t* y,
                                 unsigned int* flags, cudaStream_t s, float* zf) {
    StreamParams p = {};
    p.zf = zf;
    p.x = x;
    p.g = g;
    p.h = h;
    p.w = s1;
    p.M = M;
    p.K = K;
    p.N = N;
    p.y = y;
    p.flags = flags;
    return launch_stream_form<1, 0>(p, s);
}

cudaError_t launch_ternary_stream_prepared(const int8_t* qp, const float* scale, const int32_t* qsum,
                                           const uint32_t* w2, int M, int K, int N, float w_scale,
                                           uint16_t* y, int32_t* acc_out, unsigned int* flags,
                                           cudaStream_t s) {
    StreamParams p = {};
    p.prep = qp;
    p.pscale = scale;
    p.prsum = qsum;
    p.w = w2;
    p.w_scale = w_scale;
    p.M = M;
    p.K = K;
    p.N = N;
    p.y = y;
    p.acc_out = acc_out;
    p.flags = flags;
    return launch_stream_form<0, 1>(p, s);
}

cudaError_t launch_onebit_stream_prepared(const int8_t* planes, const float* step,
                                          const long long* tsum, const uint16_t* h,
                                          const uint32_t* s1, int M, int K, int N, uint16_t* y,
                                          unsigned int* flags, cudaStream_t s, float* zf) {
    StreamParams p = {};
    p.zf = zf;
    p.prep = planes;
    p.pscale = step;
    p.prsum64 = tsum;
    p.h = h;
    p.w = s1;
    p.M = M;
    p.K = K;
    p.N = N;
    p.y = y;
    p.flags = flags;
    return launch_stream_form<1, 1>(p, s);
}

}  // namespace bl
