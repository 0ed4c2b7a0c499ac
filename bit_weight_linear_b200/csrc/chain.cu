// chain.cu -- persistent single-token (M = 1) forward of a whole list of
// layers in ONE launch: the decode step of a stack of extreme-low-bit linear
// layers (BitNet b1.58 page, "内存和延迟": at decode sizes the time of the
// model goes to its nn.Linear layers, whose cost is reading their weights).
//
// Arithmetic per layer is that of the other decode kernels (stream.cu):
//   BitLinear (BitNet b1.58 page, "BitNet b1.58 介绍"): per-token absmax int8
//     q = rne(x * rn(127/amax)), acc = sum q*code - sum q, y = fp16((acc*s)*w_scale);
//   OneBit (OneBit page, "1. 新的 1bit 结构"): 23-bit fixed-point image X of
//     x*g in three int8 limbs, sum X*S = 2 sum X*b - sum X, y = fp16(step*Z*h).
//
// A layer's input is either given (x) or the output y of an earlier layer of
// the list.  Why one launch: a separate launch per layer costs a kernel
// boundary and then a dependent chain (read x, reduce its absmax, quantise,
// contract, write y) in front of every layer; here the weights of the next
// layers keep streaming while the current one finishes, and the activations
// of the next layer are prepared while the current one is contracted.
//
// One CTA per SM (all co-resident: cooperative launch), three warp roles:
//   warp 0      producer: one thread streams the CTA's weight stages, layer
//               after layer, through an S-slot shared-memory ring (one 3-D TMA
//               box of 16 rows x up to 16 64-byte steps per stage, plus a 2-D
//               box for a partial last step), limited only by free slots;
//   warps 1-8   contraction: u8 x s8 warp MMA (m16n8k32) over the steps of
//               each stage they own, per-tile partial sums added into shared
//               memory with integer atomics (exact in any order);
//   warps 9-15  activations and epilogue: for layers j+1.. (while warps 1-8
//               contract layer j; up to four buffers) the per-token absmax and the
//               quantisation into the permuted int8 tile; for layer j the
//               fp16 outputs, and, when a later layer reads them, one arrival
//               per CTA on the layer's completion counter (release fence).
// A layer whose input is another layer's output waits (bounded, acquire)
// until every CTA has arrived on that layer's counter, then reads its y
// through L2.  A layer with the same input as the layer before it reuses that
// layer's prepared activations.  The tiles of a layer are dealt to the CTAs
// round-robin from a per-layer rotation, so every CTA carries the same share
// of the whole list.
//
// Fused block steps (the BitNet b1.58 page keeps LLaMA's RMSNorm and SwiGLU
// around BitLinear): a layer's input may be an RMSNorm of its source and/or
// SwiGLU(y_src, y_src2), applied to the row in registers before the absmax.
// With a caller buffer the SwiGLU is instead evaluated once per element, in
// the epilogue of the later of the two sources (whose tiles are then dealt
// like the earlier one's, so each thread reads the other output it wrote
// itself), and the layer reads the finished row.
//
// Every wait is bounded (2 s): on expiry the kernel sets the device condition
// word (BL_ERR_TIMEOUT through bl_device_status), and the producer lets every
// copy it requested land before its CTA can exit.
#include "act_groups.cuh"
#include "common.cuh"
#include "decode_forms.cuh"
#include "kernels.h"
#include "tc_prims.cuh"
#include "tmap.cuh"

#include <cstring>
#include <vector>

namespace bl {

namespace {

constexpr int kMmaWarps = 8;
// 16 warps: four per SM sub-partition, whose register file then allows 128
// registers per thread (a 17th warp would put five on one and cap them at 96)
constexpr int kPrepWarps = 7;
constexpr int kPrepThreads = kPrepWarps * 32;
constexpr int kThreads = (1 + kMmaWarps + kPrepWarps) * 32;   // 512
constexpr int kFirstPrepWarp = 1 + kMmaWarps;
constexpr int kMaxTiles = 16;              // tiles of one layer per CTA
constexpr int kMaxSlots = 12;
constexpr int kStageSteps = 16;            // 64-byte steps of a row per stage: 16 KB for 16 rows
// + the [16 rows][<= 48 B] tail box, and room for the 16 bytes past it that lanes
// of a partial step read (they meet zero activations)
constexpr int kSlotBytes = 16 * kStageSteps * 64 + 1024;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kBarPrep = 1;                // named barrier of the activation/epilogue warps
constexpr int kMaxBufs = 4;                // activation buffers: layers prepared ahead

// One layer of a chain in device memory (written by bl_chain_build, read-only
// in the kernel).  448 bytes, 64-byte aligned: the tensor maps come first.
struct alignas(64) ChainLayer {
    CUtensorMap tm_main;   // [step][row][64 B] boxes of 16 rows x bsteps steps
    CUtensorMap tm_tail;   // [row][tail B] box of a partial last step
    const uint16_t* x;     // given input (src < 0)
    const uint32_t* w;     // packed weights
    uint16_t* y;
    int32_t* acc_out;      // optional (ternary)
    const uint16_t* g;     // OneBit input value vector
    const uint16_t* h;     // OneBit output value vector
    const uint16_t* norm_w;  // RMSNorm weight of the input (nullptr: none)
    float w_scale;
    int src;               // -1: x given; else the layer whose y is the input
    int K, N;
    int src2;              // -1, or SwiGLU input: silu(y_src) * y_src2
    float norm_eps;
    int steps, nfull, tail, ragged, bsteps, nch, ntile, rot;
    int has_dep;           // a later layer reads y: arrive on done[] after the epilogue
    int reuse;             // same input as the previous layer: copy its prepared activations
    // SwiGLU evaluated in this layer's epilogue, once per element: for each of
    // its rows n, swi_out[n] = fp16(silu(a) * b) with {a, b} = {y[n], y_q[n]}
    // (a = this layer's y when swi_self_a).  Layer swi_q has the same rows and
    // tile deal, so the thread that writes y[n] here wrote y_q[n] there.
    int swi_q, swi_self_a;
    uint16_t* swi_out;
    int xbuf;              // host only: the input is x = a SwiGLU buffer although src >= 0
};
static_assert(sizeof(ChainLayer) == 448, "chain layer descriptor size");

// The per-layer fields every warp role reads, 32 bytes per layer: written by
// the host next to the descriptors and copied into shared memory at launch.
// A descriptor field read from global memory costs an L2 round trip per layer
// and warp -- for the producer thread, a stall of every stage it issues.
struct alignas(16) LayerInfo {
    uint16_t ntile, rot;    // 16-row tiles; rotation of their deal over the CTAs
    uint16_t k16;           // K / 16
    int16_t src;            // -1: x given; else the producing layer
    uint8_t steps, nfull, tail, bsteps, nch;
    uint8_t flags;          // kInfoRagged | kInfoHasDep | kInfoReuse
    int16_t src2;           // -1, or the second input of a SwiGLU prologue
    const uint16_t* x;      // given input (src < 0)
    uint16_t* y;            // output
};
static_assert(sizeof(LayerInfo) == 32, "layer info size");
// kInfoXbuf: the input is x although src >= 0 (a SwiGLU evaluated by layer src's epilogue)
constexpr uint8_t kInfoRagged = 1, kInfoHasDep = 2, kInfoReuse = 4, kInfoNorm = 8, kInfoXbuf = 16;

struct ChainParams {
    const ChainLayer* layers;
    const LayerInfo* info;  // [n] in global memory
    int n;
    unsigned int* done;    // [n] arrivals of CTAs that finished a layer's epilogue
    unsigned int* flags;   // device condition word
    int S;                 // ring slots
    int nbuf;              // activation buffers (2..kMaxBufs): layer j uses buffer j % nbuf
    int astride;           // bytes between activation rows (Kmax + 16)
    int off_act, off_part, off_tok, off_bar, off_tab;
    uint64_t wait_ns;
};

// Tiles of layer L taken by CTA c of G: first, first + G, ... < ntile.
__device__ __forceinline__ int first_tile(const LayerInfo& L, int c, int G) {
    const int r = (c - (int)L.rot) % G;
    return r < 0 ? r + G : r;
}
__device__ __forceinline__ int tiles_of(const LayerInfo& L, int first, int G) {
    return first < L.ntile ? (L.ntile - 1 - first) / G + 1 : 0;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned int* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bring a read-only fp16 row (an RMSNorm weight) into L1 ahead of use: one
// prefetch per 128-byte line, spread over the activation threads.
__device__ __forceinline__ void prefetch_row_l1(const uint16_t* v, int K, int et, int nthreads) {
    for (int e = 64 * et; e < K; e += 64 * nthreads) asm volatile("prefetch.global.L1 [%0];" ::"l"(v + e));
}

// 16-byte load through L2 only (another CTA's output, after an acquire).
__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ void bar_prep() {
    asm volatile("bar.sync %0, %1;" ::"r"(kBarPrep), "r"(kPrepThreads) : "memory");
}

// Per-layer shared state of the activation/epilogue warps.
struct TokStats {
    float scale[kMaxBufs];       // ternary amax/127, OneBit amax'/kImgMax; per buffer
    int qsum[kMaxBufs];          // ternary sum q
    long long xsum[kMaxBufs];    // OneBit sum X
    uint32_t red[3][kPrepWarps];
    int redi[3][kPrepWarps];
    unsigned long long ss[kPrepWarps][2];   // RMSNorm: per-warp exact sums of squares
};

// ---- fused prologues of a layer's input (the BitNet b1.58 page keeps LLaMA's
// RMSNorm and SwiGLU around BitLinear; definitions in include/bitlinear.h)

// fp16 bits of an fp32 result t whose error is below 16 units in t's last
// place, when that error cannot change the rounding: t lies in the fp16
// normal range and at least 16 fp32 units from the midpoint between two fp16
// values (the 13 mantissa bits fp16 drops are not within 16 of 0x1000).  An
// exact zero is safe too.  Otherwise 0xffffffff: the caller takes the fp64
// definition.
__device__ __forceinline__ uint32_t half_if_safe(float t) {
    const uint32_t b = __float_as_uint(t);
    if ((b & 0x7fffffffu) == 0) return b >> 16;                  // +-0
    const uint32_t e = (b >> 23) & 0xffu;
    if (e < 113 || e > 141) return 0xffffffffu;                  // outside [2^-14, 2^15)
    const int rem = (int)(b & 0x1fffu) - 0x1000;
    if (rem >= -16 && rem <= 16) return 0xffffffffu;
    return __half_as_ushort(__float2half_rn(t));
}

// SwiGLU of one element pair of fp16 bits, the definition fp16((a / (1 +
// exp(-a))) * b) in fp64.  First in fp32: expf is within 2 units in the last
// place, the add, divide and multiply within half a unit each, and 1 + e >= 1
// adds no cancellation, so the fp32 value is within 4 units of the exact one
// and the fp64 definition's value within 2^-50 of it: where half_if_safe
// accepts the fp32 value, both round to the same fp16.
// the fp64 definition, out of line: one copy of the code for every caller
__device__ __noinline__ uint32_t swiglu1_f64(float a, float b) {
    const double x = (double)a, y = (double)b;
    return __half_as_ushort(__double2half(__dmul_rn(__ddiv_rn(x, __dadd_rn(1.0, exp(-x))), y)));
}

__device__ __forceinline__ uint32_t swiglu1(uint32_t ah, uint32_t bh) {
    const float a = __half2float(__ushort_as_half((unsigned short)ah));
    const float b = __half2float(__ushort_as_half((unsigned short)bh));
    const uint32_t f = half_if_safe(__fmul_rn(__fdiv_rn(a, __fadd_rn(1.0f, expf(-a))), b));
    return f != 0xffffffffu ? f : swiglu1_f64(a, b);
}

__device__ __forceinline__ uint4 swiglu8(uint4 a, uint4 b) {
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = swiglu1(av[i] & 0xffffu, bv[i] & 0xffffu) | (swiglu1(av[i] >> 16, bv[i] >> 16) << 16);
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// exact sum of squares of 8 fp16 elements, as a 128-bit integer in units of
// 2^-48: x = mant 2^e (mant < 2^11, e >= -24) gives x^2 2^48 < 2^80
__device__ __forceinline__ void sumsq8(uint4 a, unsigned long long& hi, unsigned long long& lo) {
    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e8 = 0; e8 < 8; ++e8) {
        const uint32_t hb = (av[e8 >> 1] >> (16 * (e8 & 1))) & 0xffffu;
        const int ex = (hb >> 10) & 31;
        const unsigned long long mant = ex ? (1024u | (hb & 1023u)) : (hb & 1023u);
        const int sh = 2 * ((ex ? ex : 1) - 25) + 48;            // 0 .. 58
        const unsigned long long sq = mant * mant;
        const unsigned long long add_lo = sq << sh, add_hi = sh ? sq >> (64 - sh) : 0ull;
        const unsigned long long nlo = lo + add_lo;
        hi += add_hi + (nlo < lo ? 1ull : 0ull);
        lo = nlo;
    }
}

// nearest double (ties to even) of the 128-bit integer hi 2^64 + lo
__device__ __forceinline__ double u128_to_double(unsigned long long hi, unsigned long long lo) {
    if (hi == 0) return __ull2double_rn(lo);
    const int sh = 64 - __clzll((long long)hi);   // drop the low sh bits, keep 64
    const unsigned long long top = sh == 64 ? hi : (hi << (64 - sh)) | (lo >> sh);
    const unsigned long long rest = sh == 64 ? lo : lo & ((1ull << sh) - 1);
    // 53 of top's 64 bits are kept: bit 0 set stands for any nonzero rest
    return ldexp(__ull2double_rn(top | (rest ? 1ull : 0ull)), sh);
}

// RMSNorm of one element, the definition fp16((x r) gamma) in fp64 with r the
// row's fp64 factor.  First in fp32 with r rounded to fp32: three roundings of
// half a unit each, so within 2 units of the exact value; half_if_safe decides
// as for SwiGLU.
__device__ __noinline__ uint32_t norm1_f64(float x, double r, float gm) {
    return __half_as_ushort(__double2half(__dmul_rn(__dmul_rn((double)x, r), (double)gm)));
}

__device__ __forceinline__ uint32_t norm1(uint32_t xh, double r, float r32, uint32_t gh) {
    const float x = __half2float(__ushort_as_half((unsigned short)xh));
    const float gm = __half2float(__ushort_as_half((unsigned short)gh));
    const uint32_t f = half_if_safe(__fmul_rn(__fmul_rn(x, r32), gm));
    return f != 0xffffffffu ? f : norm1_f64(x, r, gm);
}

__device__ __forceinline__ uint4 norm8(uint4 a, double r, float r32, uint4 gq) {
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {gq.x, gq.y, gq.z, gq.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = norm1(av[i] & 0xffffu, r, r32, gv[i] & 0xffffu) |
               (norm1(av[i] >> 16, r, r32, gv[i] >> 16) << 16);
    return make_uint4(o[0], o[1], o[2], o[3]);
}

struct Prologue {
    const uint16_t* x2;      // SwiGLU: the second input (another CTA's output; nullptr: none)
    const uint16_t* gamma;   // RMSNorm weight (nullptr: none)
    double eps;
};

// Apply the prologue to the row held in registers: chunk c (c < nch) holds
// the 8 elements at off(c).
template <int NCH, int BATCH, typename Off>
__device__ __forceinline__ void apply_prologue(uint4 (&xr)[NCH], int nch, Off off, int K,
                                               const Prologue& pro, TokStats* ts, int et) {
    if (pro.x2) {
        // BATCH loads in flight, then their chunks
#pragma unroll
        for (int c0 = 0; c0 < NCH; c0 += BATCH) {
            uint4 t[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i)
                if (c0 + i < NCH && c0 + i < nch) t[i] = ld_cg_v4(pro.x2 + off(c0 + i));
#pragma unroll
            for (int i = 0; i < BATCH; ++i)
                if (c0 + i < NCH && c0 + i < nch) xr[c0 + i] = swiglu8(xr[c0 + i], t[i]);
        }
    }
    if (pro.gamma) {
        const int pw = et >> 5, lane = et & 31;
        unsigned long long hi = 0, lo = 0;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            if (c >= nch) break;
            sumsq8(xr[c], hi, lo);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long h2 = __shfl_xor_sync(0xffffffffu, hi, o);
            const unsigned long long l2 = __shfl_xor_sync(0xffffffffu, lo, o);
            const unsigned long long nlo = lo + l2;
            hi += h2 + (nlo < lo ? 1ull : 0ull);
            lo = nlo;
        }
        if (lane == 0) {
            ts->ss[pw][0] = hi;
            ts->ss[pw][1] = lo;
        }
        bar_prep();
        // every thread forms the same r from the warps' exact partial sums (no
        // second barrier to broadcast it)
        unsigned long long H = 0, Lo = 0;
#pragma unroll
        for (int w = 0; w < kPrepWarps; ++w) {
            const unsigned long long nlo = Lo + ts->ss[w][1];
            H += ts->ss[w][0] + (nlo < Lo ? 1ull : 0ull);
            Lo = nlo;
        }
        const double ssq = ldexp(u128_to_double(H, Lo), -48);
        const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ssq, (double)K), pro.eps)));
        const float r32 = __double2float_rn(r);
#pragma unroll
        for (int c0 = 0; c0 < NCH; c0 += BATCH) {
            uint4 t[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i)
                if (c0 + i < NCH && c0 + i < nch) t[i] = ld_ro_v4(pro.gamma + off(c0 + i));
#pragma unroll
            for (int i = 0; i < BATCH; ++i)
                if (c0 + i < NCH && c0 + i < nch) xr[c0 + i] = norm8(xr[c0 + i], r, r32, t[i]);
        }
    }
}

// 16-byte chunks of x per thread held in registers: rows up to kRegChunks x 8 x
// kPrepThreads elements (ternary; OneBit: whole 32-element groups, a quarter
// as many) are prepared from registers in one read.
constexpr int kRegChunks = 10;

// Activations of layer L into buffer act ([cols][astride] bytes) for a single
// token.  K <= kRegK: x is read once into registers (every load in flight at
// once), then its absmax is reduced and it is quantised from registers
// (OneBit re-reads g, a parameter, for the products).  Longer rows: two passes
// over x (the second from L1 or L2).  `cg`: x is another CTA's output, read
// through L2.
template <int FORM, bool FUSED>
__device__ void prep_layer(int K, const uint16_t* x, const uint16_t* gvec, bool cg, const Prologue& pro,
                           uint8_t* act, int astride, TokStats* ts, int b, int et) {
    const int pw = et >> 5, lane = et & 31;
    auto ld = [&](const uint16_t* p) { return cg ? ld_cg_v4(p) : tc::ld_v4(p); };
    const bool in_regs = FORM == 0 ? K <= 8 * kRegChunks * kPrepThreads
                                   : K <= 32 * (kRegChunks / 4) * kPrepThreads;
    uint4 xr[kRegChunks];
    float amax;
    if constexpr (FORM == 0) {
        // chunk c of thread et covers elements 8 (et + c P) .. +8, P = kPrepThreads
        uint32_t mx = 0;
        // chunks of this thread: c < nc (8 (et + c P) < K)
        const int nc = (K / 8 - et + kPrepThreads - 1) / kPrepThreads;
        if (in_regs) {
#pragma unroll
            for (int c = 0; c < kRegChunks; ++c) {
                if (c >= nc) break;
                xr[c] = ld(x + 8 * (et + c * kPrepThreads));
            }
            if constexpr (FUSED)
                apply_prologue<kRegChunks, 4>(xr, nc, [&](int c) { return 8 * (et + c * kPrepThreads); }, K,
                                              pro, ts, et);
#pragma unroll
            for (int c = 0; c < kRegChunks; ++c) {
                if (c >= nc) break;
                mx = max(mx, absmax_bits_t(xr[c]));
            }
        } else {
#pragma unroll 4
            for (int c = et; c < K / 8; c += kPrepThreads) mx = max(mx, absmax_bits_t(ld(x + 8 * c)));
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) ts->red[0][pw] = mx;
        bar_prep();
        uint32_t m = 0;
#pragma unroll
        for (int w = 0; w < kPrepWarps; ++w) m = max(m, ts->red[0][w]);
        amax = hbits(m);
        const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
        int sum = 0;
        if (in_regs) {
            // a 16-element group is two 8-element chunks: chunk pairs (c, c+1)
            // of a thread cover elements 8 (et + c P) and 8 (et + (c+1) P), not
            // adjacent, so quantise 8-element halves into the permuted group:
            // byte 4j+b of the group of element e holds element 4b+j
#pragma unroll
            for (int c = 0; c < kRegChunks; ++c) {
                if (c >= nc) break;
                const int e = 8 * (et + c * kPrepThreads);
                sum += quant_half_group_t(xr[c], inv, act + (e & ~15), (e >> 3) & 1);
            }
        } else {
#pragma unroll 2
            for (int gi = et; gi < K / 16; gi += kPrepThreads)
                sum += quant_group_t(ld(x + 16 * gi), ld(x + 16 * gi + 8), inv, act + 16 * gi);
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) ts->redi[0][pw] = sum;
        bar_prep();
        if (et == 0) {
            int s = 0;
#pragma unroll
            for (int w = 0; w < kPrepWarps; ++w) s += ts->redi[0][w];
            ts->qsum[b] = s;
            ts->scale[b] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
        }
    } else {
        // chunk c of thread et: the 32-element group et + c P, as 4 x 8 halves
        // (OneBit rows are at most kRegK / 4 groups per thread in registers)
        constexpr int kG = kRegChunks / 4;
        float mx = 0.f;
        const int ng = (K / 32 - et + kPrepThreads - 1) / kPrepThreads;   // groups of this thread
        if (in_regs) {
#pragma unroll
            for (int c = 0; c < kG; ++c) {
                if (c >= ng) break;
                const int e = 32 * (et + c * kPrepThreads);
#pragma unroll
                for (int v = 0; v < 4; ++v) xr[4 * c + v] = ld(x + e + 8 * v);
            }
            if constexpr (FUSED)
                apply_prologue<kRegChunks, 2>(xr, 4 * ng,
                           [&](int c) { return 32 * (et + (c >> 2) * kPrepThreads) + 8 * (c & 3); }, K,
                           pro, ts, et);
#pragma unroll
            for (int c = 0; c < kG; ++c) {
                if (c >= ng) break;
                const int e = 32 * (et + c * kPrepThreads);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    mx = fmaxf(mx, absmax_prod(xr[4 * c + v], ld_ro_v4(gvec + e + 8 * v)));
            }
        } else {
            for (int c = et; c < K / 8; c += kPrepThreads)
                mx = fmaxf(mx, absmax_prod(ld(x + 8 * c), ld_ro_v4(gvec + 8 * c)));
        }
        const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
        if (lane == 0) ts->red[0][pw] = mb;
        bar_prep();
        uint32_t m = 0;
#pragma unroll
        for (int w = 0; w < kPrepWarps; ++w) m = max(m, ts->red[0][w]);
        amax = __uint_as_float(m);
        const float inv = amax > 0.f ? __fdiv_rn(kImgMaxF, amax) : 0.f;
        int ls[3] = {0, 0, 0};
        auto group = [&](const uint4 (&xa)[4], int gi) {
            uint4 ga[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) ga[v] = ld_ro_v4(gvec + 32 * gi + 8 * v);
            int gs[3];
            quant_group_s(xa, ga, inv, act + 32 * gi, astride, gs);
            ls[0] += gs[0];
            ls[1] += gs[1];
            ls[2] += gs[2];
        };
        if (in_regs) {
#pragma unroll
            for (int c = 0; c < kG; ++c) {
                if (c >= ng) break;
                const uint4 xa[4] = {xr[4 * c], xr[4 * c + 1], xr[4 * c + 2], xr[4 * c + 3]};
                group(xa, et + c * kPrepThreads);
            }
        } else {
            for (int gi = et; gi < K / 32; gi += kPrepThreads) {
                uint4 xa[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) xa[v] = ld(x + 32 * gi + 8 * v);
                group(xa, gi);
            }
        }
#pragma unroll
        for (int l = 0; l < 3; ++l) {
            const int v = __reduce_add_sync(0xffffffffu, ls[l]);
            if (lane == 0) ts->redi[l][pw] = v;
        }
        bar_prep();
        if (et == 0) {
            long long s = 0;
#pragma unroll
            for (int w = 0; w < kPrepWarps; ++w)
                s += 65536ll * ts->redi[0][w] + 256ll * ts->redi[1][w] + (long long)ts->redi[2][w];
            ts->xsum[b] = s;
            ts->scale[b] = amax > 0.f ? __fdiv_rn(amax, kImgMaxF) : 0.f;
        }
    }
}

// FUSED: the chain has a layer with a prologue or a SwiGLU buffer.  Chains
// without one run an instantiation that holds none of that code (its mere
// presence cost the plain chain 5-15 % in register allocation and scheduling).
template <int FORM, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1) chain_kernel(const ChainParams p) {
    using F = DF<FORM>;
    constexpr int COLS = F::kCPT;          // activation columns of the single token
    constexpr int CH = 4;                  // independent accumulator chains
    constexpr bool kMasked = FORM == 0;    // ternary: in-place masked 2-bit unpack
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, G = gridDim.x, S = p.S, n = p.n;
    const uint32_t sb = tc::smem_u32(smem);
    const int NB = p.nbuf;
    int* part = reinterpret_cast<int*>(smem + p.off_part);          // [NB][kMaxTiles*16][COLS]
    TokStats* ts = reinterpret_cast<TokStats*>(smem + p.off_tok);
    const uint32_t bar_full = sb + p.off_bar;                         // [S] stage landed
    const uint32_t bar_empty = bar_full + 8 * S;                      // [S] 8 warps done with it
    const uint32_t bar_act = bar_empty + 8 * S;                       // [NB] activations ready
    const uint32_t bar_mma = bar_act + 8 * kMaxBufs;                  // [NB] layer contracted
    const int kPartInts = NB * kMaxTiles * 16 * COLS;

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            tc::mbar_init(bar_full + 8 * i, 1);
            tc::mbar_init(bar_empty + 8 * i, kMmaWarps);
        }
        for (int i = 0; i < NB; ++i) {
            tc::mbar_init(bar_act + 8 * i, 1);
            tc::mbar_init(bar_mma + 8 * i, kMmaWarps);
        }
        tc::mbar_fence_init();
    }
    for (int i = tid; i < kPartInts; i += kThreads) part[i] = 0;
    LayerInfo* tab = reinterpret_cast<LayerInfo*>(smem + p.off_tab);
    for (int i = tid; i < 2 * n; i += kThreads)
        reinterpret_cast<uint4*>(tab)[i] = reinterpret_cast<const uint4*>(p.info)[i];
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane != 0) return;
        // Stages of this CTA in order: (layer j, tile k, chunk ch).  (A second
        // cursor that brought the stages 16 ahead of the ring into L2 with TMA
        // prefetches measured slower: 0.57 -> 0.64 ms on the 7B-shaped stack.)
        struct Cursor {
            int j, k, ch, first, T;
        };
        auto enter = [&](Cursor& q) {   // first stage at or after layer q.j
            for (; q.j < n; ++q.j) {
                q.first = first_tile(tab[q.j], c, G);
                q.T = tiles_of(tab[q.j], q.first, G);
                if (q.T > 0) break;
            }
            q.k = q.ch = 0;
        };
        auto next = [&](Cursor& q) {
            if (++q.ch < tab[q.j].nch) return;
            q.ch = 0;
            if (++q.k < q.T) return;
            ++q.j;
            enter(q);
        };
        Cursor ld{0, 0, 0, 0, 0};
        enter(ld);
        int u = 0, jprev = -1;
        bool ok = true;
        while (ld.j < n) {
            const int j = ld.j;
            const LayerInfo& L = tab[j];
            if (j != jprev) {
                jprev = j;
                if (j + 1 < n) {
                    tc::prefetch_tmap(&p.layers[j + 1].tm_main);
                    if (tab[j + 1].flags & kInfoRagged) tc::prefetch_tmap(&p.layers[j + 1].tm_tail);
                }
                // a given input two layers ahead: into L2 before its activations are prepared
                if (j + 2 < n && tab[j + 2].src < 0 && !(tab[j + 2].flags & kInfoReuse))
                    tc::bulk_prefetch_l2(tab[j + 2].x, (uint32_t)(32 * tab[j + 2].k16));
            }
            const int slot = u % S;
            if (u >= S) {
                ok = tc::mbar_wait(bar_empty + 8 * slot, ((u / S) - 1) & 1, p.flags, p.wait_ns);
                if (!ok) break;
            }
            const int steps = L.steps, nfull = L.nfull, bsteps = L.bsteps;
            const bool ragged = (L.flags & kInfoRagged) != 0;
            const int row0 = (ld.first + ld.k * G) * 16;
            const int s0 = ld.ch * bsteps, s1 = min(s0 + bsteps, steps);
            uint32_t bytes = s0 < nfull ? (uint32_t)bsteps * 1024u : 0u;
            if (ragged && s1 == steps) bytes += 16u * (uint32_t)L.tail;
            const uint32_t dst = sb + slot * kSlotBytes, bar = bar_full + 8 * slot;
            tc::mbar_arrive_expect_tx(bar, bytes);
            if (s0 < nfull) tc::tma_load_3d(dst, &p.layers[j].tm_main, 0, row0, s0, bar);
            if (ragged && s1 == steps)
                tc::tma_load_2d(dst + bsteps * 1024, &p.layers[j].tm_tail, 0, row0, bar);
            ++u;
            next(ld);
        }
        // Every copy requested lands before the CTA can exit (on the normal
        // path the contraction has consumed them and these waits return at once).
        for (int v = (u > S ? u - S : 0); v < u; ++v)
            tc::mbar_wait(bar_full + 8 * (v % S), (v / S) & 1, p.flags, kWaitNs);
        return;
    }

    if (warp <= kMmaWarps) {
        // --------------------------------------------------- contraction --
        // A stage holds at most kStageSteps = 2 x kMmaWarps steps: warp mw owns
        // steps s0 + mw and s0 + mw + kMmaWarps of every stage.
        const int mw = warp - 1;
        const int g8 = lane >> 2, t = lane & 3;
        const uint8_t* act_base = smem + p.off_act;
        int slot = 0;
        uint32_t phase = 0;
        int b = 0;            // activation buffer of layer j (= j % NB), its phase bphase
        uint32_t bphase = 0;
        for (int j = 0; j < n; ++j) {
            const LayerInfo L = tab[j];
            const int first = first_tile(L, c, G), T = tiles_of(L, first, G);
            const int steps = L.steps, nfull = L.nfull, bsteps = L.bsteps, nch = L.nch;
            const int tail = L.tail;
            if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_act + 8 * b, bphase, p.flags, p.wait_ns)))
                return;
            // B operand source of this lane's column (token limb row); lanes of the
            // unused columns read row 0
            const uint8_t* bsrc = act_base + b * COLS * p.astride + (g8 < COLS ? g8 : 0) * p.astride +
                                  t * F::kChunkK;
            int* pb = part + b * kMaxTiles * 16 * COLS;
            // This warp's (at most) two steps of a stage.  No lane is masked:
            // columns >= COLS of the MMA are never read, so lanes of other columns
            // may load any activation bytes (row 0); and the activation rows are
            // zero past K to a whole step, so the weight bytes a partial last step
            // reads past its row end meet zeros.  A layer of one stage per tile
            // uses the same activation words for every tile: they are loaded once.
            constexpr int BW_ = F::kRegs * 4;       // activation words per step and lane
            uint32_t bw[2][BW_];
            auto load_b = [&](int s0, int s1) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int s = s0 + mw + kMmaWarps * i;
                    if (s < s1) {
                        const uint8_t* src = bsrc + s * F::kStepK;
#pragma unroll
                        for (int q = 0; q < BW_ / 4; ++q) {
                            const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * q);
                            bw[i][4 * q + 0] = v.x;
                            bw[i][4 * q + 1] = v.y;
                            bw[i][4 * q + 2] = v.z;
                            bw[i][4 * q + 3] = v.w;
                        }
                    }
                }
            };
            if (nch == 1 && T > 0) load_b(0, steps);
            for (int k = 0; k < T; ++k) {
                int acc[CH][4];
#pragma unroll
                for (int cc = 0; cc < CH; ++cc) acc[cc][0] = acc[cc][1] = acc[cc][2] = acc[cc][3] = 0;
                for (int ch = 0; ch < nch; ++ch) {
                    const int s0 = ch * bsteps, s1 = min(s0 + bsteps, steps);
                    const bool has0 = s0 + mw < s1, has1 = s0 + mw + kMmaWarps < s1;
                    if (nch > 1) load_b(s0, s1);
                    if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_full + 8 * slot, phase, p.flags, p.wait_ns)))
                        return;
                    const uint8_t* slot_p = smem + slot * kSlotBytes;
                    uint4 a0[2], a1[2];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int s = s0 + mw + kMmaWarps * i;
                        if (i == 0 ? has0 : has1) {
                            if (s < nfull) {   // whole step: [step][row][64 B]
                                const uint8_t* w0 = slot_p + (s - s0) * 1024 + 64 * g8 + 16 * t;
                                a0[i] = *reinterpret_cast<const uint4*>(w0);
                                a1[i] = *reinterpret_cast<const uint4*>(w0 + 512);
                            } else {           // partial last step: tail box [row][tail B]
                                const uint8_t* w0 = slot_p + bsteps * 1024 + tail * g8 + 16 * t;
                                a0[i] = *reinterpret_cast<const uint4*>(w0);
                                a1[i] = *reinterpret_cast<const uint4*>(w0 + 8 * tail);
                            }
                        }
                    }
                    // the stage's bytes are in registers: release the slot to the producer
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar_empty + 8 * slot);
                    if (++slot == S) {
                        slot = 0;
                        phase ^= 1u;
                    }
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (!(i == 0 ? has0 : has1)) continue;
                        const uint32_t r0[4] = {a0[i].x, a0[i].y, a0[i].z, a0[i].w};
                        const uint32_t r1[4] = {a1[i].x, a1[i].y, a1[i].z, a1[i].w};
                        if constexpr (kMasked) {
                            // field jj of every byte masked in place (code * 4^jj) against
                            // activation word jj; the two words of a pair share jj, so chain
                            // jj holds 4^jj times its sum
#pragma unroll
                            for (int op = 0; op < 4; op += 2)
#pragma unroll
                                for (int jj = 0; jj < 4; ++jj) {
                                    const uint32_t m = 0x03030303u << (2 * jj);
                                    mma_u8s8_16832(acc[jj], r0[op] & m, r1[op] & m, r0[op + 1] & m,
                                                   r1[op + 1] & m, bw[i][4 * op + jj], bw[i][4 * op + 4 + jj]);
                                }
                        } else {
#pragma unroll
                            for (int om = 0; om < 4; ++om) {
                                uint32_t u0r[F::kRegs], u1r[F::kRegs];
#pragma unroll
                                for (int jj = 0; jj < F::kRegs; ++jj) {
                                    u0r[jj] = (r0[om] >> (F::kShift * jj)) & F::kMask;
                                    u1r[jj] = (r1[om] >> (F::kShift * jj)) & F::kMask;
                                }
#pragma unroll
                                for (int jj = 0; jj < F::kRegs; jj += 2)
                                    mma_u8s8_16832(acc[om % CH], u0r[jj], u1r[jj], u0r[jj + 1],
                                                   u1r[jj + 1], bw[i][om * F::kRegs + jj],
                                                   bw[i][om * F::kRegs + jj + 1]);
                            }
                        }
                    }
                }
                // tile done: fold the chains and add this warp's share into the tile's rows
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int v = 0;
#pragma unroll
                    for (int cc = 0; cc < CH; ++cc) v += kMasked ? (acc[cc][e] >> (2 * cc)) : acc[cc][e];
                    const int row = g8 + 8 * (e >> 1), col = 2 * t + (e & 1);
                    if (col < COLS) atomicAdd(pb + (k * 16 + row) * COLS + col, v);
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar_mma + 8 * b);
            if (++b == NB) {
                b = 0;
                bphase ^= 1u;
            }
        }
        return;
    }

    // ---------------------------------------- activations and epilogue --
    const int et = tid - kFirstPrepWarp * 32;     // 0 .. kPrepThreads-1
    uint8_t* act_base = smem + p.off_act;
    bool ok = true;
    bool prev_prepared = false;   // layer next_prep-1's activations are in its buffer
    int next_prep = 0, next_epi = 0;
    while (next_epi < n && ok) {
        const bool can_prep = next_prep < n && next_prep < next_epi + NB &&
                              tab[next_prep].src < next_epi && tab[next_prep].src2 < next_epi;
        if (can_prep) {
            // ---- activations of layer j into buffer j % NB
            const int j = next_prep++;
            const LayerInfo L = tab[j];
            const int K = 16 * L.k16;
            const int b = j % NB, bprev = (j + NB - 1) % NB;
            const int T = tiles_of(L, first_tile(L, c, G), G);
            uint8_t* act = act_base + b * COLS * p.astride;
            const bool prepare = T > 0;
            if (prepare) {
                if ((L.flags & kInfoReuse) && prev_prepared) {
                    // same input as layer j-1: copy its prepared activations
                    const uint8_t* prev = act_base + bprev * COLS * p.astride;
                    for (int r = 0; r < COLS; ++r)
                        for (int i = et; i < K / 16; i += kPrepThreads)
                            *reinterpret_cast<uint4*>(act + r * p.astride + 16 * i) =
                                *reinterpret_cast<const uint4*>(prev + r * p.astride + 16 * i);
                    if (et == 0) {
                        ts->scale[b] = ts->scale[bprev];
                        ts->qsum[b] = ts->qsum[bprev];
                        ts->xsum[b] = ts->xsum[bprev];
                    }
                } else {
                    // the input, g and prologue pointers, loaded before the dependency wait
                    const uint16_t* x = (L.src >= 0 && !(L.flags & kInfoXbuf)) ? tab[L.src].y : L.x;
                    const uint16_t* gvec = FORM == 1 ? p.layers[j].g : nullptr;
                    Prologue pro;
                    pro.x2 = L.src2 >= 0 ? tab[L.src2].y : nullptr;
                    pro.gamma = (L.flags & kInfoNorm) ? p.layers[j].norm_w : nullptr;
                    pro.eps = (double)p.layers[j].norm_eps;
                    // the weight is read after the row's sum of squares: fetch it
                    // while the producing layer finishes
                    if (FUSED && pro.gamma) prefetch_row_l1(pro.gamma, K, et, kPrepThreads);
                    if (L.src >= 0) {
                        // wait until every CTA has finished the producing layer(s)
                        bool got = true;
                        if (et == 0) {
                            for (int dsrc = 0; dsrc < 2 && got; ++dsrc) {
                                const int sj = dsrc == 0 ? L.src : L.src2;
                                if (sj < 0) continue;
                                const unsigned int* d = p.done + sj;
                                if (ld_acquire_u32(d) >= (unsigned)G) continue;
                                const uint64_t t0 = tc::globaltimer_ns();
                                while (ld_acquire_u32(d) < (unsigned)G) {
                                    if (tc::globaltimer_ns() - t0 > p.wait_ns) {
                                        atomicOr(p.flags, kFlagTimeout);
                                        got = false;
                                        break;
                                    }
                                    __nanosleep(32);
                                }
                            }
                        }
                        if (!tc::bar_and(kBarPrep, kPrepThreads, got)) {
                            ok = false;
                            break;
                        }
                    }
                    prep_layer<FORM, FUSED>(K, x, gvec, L.src >= 0, pro, act, p.astride, ts, b, et);
                }
                // zeros from K to a whole step in every row (a partial last step's
                // lanes past the row end multiply them)
                const int kp = (K + F::kStepK - 1) / F::kStepK * F::kStepK;
                for (int r = 0; r < COLS; ++r)
                    for (int i = K + 16 * et; i < kp; i += 16 * kPrepThreads)
                        *reinterpret_cast<uint4*>(act + r * p.astride + i) = make_uint4(0, 0, 0, 0);
            }
            prev_prepared = prepare;
            bar_prep();   // activations and token scalars written (and the scratch reads done)
            if (et == 0) tc::mbar_arrive(bar_act + 8 * b);
        } else {
            // ---- epilogue of layer j from buffer j % NB
            const int j = next_epi++;
            const LayerInfo L = tab[j];
            const int b = j % NB;
            const int first = first_tile(L, c, G), T = tiles_of(L, first, G);
            // the output pointers, loaded before the wait for the contraction
            uint16_t* y = L.y;
            int32_t* acc_out = FORM == 0 ? p.layers[j].acc_out : nullptr;
            const float w_scale = p.layers[j].w_scale;
            const uint16_t* h = FORM == 1 ? p.layers[j].h : nullptr;
            uint16_t* swi_out = FUSED ? p.layers[j].swi_out : nullptr;
            const uint16_t* yq = swi_out ? tab[p.layers[j].swi_q].y : nullptr;
            const bool self_a = p.layers[j].swi_self_a != 0;
            // one thread waits (asleep) for the contraction; the others in the barrier
            bool got = true;
            if (et == 0) got = tc::mbar_wait(bar_mma + 8 * b, (uint32_t)((j / NB) & 1), p.flags, p.wait_ns);
            if (!tc::bar_and(kBarPrep, kPrepThreads, got)) {
                ok = false;
                break;
            }
            int* pb = part + b * kMaxTiles * 16 * COLS;
            const float sc = ts->scale[b];
            for (int o = et; o < T * 16; o += kPrepThreads) {
                const int k = o >> 4, r = o & 15;
                const int nrow = (first + k * G) * 16 + r;
                uint32_t yb;
                if constexpr (FORM == 0) {
                    const int a = pb[o] - ts->qsum[b];
                    pb[o] = 0;
                    yb = __half_as_ushort(__float2half_rn(__fmul_rn(__fmul_rn((float)a, sc), w_scale)));
                    if (acc_out) acc_out[nrow] = a;
                } else {
                    const long long Z = limb_combine(pb[3 * o], pb[3 * o + 1], pb[3 * o + 2], ts->xsum[b]);
                    pb[3 * o] = pb[3 * o + 1] = pb[3 * o + 2] = 0;
                    const float z = __fmul_rn(sc, (float)Z);
                    const float hv = __half2float(__ushort_as_half(h[nrow]));
                    yb = __half_as_ushort(__float2half_rn(__fmul_rn(z, hv)));
                }
                y[nrow] = (uint16_t)yb;
                if (FUSED && swi_out) {
                    // this thread wrote y_q[nrow] in layer swi_q's epilogue
                    const uint32_t other = yq[nrow];
                    swi_out[nrow] = (uint16_t)(self_a ? swiglu1(yb, other) : swiglu1(other, yb));
                }
            }
            bar_prep();   // every output of this CTA written, partials cleared
            if ((L.flags & kInfoHasDep) && et == 0) {
                __threadfence();
                atomicAdd(p.done + j, 1u);
            }
        }
    }
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared-memory layout of a launch: ring [S][kSlotBytes] | activations
// [NB][COLS][astride] | partial sums [NB][kMaxTiles*16][COLS] int32 | token
// scalars | barriers | layer table [n].  S (ring slots) is the largest that
// fits, then NB (activation buffers, 2..4).
struct ChainSmem {
    int S, NB, astride, off_act, off_part, off_tok, off_bar, off_tab, total;
};

bool chain_smem(int form, int kmax, int n, ChainSmem& m, int s_req = 0, bool buffers_first = false) {
    const int cols = form == 0 ? 1 : 3;
    // rows padded to a whole step (256 / 512 k), +16 bytes between rows
    m.astride = (kmax + 511) / 512 * 512 + 16;
    const int tok = (int)round_up(sizeof(TokStats), 16);
    auto layout = [&](int NB, int S) {
        int off = S * kSlotBytes;
        m.off_act = off;
        off += (int)round_up((size_t)NB * cols * m.astride, 16);
        m.off_part = off;
        off += NB * kMaxTiles * 16 * cols * 4;
        m.off_tok = off;
        off += tok;
        m.off_bar = off;
        off += 8 * (2 * S + 2 * kMaxBufs);
        off = (int)round_up((size_t)off, 16);
        m.off_tab = off;
        off += (int)sizeof(LayerInfo) * n;
        m.S = S;
        m.NB = NB;
        m.total = off;
        return off <= kDecodeMaxSmem;
    };
    // s_req > 0: that many slots (with the most buffers that fit).  Otherwise
    // the most ring slots first (bytes in flight, which also carry the next
    // layers' weights across a dependency), then the most activation buffers;
    // or, with buffers_first, the most buffers first: a chain whose layers
    // mostly read given inputs can prepare up to four layers ahead.
    if (s_req > 0) {
        for (int NB = kMaxBufs; NB >= 2; --NB)
            if (layout(NB, s_req)) return true;
        return false;
    }
    if (buffers_first) {
        for (int NB = kMaxBufs; NB >= 2; --NB)
            for (int S = kMaxSlots; S >= 3; --S)
                if (layout(NB, S)) return true;
        return false;
    }
    for (int S = kMaxSlots; S >= 3; --S)
        for (int NB = kMaxBufs; NB >= 2; --NB)
            if (layout(NB, S)) return true;
    return false;
}

template <int FORM, bool FUSED>
cudaError_t launch_chain(const ChainParams& p, int smem, cudaStream_t s) {
    static KernelAttrs kattrs;
    if (cudaError_t e = kattrs.ensure(chain_kernel<FORM, FUSED>, kDecodeMaxSmem)) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(device_sm_count());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    // every CTA must be resident at once: layers wait on other CTAs' results
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeCooperative;
    attrs[0].val.cooperative = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, chain_kernel<FORM, FUSED>, p);
}

}  // namespace

// Chain buffer: descriptors [n] | layer table [n] | completion counters [n].
size_t chain_info_offset(int n) { return round_up((size_t)n * sizeof(ChainLayer), 256); }
size_t chain_done_offset(int n) { return chain_info_offset(n) + round_up((size_t)n * sizeof(LayerInfo), 256); }
size_t chain_bytes(int n_layers) { return chain_done_offset(n_layers) + round_up((size_t)n_layers * 4, 256); }

int chain_max_k(int form) { return form == 0 ? 32768 : 16384; }
int chain_max_fused_k(int form) {
    return form == 0 ? 8 * kRegChunks * kPrepThreads : 32 * (kRegChunks / 4) * kPrepThreads;
}

bl_status chain_build(int form, const bl_chain_layer* layers, int n, void* chain, size_t bytes,
                      bl_chain_plan* plan, cudaStream_t s) {
    const int G = device_sm_count();
    if (G <= 0) return BL_ERR_CUDA;
    std::vector<ChainLayer> host((size_t)n);
    std::vector<LayerInfo> info((size_t)n);
    int kmax = 0;
    bool fused = false;
    long long tiles_before = 0;
    for (int j = 0; j < n; ++j) {
        const bl_chain_layer& in = layers[j];
        ChainLayer& L = host[(size_t)j];
        std::memset(&L, 0, sizeof(L));
        L.K = in.K;
        L.N = in.N;
        L.src = in.src;
        L.src2 = in.src2;
        L.norm_w = in.norm_w;
        L.norm_eps = in.norm_eps;
        L.x = in.x;
        L.w = in.w;
        L.y = in.y;
        L.acc_out = in.acc_out;
        L.g = in.g;
        L.h = in.h;
        L.w_scale = in.w_scale;
        L.ntile = in.N / 16;
        L.rot = (int)(tiles_before % G);
        tiles_before += L.ntile;
        if (in.src >= 0) host[(size_t)in.src].has_dep = 1;
        if (in.src2 >= 0) host[(size_t)in.src2].has_dep = 1;
        L.swi_q = -1;
        if (in.src2 >= 0 || in.norm_w) fused = true;
        if (in.src2 >= 0 && in.swiglu_buf) {
            // evaluate the SwiGLU in the epilogue of the later of the two sources,
            // whose tiles are then dealt like the earlier one's; this layer reads
            // the finished input from swiglu_buf (unless that layer already
            // evaluates another SwiGLU)
            const int pi = in.src > in.src2 ? in.src : in.src2;
            const int qi = in.src > in.src2 ? in.src2 : in.src;
            ChainLayer& P = host[(size_t)pi];
            const int self_a = pi == in.src;
            if (!P.swi_out || (P.swi_out == in.swiglu_buf && P.swi_q == qi && P.swi_self_a == self_a)) {
                P.swi_out = in.swiglu_buf;
                P.swi_q = qi;
                P.swi_self_a = self_a;
                P.rot = host[(size_t)qi].rot;
                L.src = pi;
                L.src2 = -1;
                L.x = in.swiglu_buf;
                L.xbuf = 1;
            }
        }
        // the same prepared input as the layer before: same source(s), same
        // prologue, same g (OneBit)
        if (j > 0 && in.K == layers[j - 1].K && in.src == layers[j - 1].src &&
            in.src2 == layers[j - 1].src2 && (in.src >= 0 || in.x == layers[j - 1].x) &&
            in.norm_w == layers[j - 1].norm_w && (!in.norm_w || in.norm_eps == layers[j - 1].norm_eps) &&
            (form == 0 || in.g == layers[j - 1].g))
            L.reuse = 1;
        // k-steps of 64 packed bytes per row; stages of at most 16 steps, a
        // multiple of 16 when a row takes several (a warp owns the same steps
        // in every stage)
        const int wbytes = form == 0 ? in.K / 4 : in.K / 8;   // packed bytes per row
        L.nfull = wbytes / 64;
        L.tail = wbytes % 64;
        L.ragged = L.tail != 0;
        L.steps = L.nfull + L.ragged;
        L.nch = (L.steps + kStageSteps - 1) / kStageSteps;
        L.bsteps = L.nch > 1 ? kStageSteps : L.steps;
        if (L.nfull > 0) {
            const cuuint64_t dims[3] = {64, (cuuint64_t)in.N, (cuuint64_t)L.nfull};
            const cuuint64_t strides[2] = {(cuuint64_t)wbytes, 64};
            const cuuint32_t box[3] = {64, 16, (cuuint32_t)L.bsteps};
            if (!encode_u8_map(&L.tm_main, in.w, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
                return BL_ERR_CUDA;
        }
        if (L.ragged) {
            const cuuint64_t dims[2] = {(cuuint64_t)L.tail, (cuuint64_t)in.N};
            const cuuint64_t strides[1] = {(cuuint64_t)wbytes};
            const cuuint32_t box[2] = {(cuuint32_t)L.tail, 16};
            const uint8_t* tailp = reinterpret_cast<const uint8_t*>(in.w) + 64 * (size_t)L.nfull;
            if (!encode_u8_map(&L.tm_tail, tailp, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
                return BL_ERR_CUDA;
        }
        if (in.K > kmax) kmax = in.K;
        if (L.ntile > kMaxTiles * G) return BL_ERR_SHAPE;
    }
    for (int j = 0; j < n; ++j) {
        const ChainLayer& L = host[(size_t)j];
        LayerInfo& I = info[(size_t)j];
        I.ntile = (uint16_t)L.ntile;
        I.rot = (uint16_t)L.rot;
        I.k16 = (uint16_t)(L.K / 16);
        I.src = (int16_t)L.src;
        I.steps = (uint8_t)L.steps;
        I.nfull = (uint8_t)L.nfull;
        I.tail = (uint8_t)L.tail;
        I.bsteps = (uint8_t)L.bsteps;
        I.nch = (uint8_t)L.nch;
        I.flags = (uint8_t)((L.ragged ? kInfoRagged : 0) | (L.has_dep ? kInfoHasDep : 0) |
                            (L.reuse ? kInfoReuse : 0) | (L.norm_w ? kInfoNorm : 0) |
                            (L.xbuf ? kInfoXbuf : 0));
        I.src2 = (int16_t)L.src2;
        I.x = (L.src < 0 || L.xbuf) ? L.x : nullptr;
        I.y = L.y;
    }
    ChainSmem m;
    // layers reading a given input (no dependency) can be prepared far ahead
    int given = 0;
    for (int j = 0; j < n; ++j) given += layers[j].src < 0;
    if (!chain_smem(form, kmax, n, m, 0, 2 * given > n)) return BL_ERR_SHAPE;
    if (bytes < chain_bytes(n)) return BL_ERR_WORKSPACE;
    char* cb = static_cast<char*>(chain);
    if (cudaMemcpyAsync(cb, host.data(), (size_t)n * sizeof(ChainLayer), cudaMemcpyHostToDevice,
                        s) != cudaSuccess ||
        cudaMemcpyAsync(cb + chain_info_offset(n), info.data(), (size_t)n * sizeof(LayerInfo),
                        cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return BL_ERR_CUDA;
    plan->form = form;
    plan->fused = fused ? 1 : 0;
    plan->n_layers = n;
    plan->sm_count = G;
    plan->kmax = kmax;
    plan->slots = m.S;
    plan->smem_bytes = m.total;
    return BL_OK;
}

bl_status chain_run(const bl_chain_plan* plan, const void* chain, unsigned int* flags,
                    cudaStream_t s) {
    ChainSmem m;
    if (plan->slots < 3 || plan->slots > kMaxSlots ||
        !chain_smem(plan->form, plan->kmax, plan->n_layers, m, plan->slots) || m.S != plan->slots ||
        m.total != plan->smem_bytes)
        return BL_ERR_SHAPE;
    if (device_sm_count() != plan->sm_count) return BL_ERR_SHAPE;
    const int n = plan->n_layers;
    ChainParams p;
    char* cb = static_cast<char*>(const_cast<void*>(chain));
    p.layers = reinterpret_cast<const ChainLayer*>(cb);
    p.info = reinterpret_cast<const LayerInfo*>(cb + chain_info_offset(n));
    p.n = n;
    p.done = reinterpret_cast<unsigned int*>(cb + chain_done_offset(n));
    p.flags = flags;
    p.S = m.S;
    p.nbuf = m.NB;
    p.astride = m.astride;
    p.off_act = m.off_act;
    p.off_part = m.off_part;
    p.off_tok = m.off_tok;
    p.off_bar = m.off_bar;
    p.off_tab = m.off_tab;
    p.wait_ns = kWaitNs;
    // the completion counters start at zero on every run
    if (cudaMemsetAsync(p.done, 0, (size_t)n * 4, s) != cudaSuccess) return BL_ERR_CUDA;
    const cudaError_t e =
        plan->form == 0 ? (plan->fused ? launch_chain<0, true>(p, m.total, s) : launch_chain<0, false>(p, m.total, s))
                        : (plan->fused ? launch_chain<1, true>(p, m.total, s) : launch_chain<1, false>(p, m.total, s));
    return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

}  // namespace bl
