// kernels.h -- internal launchers behind the C ABI (host side, no validation:
// the ABI layer in api.cu checks shapes, pointers and workspace first).
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "bitlinear.h"

namespace bl {

// Packers (pack.cu).  Each ORs a nonzero value into *err_flag (device) when it
// meets an input value the format cannot hold.
cudaError_t launch_pack_ternary(const int8_t* w, int N, int K, uint32_t* w2,
                                unsigned int* err_flag, cudaStream_t s);
cudaError_t launch_pack_sign(const uint16_t* w, int N, int K, uint32_t* s1,
                             unsigned int* err_flag, cudaStream_t s);

// Activation preparation (quant.cu).
//   plain   : q [M][K] in natural k order, scale [M]          (bl_quant_act)
//   ternary : q [M][K] in the decode kernel's permuted order, scale, row sum
//   onebit  : 23-bit fixed-point image of x*g split into three int8 limb planes
//             [M][3][K] (permuted), fixed-point step [M], sum of the image [M] (int64)
cudaError_t launch_quant_plain(const uint16_t* x, int M, int K, int8_t* q, float* scale,
                               cudaStream_t s);
// The ternary and onebit preparations also zero `n_zero` words at `zero` (the
// prefill kernel's arrival counters) once the previous kernel has finished.
cudaError_t launch_quant_ternary_perm(const uint16_t* x, int M, int K, int8_t* qp,
                                      float* scale, int32_t* qsum, cudaStream_t s,
                                      unsigned int* zero = nullptr, int n_zero = 0);
cudaError_t launch_prep_onebit(const uint16_t* x, const uint16_t* g, int M, int K,
                               int8_t* planes, float* step, long long* tsum, cudaStream_t s,
                               unsigned int* zero = nullptr, int n_zero = 0);

// Decode-shaped (small M) packed-weight kernels on warp-level int8 MMA (skinny.cu).
cudaError_t launch_ternary_skinny(const uint32_t* w2, const int8_t* qp, const float* scale,
                                  const int32_t* qsum, int M, int K, int N, float w_scale,
                                  uint16_t* y, int32_t* acc_out, cudaStream_t s);
// OneBit launchers take an optional zf: an fp32 [M][N] copy of the output
// (z (.) h) before its fp16 rounding, for the two-plane binary layer.
cudaError_t launch_onebit_skinny(const uint32_t* s1, const int8_t* planes, const float* step,
                                 const long long* tsum, const uint16_t* h, int M, int K, int N,
                                 uint16_t* y, cudaStream_t s, float* zf = nullptr);

// Prefill-shaped (large M) GEMM on tcgen05 int8 tensor cores with TMEM
// accumulators (prefill.cu).  `flags` is the device condition word that bounded
// waits mark on timeout.
// When the tiles would leave SMs idle in the last round, the kernel shares
// that round's work out evenly in k-stages; that needs `split_ws` of
// prefill_split_bytes() bytes whose first n_counters uint32 are zero at launch
// (the activation preparation kernel zeroes them).  Without it (NULL or too
// small) every tile runs whole.
size_t prefill_split_bytes(int form, int M, int K, int N, int* n_counters);
// The same plan for an explicit SM count (host arithmetic only): activation
// rows per tile, ring stages per tile, tiles, tiles computed whole, tiles of
// the balanced round.
void prefill_plan_info(int form, int M, int K, int N, int sm_count, int plan[5]);
cudaError_t launch_ternary_prefill(const uint32_t* w2, const int8_t* qp, const float* scale,
                                   const int32_t* qsum, int M, int K, int N, float w_scale,
                                   uint16_t* y, int32_t* acc_out, unsigned int* flags,
                                   cudaStream_t s, void* split_ws = nullptr,
                                   size_t split_ws_bytes = 0);
cudaError_t launch_onebit_prefill(const uint32_t* s1, const int8_t* planes, const float* step,
                                  const long long* tsum, const uint16_t* h, int M, int K, int N,
                                  uint16_t* y, unsigned int* flags, cudaStream_t s,
                                  void* split_ws = nullptr, size_t split_ws_bytes = 0,
                                  float* zf = nullptr);

// Number of SMs of the current device (cached per device; 0 on error).
int device_sm_count();

// Largest dynamic shared memory of a CTA (227 KB on sm_100a).
constexpr int kDecodeMaxSmem = 227 * 1024;

// Device address of the condition word bounded waits mark (nullptr on error).
unsigned int* device_flags_address();

// The BitLinear forward behind bl_ternary_linear and bl_ternary_linear_noalloc
// (api.cu), with the ABI's argument checks already done.  The workspace holds
// at least ternary_act_bytes(M, K) bytes (the prepared activations, scales and
// row sums); the prefill kernel's balanced last round is used only when it
// also holds that round's scratch (bl_ternary_workspace_bytes).
size_t ternary_act_bytes(int M, int K);
// BL_FAULT_INJECT ("cuda" / "timeout"): the error every launching entry point
// returns after its argument checks, BL_OK when unset (api.cu).
bl_status fault_injected();
// The stall bl_debug_stall_next_launch asked for (its wait limit in ns), taken
// by the next streamed-decode or whole-tile tensor-core launch; 0 = none.
unsigned long long take_stall();
bl_status ternary_linear_on(const uint16_t* x, int M, int K, int N, const uint32_t* w2,
                            float w_scale, uint16_t* y, int32_t* acc_out, void* workspace,
                            size_t workspace_bytes, cudaStream_t s);

// Streamed decode (stream.cu): at most one 512-thread CTA per SM, each owning a
// contiguous range of 16-row tiles streamed through a shared-memory ring that
// is filled before the programmatic-dependent-launch wait.  prep = 0: the CTA
// prepares the activations from x; prep = 1: they come from the activation
// kernel.  stream_fits tells whether the shape has a plan.
bool stream_fits(int form, int M, int K, int N, int prep);
cudaError_t launch_ternary_stream(const uint16_t* x, const uint32_t* w2, int M, int K, int N,
                                  float w_scale, uint16_t* y, int32_t* acc_out, unsigned int* flags,
                                  cudaStream_t s);
cudaError_t launch_onebit_stream(const uint16_t* x, const uint16_t* g, const uint16_t* h,
                                 const uint32_t* s1, int M, int K, int N, uint16_t* y,
                                 unsigned int* flags, cudaStream_t s, float* zf = nullptr);
cudaError_t launch_ternary_stream_prepared(const int8_t* qp, const float* scale, const int32_t* qsum,
                                           const uint32_t* w2, int M, int K, int N, float w_scale,
                                           uint16_t* y, int32_t* acc_out, unsigned int* flags,
                                           cudaStream_t s);
cudaError_t launch_onebit_stream_prepared(const int8_t* planes, const float* step,
                                          const long long* tsum, const uint16_t* h,
                                          const uint32_t* s1, int M, int K, int N, uint16_t* y,
                                          unsigned int* flags, cudaStream_t s, float* zf = nullptr);

// Persistent single-token decode over a list of layers (chain.cu): device
// descriptors (tensor maps, tile plan) written by chain_build into the caller's
// `chain` buffer of chain_bytes(n) bytes, one cooperative launch per run.
size_t chain_bytes(int n_layers);
int chain_max_k(int form);
int chain_max_fused_k(int form);

// Two-plane binary layer (billm.cu): y = fp16(zf[:, :N] + zf[:, N:]) from the
// OneBit forward's fp32 outputs over the stacked planes, and the residual
// binarisation of a weight into those planes and scales.
cudaError_t launch_billm_combine(const float* zf, int M, int N, uint16_t* y, cudaStream_t s);
cudaError_t launch_billm_binarize(const float* W, int N, int K, uint32_t* b2, uint16_t* alpha,
                                  double* ao, double* ar, unsigned int* bad_flag, cudaStream_t s);

// SVID initialisation of a OneBit layer (svid.cu)
int svid_max_n();
size_t svid_workspace_bytes(int N, int K);
bl_status svid_run(const float* W, int N, int K, int max_iter, double tol, uint32_t* s1, uint16_t* g,
                   uint16_t* h, double* a, double* b, double* sigma, int* iters, void* workspace,
                   cudaStream_t s);   // longest row the RMSNorm / SwiGLU prologues take
bl_status chain_build(int form, const bl_chain_layer* layers, int n, void* chain, size_t bytes,
                      bl_chain_plan* plan, cudaStream_t s);
bl_status chain_run(const bl_chain_plan* plan, const void* chain, unsigned int* flags,
                    cudaStream_t s);

// Every kernel of the library runs with the whole L1/shared-memory carveout
// given to shared memory.  An SM changes its carveout only when it is idle, so
// kernels with differing carveouts could not share an SM: the next call's CTAs
// (launched early, programmatic dependent launch) would then wait for SMs to
// drain and pile up two to an SM.
template <typename Kern>
inline cudaError_t use_max_shared_carveout(Kern kern) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutMaxShared);
}

// One-time setup of a kernel's launch attributes (maximum dynamic shared
// memory, shared-memory carveout), done once per device: cudaFuncSetAttribute
// acts on the current device's context only, so a process that runs the
// library on several devices sets them on each.  Safe to call from several
// host threads.  Each launcher keeps one function-local static instance per
// kernel.
class KernelAttrs {
public:
    template <typename Kern>
    cudaError_t ensure(Kern kern, int max_dyn_smem) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
        if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lk(mu_);
        if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        if (max_dyn_smem > 0) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn_smem);
            if (e != cudaSuccess) return e;
        }
        e = use_max_shared_carveout(kern);
        if (e != cudaSuccess) return e;
        done_[dev].store(true, std::memory_order_release);
        return cudaSuccess;
    }

private:
    static constexpr int kMaxDev = 128;
    std::mutex mu_;
    std::atomic<bool> done_[kMaxDev] = {};
};

// Largest M for which the streamed decode CTA prepares the activations itself
// (ternary; OneBit, three columns per token, up to M = 2).
constexpr int kStreamFusedMaxM = 8;
constexpr int kStreamFusedMaxMOnebit = 2;

// Token counts at which the tensor-core prefill kernel is used (measured
// crossovers on 13B-shaped layers: ternary M = 16 runs 26 % faster there than
// in the prepared streamed kernel).
constexpr int kTernaryPrefillMinM = 9;
// OneBit calls take the tensor-core path from 4 tokens, and at 3 tokens on
// layers of more than 16384 rows, where the streamed plan is slower (measured
// on the 13B-shaped layers and the BiLLM layer's stacked planes).
inline bool onebit_prefill(int M, int N) { return M >= 4 || (M == 3 && N > 16384); }

}  // namespace bl
