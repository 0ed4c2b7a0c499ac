// noalloc.cu -- bl_ternary_linear_noalloc: the BitLinear forward for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run the layer: for example a plugin loaded into a host program that owns
// all device memory and hands the plugin no allocator, or a latency-critical
// loop whose rules forbid allocation because cudaMalloc can block on the whole
// device.  For them this entry point needs only inputs and outputs: its scratch
// (the prepared int8 activations, token scales and row sums) lives in a
// fixed-size array compiled into this library.  It runs the same forward as
// bl_ternary_linear (same kernels, same dispatch by shape), so results are
// identical; only the tensor-core path's balanced last round, whose scratch
// grows with the layer, is left out when it would not fit in the array (every
// tile then runs whole, with the same integers).
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds one copy of it until the process exits.  Host code cannot use
// the variable's name as a device address, so the first call on each device
// looks its address up (cudaGetSymbolAddress, with that device current) and
// caches it; make that first call before any stream capture.
#include <mutex>

#include "bitlinear.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = BL_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Address of this device's scratch array (looked up once per device).
bl_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BL_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return BL_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return BL_OK;
}

inline bool misaligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace

extern "C" bl_status bl_ternary_linear_noalloc(const uint16_t* x, int M, int K, int N,
                                               const uint32_t* w2, float w_scale, uint16_t* y,
                                               int32_t* acc_out, bl_stream_t stream) {
    if (M < 0 || N < 0 || N % 16 != 0 || K <= 0 || K % 128 != 0 || K > (1 << 20) ||
        M > (1 << 24) || N > (1 << 24))
        return BL_ERR_SHAPE;
    if (M == 0 || N == 0) return BL_OK;
    if (!x || !w2 || !y) return BL_ERR_NULL;
    if (misaligned16(x) || misaligned16(w2) || misaligned16(y) || misaligned16(acc_out))
        return BL_ERR_ALIGN;
    // scratch layout: permuted q [M][K] | token scales [M] | row sums [M], each
    // 256-byte aligned (the layout of bl_ternary_linear's workspace)
    if (bl::ternary_act_bytes(M, K) > kScratchBytes) return BL_ERR_SCRATCH_LIMIT;
    if (bl_status st = bl::fault_injected()) return st;
    void* base = nullptr;
    if (bl_status st = scratch_address(&base)) return st;
    // Every scratch byte the kernels read is first written by this call's
    // activation kernel (which also zeroes the balanced round's counters), so
    // nothing needs clearing between calls.
    return bl::ternary_linear_on(x, M, K, N, w2, w_scale, y, acc_out, base, kScratchBytes,
                                 reinterpret_cast<cudaStream_t>(stream));
}
