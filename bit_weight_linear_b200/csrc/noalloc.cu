// noalloc.cu -- bl_ternary_linear_noalloc: the BitLinear forward for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run the layer: for example a plugin loaded into a host program that owns
// all device memory and hands the plugin no allocator, or a latency-critical
// loop whose rules forbid allocation because cudaMalloc can block on the whole
// device.  For them this entry point needs only inputs and outputs: its scratch
// (the prepared int8 activations, token scales and row sums) lives in a
// fixed-size array compiled into this library.  The arithmetic and the kernels
// are those of bl_ternary_linear's two-kernel path (activation preparation,
// then the packed-weight contraction), so results are identical.
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

inline size_t round256(size_t v) { return (v + 255) / 256 * 256; }

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
    // scratch layout: permuted q [M][K] | token scales [M] | row sums [M], each 256-aligned
    const size_t off_scale = round256((size_t)M * (size_t)K);
    const size_t off_rsum = off_scale + round256((size_t)M * sizeof(float));
    const size_t need = off_rsum + round256((size_t)M * sizeof(int32_t));
    if (need > kScratchBytes) return BL_ERR_SCRATCH_LIMIT;

    void* base = nullptr;
    if (bl_status st = scratch_address(&base)) return st;
    unsigned int* flags = bl::device_flags_address();
    if (!flags) return BL_ERR_CUDA;
    char* ws = static_cast<char*>(base);
    int8_t* qp = reinterpret_cast<int8_t*>(ws);
    float* sc = reinterpret_cast<float*>(ws + off_scale);
    int32_t* qs = reinterpret_cast<int32_t*>(ws + off_rsum);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // Every scratch byte read below is first written by this call's preparation
    // kernel, so nothing needs clearing between calls.
    if (bl::launch_quant_ternary_perm(x, M, K, qp, sc, qs, s) != cudaSuccess) return BL_ERR_CUDA;
    cudaError_t e;
    if (M >= bl::kTernaryPrefillMinM)
        e = bl::launch_ternary_prefill(w2, qp, sc, qs, M, K, N, w_scale, y, acc_out, flags, s);
    else
        e = bl::launch_ternary_skinny(w2, qp, sc, qs, M, K, N, w_scale, y, acc_out, s);
    return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}
