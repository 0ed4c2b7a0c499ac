// api.cu -- the C ABI (include/bitlinear.h): argument validation, workspace
// layout and shape dispatch.  No allocation happens here; all buffers are the
// caller's.
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bitlinear.h"
#include "common.cuh"
#include "kernels.h"

namespace bl {
__device__ unsigned int g_device_flags = 0;
// Error word of the packers (one per device; packer calls must not overlap).
__device__ unsigned int g_pack_error = 0;
}  // namespace bl

namespace {

constexpr size_t kAlign = 256;
// chain length: the layer table lives in shared memory (32 bytes a layer) and
// layer indexes are 16-bit there
constexpr int kMaxChainLayers = 2048;

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

inline bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

inline cudaStream_t cs(bl_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

bl_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BL_OK : BL_ERR_CUDA; }

// Shape rules shared by every entry point.  Sizes are also capped so that
// M*K, N*K and M*N byte counts stay far inside size_t and int32 indexing of
// rows.
bl_status check_mk(int M, int K) {
    if (M < 0 || K <= 0 || K % 128 != 0) return BL_ERR_SHAPE;
    if (K > (1 << 20) || M > (1 << 24)) return BL_ERR_SHAPE;
    return BL_OK;
}

bl_status check_nk(int N, int K) {
    if (N < 0 || N % 16 != 0 || K <= 0 || K % 128 != 0) return BL_ERR_SHAPE;
    if (K > (1 << 20) || N > (1 << 24)) return BL_ERR_SHAPE;
    return BL_OK;
}

// Workspace layouts (offsets in bytes, each region 256-byte aligned):
//   ternary: [0] permuted q  M*K int8 | scale M fp32 | row sums M int32 | split
//   onebit : [0] limb planes 3*M*K int8 | step M fp32 | image sums M int64 | split
// `split` is the prefill kernel's scratch for sharing out its last round
// (arrival counters + partial accumulators); empty unless the call takes the
// prefill path and its tiles leave SMs idle in the last round.
struct WsLayout {
    size_t act, scale, rsum, split, split_bytes, total;
    int n_ctr;
};

WsLayout ws_layout(int form, int M, int K, int N) {
    WsLayout l;
    l.act = 0;
    l.scale = align_up((size_t)M * (size_t)K * (size_t)(form == 0 ? 1 : 3));
    l.rsum = l.scale + align_up((size_t)M * sizeof(float));
    l.split = l.rsum + align_up((size_t)M * (form == 0 ? sizeof(int32_t) : sizeof(long long)));
    l.split_bytes = 0;
    l.n_ctr = 0;
    const bool prefill = form == 0 ? M >= bl::kTernaryPrefillMinM : bl::onebit_prefill(M, N);
    if (prefill) l.split_bytes = bl::prefill_split_bytes(form, M, K, N, &l.n_ctr);
    l.total = l.split + align_up(l.split_bytes);
    return l;
}

bl_status pack_finish(cudaError_t launch_err, cudaStream_t s) {
    if (launch_err != cudaSuccess) return BL_ERR_CUDA;
    unsigned int host_err = 0;
    if (cudaMemcpyFromSymbolAsync(&host_err, bl::g_pack_error, sizeof(host_err), 0,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return BL_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
    return host_err ? BL_ERR_INVALID_VALUE : BL_OK;
}

unsigned int* device_flags() {
    unsigned int* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), bl::g_device_flags) != cudaSuccess)
        return nullptr;
    return p;
}

bl_status pack_begin(unsigned int** flag, cudaStream_t s) {
    static const unsigned int zero = 0;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(flag), bl::g_pack_error) != cudaSuccess)
        return BL_ERR_CUDA;
    if (cudaMemcpyToSymbolAsync(bl::g_pack_error, &zero, sizeof(zero), 0,
                                cudaMemcpyHostToDevice, s) != cudaSuccess)
        return BL_ERR_CUDA;
    return BL_OK;
}

}  // namespace

unsigned int* bl::device_flags_address() { return device_flags(); }

int bl::device_sm_count() {
    static std::mutex mu;
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cached[dev] = n;
    }
    return cached[dev];
}

// Host-side fault injection for callers' error paths: with the environment
// variable BL_FAULT_INJECT set to "cuda" or "timeout", every entry point that
// would launch work returns BL_ERR_CUDA or BL_ERR_TIMEOUT after validating its
// arguments and before any CUDA call.  Read on every call (a test may change
// it between calls).  Nothing on the device is touched.
bl_status bl::fault_injected() {
    const char* v = std::getenv("BL_FAULT_INJECT");
    if (v == nullptr || *v == 0) return BL_OK;
    if (std::strcmp(v, "cuda") == 0) return BL_ERR_CUDA;
    if (std::strcmp(v, "timeout") == 0) return BL_ERR_TIMEOUT;
    return BL_OK;
}

namespace {
// Pending stall of the next streamed-decode or whole-tile tensor-core launch
// (bl_debug_stall_next_launch); 0 = none.
std::atomic<unsigned long long> g_stall_next{0};
}  // namespace

unsigned long long bl::take_stall() {
    if (g_stall_next.load(std::memory_order_relaxed) == 0) return 0;
    return g_stall_next.exchange(0);
}

size_t bl::ternary_act_bytes(int M, int K) { return ws_layout(0, M, K, 0).split; }

bl_status bl::ternary_linear_on(const uint16_t* x, int M, int K, int N, const uint32_t* w2,
                                float w_scale, uint16_t* y, int32_t* acc_out, void* workspace,
                                size_t workspace_bytes, cudaStream_t s) {
    if (bl_status st = bl::fault_injected()) return st;
    unsigned int* flags = device_flags();
    if (!flags) return BL_ERR_CUDA;
    if (M <= bl::kStreamFusedMaxM && bl::stream_fits(0, M, K, N, 0))
        return from_cuda(bl::launch_ternary_stream(x, w2, M, K, N, w_scale, y, acc_out, flags, s));
    WsLayout l = ws_layout(0, M, K, N);
    if (workspace_bytes < l.total) {   // room for the activations only: whole prefill tiles
        l.split_bytes = 0;
        l.n_ctr = 0;
    }
    char* ws = static_cast<char*>(workspace);
    int8_t* qp = reinterpret_cast<int8_t*>(ws + l.act);
    float* sc = reinterpret_cast<float*>(ws + l.scale);
    int32_t* qs = reinterpret_cast<int32_t*>(ws + l.rsum);
    unsigned int* ctr = reinterpret_cast<unsigned int*>(ws + l.split);
    cudaError_t e = bl::launch_quant_ternary_perm(x, M, K, qp, sc, qs, s, ctr, l.n_ctr);
    if (e != cudaSuccess) return BL_ERR_CUDA;
    if (M >= bl::kTernaryPrefillMinM) {
        e = bl::launch_ternary_prefill(w2, qp, sc, qs, M, K, N, w_scale, y, acc_out, flags, s,
                                       l.split_bytes ? ws + l.split : nullptr, l.split_bytes);
    } else {
        e = bl::stream_fits(0, M, K, N, 1)
                ? bl::launch_ternary_stream_prepared(qp, sc, qs, w2, M, K, N, w_scale, y, acc_out,
                                                     flags, s)
                : bl::launch_ternary_skinny(w2, qp, sc, qs, M, K, N, w_scale, y, acc_out, s);
    }
    return from_cuda(e);
}

extern "C" {

const char* bl_status_string(int status) {
    switch (status) {
        case BL_OK: return "BL_OK";
        case BL_ERR_NULL: return "BL_ERR_NULL: a required pointer is NULL";
        case BL_ERR_SHAPE: return "BL_ERR_SHAPE: M, N or K violates the shape rules";
        case BL_ERR_ALIGN: return "BL_ERR_ALIGN: a pointer is not 16-byte aligned";
        case BL_ERR_INVALID_VALUE: return "BL_ERR_INVALID_VALUE: an input value the format cannot hold";
        case BL_ERR_CUDA: return "BL_ERR_CUDA: a CUDA call or kernel launch failed";
        case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT: a bounded device-side wait expired";
        case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE: workspace missing or too small";
        case BL_ERR_SCRATCH_LIMIT:
            return "BL_ERR_SCRATCH_LIMIT: shape exceeds the fixed scratch of the no-allocation entry point";
        default: return "unknown bl_status";
    }
}

int bl_abi_version(void) { return 100; }

bl_status bl_pack_ternary(const int8_t* w, int N, int K, uint32_t* w2, bl_stream_t stream) {
    if (bl_status st = check_nk(N, K)) return st;
    if (N == 0) return BL_OK;
    if (!w || !w2) return BL_ERR_NULL;
    if (misaligned(w) || misaligned(w2)) return BL_ERR_ALIGN;
    if (bl_status st = bl::fault_injected()) return st;
    unsigned int* flag = nullptr;
    if (bl_status st = pack_begin(&flag, cs(stream))) return st;
    return pack_finish(bl::launch_pack_ternary(w, N, K, w2, flag, cs(stream)), cs(stream));
}

bl_status ob_pack_sign(const uint16_t* w, int N, int K, uint32_t* s1, bl_stream_t stream) {
    if (bl_status st = check_nk(N, K)) return st;
    if (N == 0) return BL_OK;
    if (!w || !s1) return BL_ERR_NULL;
    if (misaligned(w) || misaligned(s1)) return BL_ERR_ALIGN;
    if (bl_status st = bl::fault_injected()) return st;
    unsigned int* flag = nullptr;
    if (bl_status st = pack_begin(&flag, cs(stream))) return st;
    return pack_finish(bl::launch_pack_sign(w, N, K, s1, flag, cs(stream)), cs(stream));
}

bl_status bl_quant_act(const uint16_t* x, int M, int K, int8_t* q, float* scale,
                       bl_stream_t stream) {
    if (bl_status st = check_mk(M, K)) return st;
    if (M == 0) return BL_OK;
    if (!x || !q || !scale) return BL_ERR_NULL;
    if (misaligned(x) || misaligned(q) || misaligned(scale)) return BL_ERR_ALIGN;
    if (bl_status st = bl::fault_injected()) return st;
    return from_cuda(bl::launch_quant_plain(x, M, K, q, scale, cs(stream)));
}

size_t bl_ternary_workspace_bytes(int M, int K, int N) {
    if (check_mk(M, K) != BL_OK || check_nk(N, K) != BL_OK) return 0;
    return ws_layout(0, M, K, N).total;
}

bl_status bl_ternary_linear(const uint16_t* x, int M, int K, int N, const uint32_t* w2,
                            float w_scale, uint16_t* y, int32_t* acc_out, void* workspace,
                            size_t workspace_bytes, bl_stream_t stream) {
    if (bl_status st = check_mk(M, K)) return st;
    if (bl_status st = check_nk(N, K)) return st;
    if (M == 0 || N == 0) return BL_OK;
    if (!x || !w2 || !y) return BL_ERR_NULL;
    if (misaligned(x) || misaligned(w2) || misaligned(y) || misaligned(acc_out))
        return BL_ERR_ALIGN;
    const WsLayout l = ws_layout(0, M, K, N);
    if (!workspace || workspace_bytes < l.total) return BL_ERR_WORKSPACE;
    if (misaligned(workspace)) return BL_ERR_ALIGN;
    return bl::ternary_linear_on(x, M, K, N, w2, w_scale, y, acc_out, workspace, workspace_bytes,
                                 cs(stream));
}

size_t ob_workspace_bytes(int M, int K, int N) {
    if (check_mk(M, K) != BL_OK || check_nk(N, K) != BL_OK || K > 65536) return 0;
    return ws_layout(1, M, K, N).total;
}

// The OneBit forward (argument checks done): the fused streamed kernel for the
// smallest M, else activation preparation and then the streamed, skinny or
// tensor-core contraction.  zf: optional fp32 copy of the output.
static bl_status onebit_forward(const uint16_t* x, int M, int K, int N, const uint32_t* s1,
                                const uint16_t* g, const uint16_t* h, uint16_t* y, float* zf,
                                char* ws, const WsLayout& l, cudaStream_t s) {
    unsigned int* flags = device_flags();
    if (!flags) return BL_ERR_CUDA;
    if (M <= bl::kStreamFusedMaxMOnebit && bl::stream_fits(1, M, K, N, 0))
        return from_cuda(bl::launch_onebit_stream(x, g, h, s1, M, K, N, y, flags, s, zf));
    int8_t* planes = reinterpret_cast<int8_t*>(ws + l.act);
    float* step = reinterpret_cast<float*>(ws + l.scale);
    long long* ts = reinterpret_cast<long long*>(ws + l.rsum);
    unsigned int* ctr = reinterpret_cast<unsigned int*>(ws + l.split);
    cudaError_t e = bl::launch_prep_onebit(x, g, M, K, planes, step, ts, s, ctr, l.n_ctr);
    if (e != cudaSuccess) return BL_ERR_CUDA;
    if (bl::onebit_prefill(M, N)) {
        e = bl::launch_onebit_prefill(s1, planes, step, ts, h, M, K, N, y, flags, s, ws + l.split,
                                      l.split_bytes, zf);
    } else {
        e = bl::stream_fits(1, M, K, N, 1)
                ? bl::launch_onebit_stream_prepared(planes, step, ts, h, s1, M, K, N, y, flags, s, zf)
                : bl::launch_onebit_skinny(s1, planes, step, ts, h, M, K, N, y, s, zf);
    }
    return from_cuda(e);
}

bl_status ob_linear(const uint16_t* x, int M, int K, int N, const uint32_t* s1,
                    const uint16_t* g, const uint16_t* h, uint16_t* y, void* workspace,
                    size_t workspace_bytes, bl_stream_t stream) {
    if (bl_status st = check_mk(M, K)) return st;
    if (bl_status st = check_nk(N, K)) return st;
    if (K > 65536) return BL_ERR_SHAPE;
    if (M == 0 || N == 0) return BL_OK;
    if (!x || !s1 || !g || !h || !y) return BL_ERR_NULL;
    if (misaligned(x) || misaligned(s1) || misaligned(g) || misaligned(h) || misaligned(y))
        return BL_ERR_ALIGN;
    const WsLayout l = ws_layout(1, M, K, N);
    if (!workspace || workspace_bytes < l.total) return BL_ERR_WORKSPACE;
    if (misaligned(workspace)) return BL_ERR_ALIGN;
    if (bl_status st = bl::fault_injected()) return st;
    return onebit_forward(x, M, K, N, s1, g, h, y, nullptr, static_cast<char*>(workspace), l,
                          cs(stream));
}

// Two-plane binary layer: the OneBit forward over the stacked planes (2N rows,
// g = 1, h = alpha) writes fp32 products zf [M][2N] (and an fp16 copy in
// scratch), then y = fp16(zf[:, :N] + zf[:, N:]).
//   workspace: OneBit layout for (M, K, 2N) | zf M*2N fp32 | scratch y M*2N fp16
struct BillmWs {
    WsLayout ob;
    size_t zf, ysc, total;
};

static BillmWs billm_ws(int M, int K, int N) {
    BillmWs b;
    b.ob = ws_layout(1, M, K, 2 * N);
    b.zf = b.ob.total;
    b.ysc = b.zf + align_up((size_t)M * 2 * N * sizeof(float));
    b.total = b.ysc + align_up((size_t)M * 2 * N * sizeof(uint16_t));
    return b;
}

static bl_status check_billm_shape(int M, int K, int N) {
    if (bl_status st = check_mk(M, K)) return st;
    if (bl_status st = check_nk(N, K)) return st;
    if (K > 65536 || N > (1 << 23)) return BL_ERR_SHAPE;
    return BL_OK;
}

size_t billm_workspace_bytes(int M, int K, int N) {
    if (check_billm_shape(M, K, N) != BL_OK) return 0;
    return billm_ws(M, K, N).total;
}

bl_status billm_linear(const uint16_t* x, int M, int K, int N, const uint32_t* b2,
                       const uint16_t* alpha, uint16_t* y, void* workspace, size_t workspace_bytes,
                       bl_stream_t stream) {
    if (bl_status st = check_billm_shape(M, K, N)) return st;
    if (M == 0 || N == 0) return BL_OK;
    if (!x || !b2 || !alpha || !y) return BL_ERR_NULL;
    if (misaligned(x) || misaligned(b2) || misaligned(alpha) || misaligned(y)) return BL_ERR_ALIGN;
    const BillmWs l = billm_ws(M, K, N);
    if (!workspace || workspace_bytes < l.total) return BL_ERR_WORKSPACE;
    if (misaligned(workspace)) return BL_ERR_ALIGN;
    if (bl_status st = bl::fault_injected()) return st;
    char* ws = static_cast<char*>(workspace);
    float* zf = reinterpret_cast<float*>(ws + l.zf);
    uint16_t* ysc = reinterpret_cast<uint16_t*>(ws + l.ysc);
    if (bl_status st = onebit_forward(x, M, K, 2 * N, b2, nullptr, alpha, ysc, zf, ws, l.ob, cs(stream)))
        return st;
    return from_cuda(bl::launch_billm_combine(zf, M, N, y, cs(stream)));
}

bl_status billm_binarize(const float* W, int N, int K, uint32_t* b2, uint16_t* alpha,
                         double* alpha_o, double* alpha_r, bl_stream_t stream) {
    if (bl_status st = check_nk(N, K)) return st;
    if (N > (1 << 23)) return BL_ERR_SHAPE;
    if (N == 0) return BL_OK;
    if (!W || !b2 || !alpha) return BL_ERR_NULL;
    if (misaligned(W) || misaligned(b2) || misaligned(alpha) || misaligned(alpha_o) ||
        misaligned(alpha_r))
        return BL_ERR_ALIGN;
    if (bl_status st = bl::fault_injected()) return st;
    unsigned int* flag = nullptr;
    if (bl_status st = pack_begin(&flag, cs(stream))) return st;
    return pack_finish(bl::launch_billm_binarize(W, N, K, b2, alpha, alpha_o, alpha_r, flag, cs(stream)),
                       cs(stream));
}

static bl_status check_svid_shape(int N, int K) {
    if (bl_status st = check_nk(N, K)) return st;
    if (N > bl::svid_max_n()) return BL_ERR_SHAPE;
    return BL_OK;
}

size_t ob_svid_workspace_bytes(int N, int K) {
    if (check_svid_shape(N, K) != BL_OK || N == 0) return 0;
    return bl::svid_workspace_bytes(N, K);
}

bl_status ob_svid(const float* W, int N, int K, int max_iter, double tol, uint32_t* s1, uint16_t* g,
                  uint16_t* h, double* a, double* b, double* sigma, int* iters, void* workspace,
                  size_t workspace_bytes, bl_stream_t stream) {
    if (bl_status st = check_svid_shape(N, K)) return st;
    if (max_iter < 1 || !(tol >= 0.0)) return BL_ERR_SHAPE;
    if (N == 0) return BL_OK;
    if (!W || !s1 || !g || !h) return BL_ERR_NULL;
    if (misaligned(W) || misaligned(s1) || misaligned(g) || misaligned(h) || misaligned(a) ||
        misaligned(b))
        return BL_ERR_ALIGN;
    if (!workspace || workspace_bytes < bl::svid_workspace_bytes(N, K)) return BL_ERR_WORKSPACE;
    if (misaligned(workspace)) return BL_ERR_ALIGN;
    if (bl_status st = bl::fault_injected()) return st;
    return bl::svid_run(W, N, K, max_iter, tol, s1, g, h, a, b, sigma, iters, workspace, cs(stream));
}

bl_status bl_prefill_plan(int form, int M, int K, int N, int sm_count, int* plan) {
    if (!plan) return BL_ERR_NULL;
    if (form != 0 && form != 1) return BL_ERR_SHAPE;
    if (bl_status st = check_mk(M, K)) return st;
    if (bl_status st = check_nk(N, K)) return st;
    if (M == 0 || N == 0 || sm_count <= 0) return BL_ERR_SHAPE;
    bl::prefill_plan_info(form, M, K, N, sm_count, plan);
    return BL_OK;
}

size_t bl_chain_bytes(int n_layers) {
    if (n_layers <= 0 || n_layers > kMaxChainLayers) return 0;
    return bl::chain_bytes(n_layers);
}

bl_status bl_chain_build(int form, const bl_chain_layer* layers, int n_layers, void* chain,
                         size_t chain_bytes, bl_chain_plan* plan, bl_stream_t stream) {
    if (!layers || !chain || !plan) return BL_ERR_NULL;
    if ((form != 0 && form != 1) || n_layers <= 0 || n_layers > kMaxChainLayers) return BL_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(chain) & 255u) != 0) return BL_ERR_ALIGN;
    for (int j = 0; j < n_layers; ++j) {
        const bl_chain_layer& L = layers[j];
        if (L.K <= 0 || L.K % 128 != 0 || L.K > bl::chain_max_k(form) || L.N <= 0 || L.N % 16 != 0 ||
            L.N > (1 << 24))
            return BL_ERR_SHAPE;
        if (L.src < -1 || L.src >= j) return BL_ERR_SHAPE;
        if (L.src >= 0 && layers[L.src].N != L.K) return BL_ERR_SHAPE;
        if (L.src2 < -1 || L.src2 >= j || (L.src2 >= 0 && (L.src < 0 || layers[L.src2].N != L.K)))
            return BL_ERR_SHAPE;
        // the fused prologues work on a row held in registers
        if ((L.src2 >= 0 || L.norm_w) && L.K > bl::chain_max_fused_k(form)) return BL_ERR_SHAPE;
        if (L.norm_w && !(L.norm_eps >= 0.f)) return BL_ERR_SHAPE;
        if ((L.src < 0 && !L.x) || !L.w || !L.y || (form == 1 && (!L.g || !L.h))) return BL_ERR_NULL;
        if ((L.src < 0 && misaligned(L.x)) || misaligned(L.w) || misaligned(L.y) ||
            misaligned(L.acc_out) || misaligned(L.g) || misaligned(L.h) || misaligned(L.norm_w) ||
            misaligned(L.swiglu_buf))
            return BL_ERR_ALIGN;
        if (L.swiglu_buf && L.src2 < 0) return BL_ERR_SHAPE;
    }
    if (chain_bytes < bl::chain_bytes(n_layers)) return BL_ERR_WORKSPACE;
    if (bl_status st = bl::fault_injected()) return st;
    return bl::chain_build(form, layers, n_layers, chain, chain_bytes, plan, cs(stream));
}

static bl_status check_chain_plan(const bl_chain_plan* plan, const void* chain) {
    if (!plan || !chain) return BL_ERR_NULL;
    if ((plan->form != 0 && plan->form != 1) || plan->n_layers <= 0 ||
        plan->n_layers > kMaxChainLayers || (plan->fused != 0 && plan->fused != 1))
        return BL_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(chain) & 255u) != 0) return BL_ERR_ALIGN;
    return BL_OK;
}

bl_status bl_chain_run(const bl_chain_plan* plan, const void* chain, bl_stream_t stream) {
    if (bl_status st = check_chain_plan(plan, chain)) return st;
    if (bl_status st = bl::fault_injected()) return st;
    unsigned int* flags = device_flags();
    if (!flags) return BL_ERR_CUDA;
    return bl::chain_run(plan, chain, flags, cs(stream));
}

bl_status bl_chain_run_host(const bl_chain_plan* plan, const void* chain, const bl_copy* in,
                            int n_in, const bl_copy* out, int n_out, bl_stream_t stream) {
    if (bl_status st = check_chain_plan(plan, chain)) return st;
    if (n_in < 0 || n_out < 0) return BL_ERR_SHAPE;
    if ((n_in > 0 && !in) || (n_out > 0 && !out)) return BL_ERR_NULL;
    for (int i = 0; i < n_in; ++i)
        if (in[i].bytes && (!in[i].src || !in[i].dst)) return BL_ERR_NULL;
    for (int i = 0; i < n_out; ++i)
        if (out[i].bytes && (!out[i].src || !out[i].dst)) return BL_ERR_NULL;
    if (bl_status st = bl::fault_injected()) return st;
    unsigned int* flags = device_flags();
    if (!flags) return BL_ERR_CUDA;
    for (int i = 0; i < n_in; ++i)
        if (in[i].bytes && cudaMemcpyAsync(in[i].dst, in[i].src, in[i].bytes, cudaMemcpyHostToDevice,
                                           cs(stream)) != cudaSuccess)
            return BL_ERR_CUDA;
    if (bl_status st = bl::chain_run(plan, chain, flags, cs(stream))) return st;
    for (int i = 0; i < n_out; ++i)
        if (out[i].bytes && cudaMemcpyAsync(out[i].dst, out[i].src, out[i].bytes, cudaMemcpyDeviceToHost,
                                            cs(stream)) != cudaSuccess)
            return BL_ERR_CUDA;
    return BL_OK;
}

bl_status bl_debug_stall_next_launch(unsigned long long wait_limit_ns) {
    g_stall_next.store(wait_limit_ns);
    return BL_OK;
}

bl_status bl_device_status(bl_stream_t stream) {
    if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return BL_ERR_CUDA;
    unsigned int flags = 0;
    static const unsigned int zero = 0;
    if (cudaMemcpyFromSymbol(&flags, bl::g_device_flags, sizeof(flags)) != cudaSuccess)
        return BL_ERR_CUDA;
    if (flags && cudaMemcpyToSymbol(bl::g_device_flags, &zero, sizeof(zero)) != cudaSuccess)
        return BL_ERR_CUDA;
    return (flags & bl::kFlagTimeout) ? BL_ERR_TIMEOUT : BL_OK;
}

}  // extern "C"
