// svid.cu -- SVID initialisation of a OneBit layer on the device.
//
// OneBit page ("清华、哈工大把大模型压缩到了1bit…"), "2. 基于 SVID 初始化量化模型":
// a trained weight W [N, K] is split into its sign matrix S = sign(W) and a
// rank-1 approximation of |W| = a b^T, so W ~ S (.) (a b^T); the layer then
// uses h = a (output side, length N) and g = b (input side, length K), which
// is the order swap of the same section:  x (S (.) a b^T)^T = ((x (.) b) S^T) (.) a.
// The rank-1 factor is the leading singular pair of |W| (the SVD reading of
// the page's "SVD or NMF"), split as a = sqrt(sigma) u, b = sqrt(sigma) v,
// found by power iteration from v = 1/sqrt(K):
//     u = |W| v / || |W| v ||,   v' = |W|^T u,   sigma = ||v'||,   v = v' / sigma
// until |sigma - sigma_prev| <= tol * sigma (from the second iteration on).
//
// Per iteration three kernels, all fp64 in the arithmetic (W is fp32):
//   row pass     u_raw[n] = sum_k |W[n,k]| v[k] / ||v||       (a warp per row)
//   column pass  part[s][k] = sum_{n in split s} |W[n,k]| u_raw[n] / ||u_raw||
//                (a thread per column, rows split over blockIdx.y)
//   finish       v[k] = sum_s part[s][k]; sigma = ||v||; convergence test
// Norms are reduced per CTA and then by the last CTA to finish (a ticket
// counter), each in a fixed order, so a run is deterministic.  Once the
// convergence flag is set, the kernels of later iterations return at once.
// W (64 MB at 4096 x 4096) stays in L2 across iterations; every pass is
// bound by reading it (4 bytes per element per pass).
#include <cmath>
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace bl {
namespace {

constexpr int kRowWarps = 8;          // rows per CTA of the row pass
constexpr int kColThreads = 256;      // columns per CTA of the column pass
constexpr int kMaxSplits = 128;       // row splits of the column pass
constexpr int kFinThreads = 256;
constexpr int kMaxRowsPerSplit = 4096;   // rows a column-pass CTA stages (N <= 128 x 4096)

struct SvidState {
    double vnorm;       // ||v|| of the current v (sigma after a column pass)
    double unorm;       // ||u_raw|| of the last row pass
    double prev;        // sigma of the previous iteration
    double tol;
    int it;             // completed iterations
    int done;           // converged: later kernels return at once
    unsigned int ticket_row, ticket_fin;
    unsigned int bad;   // a non-finite W element was seen
    int max_iter;
};

struct SvidWs {
    size_t state, u, v, part, red, total;
    int splits, rows_per_split;
};

SvidWs svid_layout(int N, int K) {
    SvidWs l;
    l.splits = N < kMaxSplits ? N : kMaxSplits;
    l.rows_per_split = (N + l.splits - 1) / l.splits;
    l.splits = (N + l.rows_per_split - 1) / l.rows_per_split;
    const int row_ctas = (N + kRowWarps - 1) / kRowWarps;
    const int fin_ctas = (K + kFinThreads - 1) / kFinThreads;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) / 256 * 256; return o; };
    l.state = take(sizeof(SvidState));
    l.u = take((size_t)N * 8);
    l.v = take((size_t)K * 8);
    l.part = take((size_t)l.splits * K * 8);
    l.red = take((size_t)(row_ctas > fin_ctas ? row_ctas : fin_ctas) * 8);
    l.total = off;
    return l;
}

// sign bits (bit k%32 of word [n][k/32] is 1 iff W >= 0, -0 included) and a
// finiteness check; one thread per word
__global__ void __launch_bounds__(256) svid_sign_kernel(const float* __restrict__ W, size_t nwords,
                                                        uint32_t* __restrict__ s1, SvidState* st) {
    const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    if (i >= nwords) return;
    const float* src = W + 32 * i;
    uint32_t word = 0;
    bool bad = false;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = ld_stream_v4(src + 4 * c);
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t mag = in[e] & 0x7fffffffu;
            bad |= mag >= 0x7f800000u;                        // inf or NaN
            const bool neg = (in[e] >> 31) && mag != 0;       // -0 counts as +1
            word |= (neg ? 0u : 1u) << (4 * c + e);
        }
    }
    s1[i] = word;
    if (bad) atomicOr(&st->bad, 1u);
}

__global__ void svid_init_kernel(double* v, int K, SvidState* st, double tol, int max_iter) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k < K) v[k] = 1.0;
    if (k == 0) {
        st->vnorm = sqrt((double)K);
        st->unorm = 0.0;
        st->prev = 0.0;
        st->tol = tol;
        st->it = 0;
        st->done = 0;
        st->ticket_row = 0;
        st->ticket_fin = 0;
        st->bad = 0;
        st->max_iter = max_iter;
    }
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum the CTA's per-warp values in warp order; the last CTA of the grid to
// arrive (ticket) sums the per-CTA values in CTA order and returns true with
// the total in *total (thread 0 only).
__device__ bool grid_sum_last(double mine_warp, double* sm_warps, int nwarps, double* red,
                              unsigned int* ticket, double* total) {
    __shared__ bool last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sm_warps[warp] = mine_warp;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int w = 0; w < nwarps; ++w) s += sm_warps[w];
        red[blockIdx.x] = s;
        __threadfence();
        const unsigned int t = atomicAdd(ticket, 1u);
        last = t == gridDim.x - 1;
        if (last) {
            __threadfence();
            double g = 0.0;
            for (unsigned int b = 0; b < gridDim.x; ++b) g += __ldcg(red + b);
            *total = g;
            *ticket = 0;
        }
    }
    __syncthreads();
    return last;
}

// u_raw[n] = sum_k |W[n,k]| v[k] / ||v||, and ||u_raw||
__global__ void __launch_bounds__(kRowWarps * 32) svid_row_kernel(const float* __restrict__ W, int N,
                                                                  int K, const double* __restrict__ v,
                                                                  double* __restrict__ u, double* red,
                                                                  SvidState* st) {
    if (*(volatile int*)&st->done) return;
    __shared__ double sm[kRowWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kRowWarps + warp;
    const double vn = st->vnorm;
    double acc = 0.0;
    if (n < N) {
        const float* row = W + (size_t)n * K;
#pragma unroll 4
        for (int k = 4 * lane; k < K; k += 128) {
            const float4 w = *reinterpret_cast<const float4*>(row + k);
            const double2 v01 = __ldg(reinterpret_cast<const double2*>(v + k));
            const double2 v23 = __ldg(reinterpret_cast<const double2*>(v + k + 2));
            acc = fma(fabs((double)w.x), v01.x, acc);
            acc = fma(fabs((double)w.y), v01.y, acc);
            acc = fma(fabs((double)w.z), v23.x, acc);
            acc = fma(fabs((double)w.w), v23.y, acc);
        }
        acc = warp_sum_d(acc) / vn;
        if (lane == 0) u[n] = acc;
    }
    double total;
    if (grid_sum_last(n < N ? acc * acc : 0.0, sm, kRowWarps, red, &st->ticket_row, &total) &&
        threadIdx.x == 0)
        st->unorm = sqrt(total);
}

// part[s][k] = sum over the split's rows of |W[n,k]| u_raw[n] / ||u_raw||
__global__ void __launch_bounds__(kColThreads) svid_col_kernel(const float* __restrict__ W, int N,
                                                               int K, const double* __restrict__ u,
                                                               double* __restrict__ part,
                                                               int rows_per_split, SvidState* st) {
    if (*(volatile int*)&st->done) return;
    extern __shared__ double su[];   // [rows_per_split] <= kMaxRowsPerSplit (32 KB)
    const int n0 = blockIdx.y * rows_per_split;
    const int nr = min(rows_per_split, N - n0);
    for (int i = threadIdx.x; i < nr; i += blockDim.x) su[i] = u[n0 + i];
    __syncthreads();
    const int k = blockIdx.x * kColThreads + threadIdx.x;
    if (k >= K) return;
    const double un = st->unorm;
    const float* col = W + (size_t)n0 * K + k;
    double acc = 0.0;
#pragma unroll 8
    for (int i = 0; i < nr; ++i) acc = fma(fabs((double)col[(size_t)i * K]), su[i], acc);
    part[(size_t)blockIdx.y * K + k] = acc / un;
}

// v[k] = sum_s part[s][k]; sigma = ||v||; convergence test
__global__ void __launch_bounds__(kFinThreads) svid_fin_kernel(const double* __restrict__ part,
                                                               int splits, int K, double* v,
                                                               double* red, SvidState* st) {
    if (*(volatile int*)&st->done) return;
    __shared__ double sm[kFinThreads / 32];
    const int k = blockIdx.x * kFinThreads + threadIdx.x;
    double s = 0.0;
    if (k < K) {
        for (int i = 0; i < splits; ++i) s += part[(size_t)i * K + k];
        v[k] = s;
    }
    double total;
    if (grid_sum_last(warp_sum_d(k < K ? s * s : 0.0), sm, kFinThreads / 32, red, &st->ticket_fin,
                      &total) &&
        threadIdx.x == 0) {
        const double sigma = sqrt(total);
        const int it = st->it + 1;
        st->it = it;
        st->vnorm = sigma;
        if (it >= st->max_iter || (it > 1 && fabs(sigma - st->prev) <= st->tol * sigma)) st->done = 1;
        st->prev = sigma;
    }
}

// a = sqrt(sigma) u_raw / ||u_raw||, b = sqrt(sigma) v / sigma; h = fp16(a), g = fp16(b)
__global__ void svid_out_kernel(const double* __restrict__ u, const double* __restrict__ v, int N,
                                int K, const SvidState* st, uint16_t* g, uint16_t* h, double* a_out,
                                double* b_out) {
    const double sigma = st->vnorm, r = sqrt(sigma), un = st->unorm;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N + K; i += gridDim.x * blockDim.x) {
        if (i < N) {
            const double a = r * (u[i] / un);
            h[i] = __half_as_ushort(__double2half(a));
            if (a_out) a_out[i] = a;
        } else {
            const int k = i - N;
            const double b = r * (v[k] / sigma);
            g[k] = __half_as_ushort(__double2half(b));
            if (b_out) b_out[k] = b;
        }
    }
}

}  // namespace

int svid_max_n() { return kMaxSplits * kMaxRowsPerSplit; }
size_t svid_workspace_bytes(int N, int K) { return svid_layout(N, K).total; }

// Host driver: iterations are queued in batches; after each batch the
// convergence flag is read back (the call synchronises the stream).
bl_status svid_run(const float* W, int N, int K, int max_iter, double tol, uint32_t* s1, uint16_t* g,
                   uint16_t* h, double* a, double* b, double* sigma, int* iters, void* workspace,
                   cudaStream_t s) {
    const SvidWs l = svid_layout(N, K);
    char* ws = static_cast<char*>(workspace);
    SvidState* st = reinterpret_cast<SvidState*>(ws + l.state);
    double* u = reinterpret_cast<double*>(ws + l.u);
    double* v = reinterpret_cast<double*>(ws + l.v);
    double* part = reinterpret_cast<double*>(ws + l.part);
    double* red = reinterpret_cast<double*>(ws + l.red);
    const size_t nwords = (size_t)N * (K / 32);
    svid_init_kernel<<<(K + 255) / 256, 256, 0, s>>>(v, K, st, tol, max_iter);
    svid_sign_kernel<<<(unsigned)((nwords + 255) / 256), 256, 0, s>>>(W, nwords, s1, st);
    if (cudaGetLastError() != cudaSuccess) return BL_ERR_CUDA;
    const dim3 col_grid((K + kColThreads - 1) / kColThreads, l.splits);
    SvidState hs;
    int queued = 0;
    // batches of 1, 2, 4, 8, 8, ...: few read-backs for fast convergence,
    // few idle launches after it
    for (int batch = 1; queued < max_iter; batch = batch < 8 ? 2 * batch : 8) {
        const int nb = std::min(batch, max_iter - queued);
        for (int i = 0; i < nb; ++i) {
            svid_row_kernel<<<(N + kRowWarps - 1) / kRowWarps, kRowWarps * 32, 0, s>>>(W, N, K, v, u,
                                                                                       red, st);
            svid_col_kernel<<<col_grid, kColThreads, (size_t)l.rows_per_split * 8, s>>>(
                W, N, K, u, part, l.rows_per_split, st);
            svid_fin_kernel<<<(K + kFinThreads - 1) / kFinThreads, kFinThreads, 0, s>>>(
                part, l.splits, K, v, red, st);
        }
        queued += nb;
        if (cudaGetLastError() != cudaSuccess ||
            cudaMemcpyAsync(&hs, st, sizeof(hs), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return BL_ERR_CUDA;
        if (hs.bad) return BL_ERR_INVALID_VALUE;
        if (hs.done) break;
    }
    svid_out_kernel<<<(N + K + 255) / 256, 256, 0, s>>>(u, v, N, K, st, g, h, a, b);
    if (cudaGetLastError() != cudaSuccess ||
        cudaMemcpyAsync(&hs, st, sizeof(hs), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return BL_ERR_CUDA;
    if (sigma) *sigma = hs.vnorm;
    if (iters) *iters = hs.it;
    return BL_OK;
}

}  // namespace bl
