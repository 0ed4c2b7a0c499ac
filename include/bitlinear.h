/*
 * bitlinear.h -- C ABI of libbitlinear.so: the forward pass of the two
 * extreme-low-bit linear layers that replace nn.Linear, on NVIDIA B200
 * (sm_100a).
 *
 *   BitLinear (BitNet b1.58 page, "微软、国科大开启1Bit时代：大模型转三进制，速度快4倍能耗降至1/41",
 *   section "BitNet b1.58 介绍"): ternary weights {-1, 0, +1}, activations
 *   quantised per token to 8 bits over the symmetric range [-127, 127] (no
 *   zero point), no bias.  The contraction is integer add/subtract
 *   (section "能耗"); the weights are stored 2 bits each (section "内存和延迟").
 *
 *   OneBit linear (OneBit page, "清华、哈工大把大模型压缩到了1bit，把大模型放在手机里跑的愿望就快要实现了！",
 *   section "1. 新的 1bit 结构"): a +-1 sign matrix S and two fp16 value
 *   vectors g (input side, length K) and h (output side, length N):
 *       y = ((x (.) g) . S^T) (.) h
 *   stored as one bit per sign (section "讨论与分析 / 1. 效率").
 *
 * Conventions for every entry point:
 *   - Tensors are row-major.  x is [M, K], y is [M, N], weights are [N, K]
 *     (nn.Linear orientation: y = x W^T).  fp16 values are passed as their
 *     IEEE binary16 bit patterns (uint16_t).
 *   - Every pointer is caller-owned DEVICE memory (cudaMalloc or torch),
 *     16-byte aligned.  The library allocates and frees nothing.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream)
 *     except the two packers, which synchronise `stream` to report invalid
 *     input values.
 *   - Overlap with the preceding kernel (programmatic dependent launch): the
 *     linear layers start streaming their PARAMETERS (w2 / s1, g, h) into
 *     on-chip memory while the kernel queued just before them on `stream` is
 *     still running, and read x (and the workspace) only after it completes.
 *     So parameters must not be written by the kernel immediately preceding a
 *     call on the same stream; activations may be.  (The packers synchronise,
 *     so packing and then calling is always safe.)
 *   - Shapes: M >= 0 and N >= 0 (0 is a no-op returning BL_OK); N % 16 == 0;
 *     K > 0 and K % 128 == 0.  Anything else returns BL_ERR_SHAPE without
 *     touching memory.
 *   - Errors are returned, never raised on the device: validation errors are
 *     detected before any launch; a failed launch returns BL_ERR_CUDA.
 *   - Fault injection for callers' error paths: when the environment variable
 *     BL_FAULT_INJECT is "cuda" or "timeout", every entry point that launches
 *     work returns BL_ERR_CUDA or BL_ERR_TIMEOUT right after validating its
 *     arguments, without any CUDA call (read on every call).
 *
 * Packed weight formats (bit-exact ABI; little-endian 32-bit words):
 *   w2 (ternary): uint32 [N][K/16]; weight (n,k) is the 2-bit field at bits
 *       2*(k%16) .. 2*(k%16)+1 of word [n][k/16], holding t+1
 *       (0 -> -1, 1 -> 0, 2 -> +1; 3 is never written).
 *   s1 (sign):    uint32 [N][K/32]; bit k%32 of word [n][k/32] is 1 iff
 *       sign(w[n][k]) = +1, with sign(+0) = sign(-0) = +1.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *bl_stream_t;

typedef enum {
    BL_OK = 0,
    BL_ERR_NULL = 1,          /* a required pointer is NULL */
    BL_ERR_SHAPE = 2,         /* M, N or K outside the rules above */
    BL_ERR_ALIGN = 3,         /* a pointer is not 16-byte aligned */
    BL_ERR_INVALID_VALUE = 4, /* an input value outside the format (packers) */
    BL_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
    BL_ERR_TIMEOUT = 6,       /* a bounded device-side wait expired */
    BL_ERR_WORKSPACE = 7,     /* workspace missing or smaller than required */
    BL_ERR_SCRATCH_LIMIT = 8  /* shape needs more than bl_ternary_linear_noalloc's fixed scratch */
} bl_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *bl_status_string(int status);

/* ABI version of this header (major * 100 + minor). */
int bl_abi_version(void);

/*
 * bl_pack_ternary -- pack ternary weights into the 2-bit w2 format above.
 * BitNet b1.58 page, "BitNet b1.58 介绍" (weights in {-1,0,1}) and "内存和延迟"
 * (2-bit storage).
 *   w  : int8 [N, K], each value in {-1, 0, 1}
 *   w2 : uint32 [N, K/16] output
 * Synchronises `stream`.  Any value outside {-1,0,1} -> BL_ERR_INVALID_VALUE
 * (w2 contents are then unspecified).  Concurrent packer calls on one device
 * share one error word: do not overlap them.
 */
bl_status bl_pack_ternary(const int8_t *w, int N, int K, uint32_t *w2, bl_stream_t stream);

/*
 * ob_pack_sign -- pack sign(W) into the 1-bit s1 format above.
 * OneBit page, "3. 通过知识蒸馏迁移原模型能力": after training, the parameters
 * after Sign() are saved and used directly at inference.
 *   w  : fp16 [N, K] (any finite values; +-0 packs as +1)
 *   s1 : uint32 [N, K/32] output
 * Synchronises `stream`.  A NaN input -> BL_ERR_INVALID_VALUE.
 */
bl_status ob_pack_sign(const uint16_t *w, int N, int K, uint32_t *s1, bl_stream_t stream);

/*
 * bl_quant_act -- per-token absmax activation quantisation.
 * BitNet b1.58 page, "BitNet b1.58 介绍": each token's activations are scaled
 * into [-Qb, Qb] (Qb = 127), removing the zero point.  Per token m, in IEEE
 * fp32 with round-to-nearest-even:
 *     amax = max_k |x[m,k]|;  inv = 127 / amax;
 *     q[m,k] = clamp(rne(x[m,k] * inv), -127, 127);  scale[m] = amax / 127
 * An all-zero token gives q = 0 and scale 0.  Non-finite inputs are
 * undefined.
 *   x     : fp16 [M, K]
 *   q     : int8 [M, K] output
 *   scale : fp32 [M] output
 */
bl_status bl_quant_act(const uint16_t *x, int M, int K, int8_t *q, float *scale,
                       bl_stream_t stream);

/* Workspace bytes bl_ternary_linear needs for this shape (a multiple of 256),
 * 0 for an invalid shape.  The size depends on the current device's SM count:
 * for prefill-sized M, when the (128-row x token) tiles would leave SMs idle
 * in the last round, it includes scratch (per-tile arrival counters and two
 * int32 partial tiles per SM) that lets the kernel share that round out in
 * k-stages.  Query it with the device that will run the call current. */
size_t bl_ternary_workspace_bytes(int M, int K, int N);

/*
 * bl_ternary_linear -- BitLinear forward, y = BitLinear(x; W, w_scale).
 * BitNet b1.58 page, "BitNet b1.58 介绍" (8-bit per-token activations, ternary
 * weights, no bias) and "能耗" (the contraction is INT8 additions):
 *     (q, s) = bl_quant_act(x)
 *     acc[m,n] = sum_k q[m,k] * t[n,k]                 (exact int32)
 *     y[m,n]   = fp16_rne( ((float)acc[m,n] * s[m]) * w_scale )
 *   x         : fp16 [M, K]
 *   w2        : packed ternary weights, uint32 [N, K/16]
 *   w_scale   : per-tensor weight scale (fp32, host value)
 *   y         : fp16 [M, N] output
 *   acc_out   : optional int32 [M, N] output of the accumulators (NULL = skip)
 *   workspace : device scratch of at least bl_ternary_workspace_bytes(M,K,N)
 *               bytes, used only during the call (stream-ordered); calls that
 *               overlap on the GPU need separate workspaces.
 * Invalid codes (3) in w2 are undefined behaviour (bl_pack_ternary never
 * writes them).
 */
bl_status bl_ternary_linear(const uint16_t *x, int M, int K, int N, const uint32_t *w2,
                            float w_scale, uint16_t *y, int32_t *acc_out,
                            void *workspace, size_t workspace_bytes, bl_stream_t stream);

/* Workspace bytes ob_linear needs for this shape (a multiple of 256), 0 for an
 * invalid shape; device-dependent like bl_ternary_workspace_bytes. */
size_t ob_workspace_bytes(int M, int K, int N);

/*
 * ob_linear -- OneBit linear forward.
 * OneBit page, "1. 新的 1bit 结构": y = ((x (.) g) . S^T) (.) h, with S = +-1
 * (packed s1) and fp16 value vectors g [K] and h [N].
 * The contraction is accumulated exactly in integers on a per-token
 * fixed-point image of x (.) g with 2^22 - 1 levels (error of that image
 * <= 2^-23 of the token's max |x (.) g| per element), contracted as three
 * int8 limbs, then scaled in fp32 and rounded once to fp16.  K <= 65536.
 *   x, y      : fp16 [M, K] in, fp16 [M, N] out
 *   s1        : packed signs, uint32 [N, K/32]
 *   g, h      : fp16 [K], fp16 [N]
 *   workspace : device scratch of at least ob_workspace_bytes(M,K,N) bytes
 *               (stream-ordered; overlapping calls need separate workspaces)
 */
bl_status ob_linear(const uint16_t *x, int M, int K, int N, const uint32_t *s1,
                    const uint16_t *g, const uint16_t *h, uint16_t *y,
                    void *workspace, size_t workspace_bytes, bl_stream_t stream);

/*
 * Two-plane binary layer (BiLLM page, "BiLLM: Pushing the Limit of
 * Post-Training Quantization for LLMs", section "方法细节：残差近似与最优断点拆分",
 * step 2, binary residual approximation): W ~ alpha_o (.) B_o + alpha_r (.) B_r,
 * both B = +-1, one scale per output row (the reading taken here), fp16
 * activations not quantised:
 *     y = fp16( alpha_o (.) (x B_o^T) + alpha_r (.) (x B_r^T) )
 * Stored form (a OneBit layer of 2N rows with g = 1):
 *   b2    : uint32 [2N, K/32] in the s1 format: rows 0..N-1 = B_o,
 *           rows N..2N-1 = B_r
 *   alpha : fp16 [2N]: alpha_o, then alpha_r
 * Arithmetic: each plane's contraction is exact in integers on the 23-bit
 * fixed-point image of x (as ob_linear with g = 1); each plane's product
 * s * Z * alpha is formed in fp32, the two are added in fp32 and rounded once
 * to fp16.  K <= 65536, N <= 2^23.
 */
size_t billm_workspace_bytes(int M, int K, int N);
bl_status billm_linear(const uint16_t *x, int M, int K, int N, const uint32_t *b2,
                       const uint16_t *alpha, uint16_t *y, void *workspace,
                       size_t workspace_bytes, bl_stream_t stream);

/*
 * billm_binarize -- the residual binarisation of a weight, on the device:
 * per row n, alpha_o = mean_k |W[n][k]|, B_o = sign(W[n]), R = W[n] - alpha_o
 * B_o, alpha_r = mean_k |R[k]|, B_r = sign(R) (sign(0) = +1), in fp64 (the
 * mean absolute value is the least-squares scale of a sign plane).  Writes b2
 * and alpha (fp16, rounded to nearest even) in the stored form above, and
 * optionally fp64 [N] copies of alpha_o and alpha_r (device, or NULL).
 * W is fp32 [N, K] (a NaN or inf -> BL_ERR_INVALID_VALUE).  Synchronises
 * `stream` like the packers, and shares their error word.
 */
bl_status billm_binarize(const float *W, int N, int K, uint32_t *b2, uint16_t *alpha,
                         double *alpha_o, double *alpha_r, bl_stream_t stream);

/* Workspace bytes ob_svid needs (a multiple of 256), 0 for an invalid shape. */
size_t ob_svid_workspace_bytes(int N, int K);

/*
 * ob_svid -- SVID initialisation of a OneBit layer from a trained weight.
 * OneBit page, "2. 基于 SVID 初始化量化模型": W ~ sign(W) (.) (a b^T) with a b^T
 * a rank-1 approximation of |W|; the layer's value vectors are then h = a and
 * g = b (the order swap of the same section makes ob_linear compute x W^T
 * with this approximation).  Reading taken here: the rank-1 factor is the
 * leading singular pair (sigma, u, v) of |W| (the SVD choice of "SVD or
 * NMF"), a = sqrt(sigma) u, b = sqrt(sigma) v, found by power iteration from
 * v = 1/sqrt(K):
 *     u = |W| v / || |W| v ||,  v' = |W|^T u,  sigma = ||v'||,  v = v' / sigma
 * stopping after iteration i >= 2 when |sigma_i - sigma_{i-1}| <= tol * sigma_i,
 * or after max_iter iterations.  Arithmetic in fp64 (u, v >= 0 throughout).
 *   W         : fp32 [N, K], finite (a NaN or inf -> BL_ERR_INVALID_VALUE)
 *   s1        : packed sign(W), uint32 [N, K/32] (the s1 format; +-0 -> +1)
 *   g, h      : fp16 [K] = fp16(b), fp16 [N] = fp16(a), round to nearest even
 *   a, b      : optional device fp64 [N], [K] copies of a and b (NULL: skipped)
 *   sigma     : optional HOST double: the last sigma
 *   iters     : optional HOST int: iterations run
 *   workspace : device scratch of at least ob_svid_workspace_bytes(N, K) bytes
 * N % 16 == 0 and N <= 524288, K % 128 == 0, max_iter >= 1, tol >= 0, else
 * BL_ERR_SHAPE.  Synchronises `stream` (it reads the convergence test back
 * every few iterations).  A weight-preparation call, not a layer forward.
 */
bl_status ob_svid(const float *W, int N, int K, int max_iter, double tol, uint32_t *s1,
                  uint16_t *g, uint16_t *h, double *a, double *b, double *sigma, int *iters,
                  void *workspace, size_t workspace_bytes, bl_stream_t stream);

/*
 * bl_ternary_linear_noalloc -- bl_ternary_linear for callers that cannot
 * allocate device memory.  (No counterpart on the pages: this is a calling
 * convention, not part of the method.)
 *
 * Some callers cannot call cudaMalloc or any other allocator where they run the
 * layer -- for example a plugin inside a host program that owns all device
 * memory and gives the plugin no allocator, or a latency-critical loop that
 * forbids allocation because cudaMalloc can block the whole device.  This entry
 * point takes no workspace: its scratch is a fixed array of
 * BL_NOALLOC_SCRATCH_BYTES compiled into the library, held by every GPU that
 * loads the library until the process exits.  It runs the same kernels as
 * bl_ternary_linear, chosen the same way by shape, and gives identical results
 * (same arguments minus the workspace); only the tensor-core path's balanced
 * last round is skipped when its scratch would not fit in the array.
 *   - Shapes needing more than the array, i.e. when
 *       round256(M*K) + round256(4*M) + round256(4*M) > BL_NOALLOC_SCRATCH_BYTES
 *     (M*K up to about 16.7 million int8 activations), return
 *     BL_ERR_SCRATCH_LIMIT before anything is launched.
 *   - It allocates nothing and frees nothing.
 *   - The first call on each device looks up that device's copy of the array
 *     (with the caller's device current); make that first call before any
 *     stream capture.
 *   - All calls on a device share the one array, and it keeps the previous
 *     call's contents (each call overwrites what it reads, so no clearing is
 *     needed).  Calls that may overlap on the GPU (different streams without
 *     ordering between them) race on it: order them, or use bl_ternary_linear
 *     with separate workspaces.
 */
#define BL_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
bl_status bl_ternary_linear_noalloc(const uint16_t *x, int M, int K, int N, const uint32_t *w2,
                                    float w_scale, uint16_t *y, int32_t *acc_out,
                                    bl_stream_t stream);

/*
 * Decode chains: the single-token (M = 1) forward of a whole list of layers
 * in ONE persistent launch -- the decode step of a stack of BitLinear or
 * OneBit layers (BitNet b1.58 page, "内存和延迟": at decode sizes the model's
 * time goes to its linear layers).  Per layer the arithmetic is exactly that
 * of bl_ternary_linear / ob_linear at M = 1 (same outputs, bit for bit).
 *
 * A layer's input is either given (x) or the output y of an EARLIER layer of
 * the list (src): the kernel then waits, inside the launch, until every part
 * of that layer's y is written.  Layers whose inputs do not depend on each
 * other overlap; the weights of later layers stream while earlier ones finish.
 *
 * The fused steps of a LLaMA-like block (the BitNet b1.58 page keeps RMSNorm
 * and SwiGLU around BitLinear) run inside the launch: an RMSNorm of a layer's
 * input (norm_w) and SwiGLU of two earlier outputs (src2) -- on rows of at
 * most 17920 (ternary) / 14336 (OneBit) elements.  Consecutive layers with the
 * same input (q, k, v; gate, up) prepare it once.
 *
 * Usage: describe the layers, call bl_chain_build once (it writes the device
 * descriptors, including TMA tensor maps, into the caller's `chain` buffer and
 * fills `plan`), then bl_chain_run as often as needed (graph-capturable: one
 * 4*n-byte memset node and one kernel node).  Weights, g, h and the pointers
 * are baked into the chain: rebuild it if any of them changes; the CONTENTS of
 * given inputs x may change between runs.  Runs of the same chain must not
 * overlap on the GPU (they share its counters).
 */
typedef struct {
    const uint16_t *x;     /* fp16 [K] input, or NULL when src >= 0 */
    int src;               /* -1: x is given; else the index (< this layer's) of
                              the layer whose output y is this layer's input
                              (its N must equal this layer's K) */
    int K, N;              /* K % 128 == 0, K <= 32768 (ternary) / 16384
                              (OneBit); N % 16 == 0 */
    const uint32_t *w;     /* packed weights: w2 [N, K/16] or s1 [N, K/32] */
    float w_scale;         /* ternary per-tensor weight scale */
    const uint16_t *g;     /* OneBit input value vector fp16 [K] (else NULL) */
    const uint16_t *h;     /* OneBit output value vector fp16 [N] (else NULL) */
    uint16_t *y;           /* fp16 [N] output */
    int32_t *acc_out;      /* optional int32 [N] accumulators (ternary), or NULL */
    int src2;              /* -1, or (with src >= 0) the index of a second earlier
                              layer: the input is then SwiGLU of the two outputs,
                              fp16(silu(y_src) * y_src2), silu(a) = a/(1+exp(-a)),
                              in fp64 (its N must equal this layer's K too) */
    const uint16_t *norm_w; /* NULL, or the fp16 [K] weight of an RMSNorm of the
                              input before it is quantised:
                              fp16((x * r) * norm_w), r = 1/sqrt(sum x^2/K + eps),
                              the sum of squares exact, the rest in fp64 */
    float norm_eps;        /* eps of that RMSNorm */
    uint16_t *swiglu_buf;  /* NULL, or (with src2 >= 0) a caller-owned fp16 [K]
                              device buffer: the SwiGLU is then evaluated once per
                              element, in the epilogue of the later of layers src
                              and src2, and stored here for this layer to read
                              (with NULL every CTA evaluates the whole row).  Same
                              results either way.  The chain writes it during
                              every run; give each SwiGLU layer its own buffer. */
} bl_chain_layer;

typedef struct {           /* filled by bl_chain_build; pass unchanged to bl_chain_run */
    int form;              /* 0 = BitLinear (ternary), 1 = OneBit */
    int n_layers;
    int sm_count;          /* the device's SM count the plan was made for */
    int kmax;              /* largest K of the chain */
    int slots;             /* weight-ring slots per CTA */
    int smem_bytes;        /* shared memory per CTA */
    int fused;             /* 1: some layer has an RMSNorm or SwiGLU prologue */
} bl_chain_plan;

/* Device bytes of the chain buffer for n_layers layers, 1 <= n_layers <= 2048
 * (0 if out of range). */
size_t bl_chain_bytes(int n_layers);

/*
 * bl_chain_build -- validate the layers and write the chain into `chain`
 * (caller-owned device memory, 256-byte aligned, >= bl_chain_bytes(n_layers)).
 * Synchronises `stream` (a host-to-device copy of the descriptors).  Errors:
 * BL_ERR_NULL / BL_ERR_ALIGN for pointers (16-byte alignment as everywhere),
 * BL_ERR_SHAPE for a shape or src outside the rules above or a layer too wide
 * for one launch (N/16 tiles > 16 per SM), BL_ERR_WORKSPACE if the buffer is
 * too small.  Make the device that will run the chain current.
 */
bl_status bl_chain_build(int form, const bl_chain_layer *layers, int n_layers, void *chain,
                         size_t chain_bytes, bl_chain_plan *plan, bl_stream_t stream);

/*
 * bl_chain_run -- one decode step over the chain, asynchronous on `stream`:
 * zeroes the chain's completion counters, then one cooperative launch of one
 * CTA per SM.  BL_ERR_SHAPE if `plan` does not match the current device.
 */
bl_status bl_chain_run(const bl_chain_plan *plan, const void *chain, bl_stream_t stream);

/* One host<->device copy of bl_chain_run_host: `bytes` bytes between a host
 * buffer (pinned, for the copy to be asynchronous) and a device buffer. */
typedef struct {
    const void *src;       /* host (inputs) or device (outputs) */
    void *dst;             /* device (inputs) or host (outputs) */
    size_t bytes;
} bl_copy;

/*
 * bl_chain_run_host -- one decode step with host buffers, all on `stream`:
 * copy each of the n_in inputs from host to the device buffers the chain reads
 * (its layers' given x), run the chain as bl_chain_run does, then copy each of
 * the n_out outputs (layers' y) back to host memory.  One cudaMemcpyAsync per
 * copy; nothing is synchronised (wait on `stream` before reading the outputs).
 * Steps on two streams over two chains (each with its own buffers) overlap one
 * step's copies with the other's kernel.  Errors: as bl_chain_run, plus
 * BL_ERR_NULL for a copy with bytes > 0 and a NULL pointer, BL_ERR_SHAPE for
 * negative counts.
 */
bl_status bl_chain_run_host(const bl_chain_plan *plan, const void *chain, const bl_copy *in,
                            int n_in, const bl_copy *out, int n_out, bl_stream_t stream);

/*
 * bl_prefill_plan -- diagnostic: how the tensor-core (prefill) path would run
 * a call of this shape on a device with `sm_count` SMs (form 0 = ternary,
 * 1 = OneBit, whose tiles hold two limb rows per token).  Fills plan[5]:
 *   plan[0] activation rows per tile, plan[1] ring stages per tile,
 *   plan[2] tiles, plan[3] tiles computed whole (one CTA each),
 *   plan[4] tiles shared out in k-stages over sm_count CTAs in a balanced
 *           last round (0: none).
 * Host arithmetic only (no CUDA call).  BL_ERR_NULL without plan,
 * BL_ERR_SHAPE for an invalid form or shape, M = 0, N = 0 or sm_count <= 0.
 */
bl_status bl_prefill_plan(int form, int M, int K, int N, int sm_count, int *plan);

/*
 * bl_debug_stall_next_launch -- test hook for the bounded device-side waits
 * (no counterpart on the pages).  The next launch in this process of the
 * streamed decode kernel (small M) or of the whole-tile tensor-core kernel
 * (prefill M) leaves the first pipeline stage of its CTA 0 unrequested, so a
 * wait in that CTA never sees its data: it gives up after wait_limit_ns
 * (instead of 2 s), the kernel records BL_ERR_TIMEOUT for bl_device_status,
 * lets every copy it did request land, frees its tensor memory and returns.
 * That launch's outputs are then incomplete.  Later launches are unaffected.
 * 0 cancels a pending stall.  Host-side only; not for concurrent use.
 */
bl_status bl_debug_stall_next_launch(unsigned long long wait_limit_ns);

/*
 * bl_device_status -- synchronise `stream` and report (then clear) any
 * device-side condition the library's kernels recorded since the last call:
 * BL_ERR_TIMEOUT if a bounded wait inside a kernel gave up, else BL_OK
 * (or BL_ERR_CUDA if the synchronisation itself failed).
 */
bl_status bl_device_status(bl_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* BITLINEAR_H */
