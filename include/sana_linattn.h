/*
 * sana_linattn.h -- C ABI of the B200 (sm_100a) library for SANA's multi-head
 * ReLU linear attention with QK-RMSNorm.
 *
 * The operation (Eq. (1) of "Sana: Efficient High-Resolution Image Synthesis
 * with Linear Diffusion Transformers", section 2.1, with the QK-Norm of "SANA
 * 1.5: Efficient Scaling of Training-Time and Inference-Time Compute in Linear
 * Diffusion Transformer", section "Model architecture"):
 *
 *   phi(x)  = ReLU(g * x / sqrt(mean_d(x_d^2) + eps))  per token and head
 *             (the mean over the head's D channels; with the norm off,
 *             phi(x) = ReLU(x))
 *   S_{b,h} = sum_n phi(K_{b,n,h})^T [V_{b,n,h} | 1]    (D x (D+1), fp32)
 *   O_{b,n,h} = phi(Q_{b,n,h}) S[:, :D] / (phi(Q_{b,n,h}) S[:, D] + eps)
 *
 * The sums run over all N tokens (non-causal).  The same eps is the RMSNorm
 * epsilon and the denominator's.  Accumulation is fp32 throughout, so sums far
 * beyond the fp16 range (the overflow the SANA-1.5 page attributes to growing
 * attention sums) stay finite.
 *
 * Conventions shared by every entry point:
 *   - Tensors are row-major (B, N, C) with C = H * D and channel c = h*D + d.
 *     D = C / H must be 32 (anything else returns SANA_EUNSUPPORTED).
 *   - Every pointer is DEVICE memory owned by the caller (the library never
 *     allocates, frees or keeps a pointer after the call returns).
 *   - q, k, v, x, Wqkv and out must be 16-byte aligned; the workspace 256-byte
 *     aligned; gains 4-byte aligned.  out must not overlap any input.
 *   - gq == NULL && gk == NULL switches the RMSNorm off (phi = ReLU); gains are
 *     fp32 vectors of length C.  Passing exactly one of them is SANA_EINVAL.
 *   - Work is enqueued on `stream` asynchronously; the call never synchronises.
 *     Argument errors are returned before anything is enqueued.  A failed
 *     launch returns SANA_ECUDA; faults during execution surface at the
 *     caller's next synchronisation, as for any CUDA kernel.
 *   - B == 0 or N == 0 is an empty problem: nothing is launched and SANA_OK is
 *     returned (sana_linattn_kv_state then zero-fills its state output).
 *   - For a given shape, dtype and device two calls give bitwise-identical
 *     results: split counts are a fixed function of the shape and partial sums
 *     are combined in a fixed order.
 */
#ifndef SANA_LINATTN_H
#define SANA_LINATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define SANA_API __attribute__((visibility("default")))
#else
#define SANA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SANA_OK = 0,
    SANA_EINVAL = -1,        /* bad shape, NULL pointer, eps < 0, overlap, dtype   */
    SANA_EALIGN = -2,        /* a pointer violates its alignment requirement       */
    SANA_EUNSUPPORTED = -3,  /* well-formed but not supported (D != 32, too large) */
    SANA_EWORKSPACE = -4,    /* workspace NULL or smaller than the queried size    */
    SANA_ECUDA = -5,         /* a CUDA launch or runtime call failed               */
    SANA_ESCRATCH = -6       /* too large for sana_linattn_forward_noalloc's scratch */
} sana_status;

typedef enum {
    SANA_BF16 = 0,           /* bf16 inputs and output, fp32 arithmetic            */
    SANA_F32 = 1             /* fp32 inputs and output, fp32 arithmetic            */
} sana_dtype;

/* Bytes of device workspace that sana_linattn_forward (fused == 0),
 * sana_linattn_kv_state (fused == 0), sana_linattn_qkv_fused and
 * sana_linattn_qkv_fused_w8a8 (fused == 1) or sana_linattn_forward_causal
 * (fused == 2) needs for this shape.  Returns 0 for an invalid or empty shape. */
SANA_API size_t sana_linattn_workspace_bytes(int64_t B, int64_t N, int C, int H, int fused);

/* Eq. (1) end to end on projected q, k, v.
 * q, k, v, out: (B, N, C) in `dtype`.  gq, gk: fp32 [C] or both NULL.
 * workspace: at least sana_linattn_workspace_bytes(B, N, C, H, 0) bytes; its
 * contents on entry do not matter and are garbage on exit.
 * bf16 with C <= 4096 runs on the tensor cores: short problems (N <= 1024 and at
 * most 400 CTAs of 128 tokens x 4 heads, e.g. the 1024px latent at batch 1 to 3)
 * as ONE launch of thread-block clusters that reduce the state among their CTAs
 * through distributed shared memory; everything else as two persistent passes
 * (the state, then its application).  fp32 and wider problems run CUDA-core
 * kernels.  Either way the result is a fixed function of the inputs (reductions
 * in a fixed order: bitwise reproducible). */
SANA_API int sana_linattn_forward(const void* q, const void* k, const void* v,
                         const float* gq, const float* gk, void* out,
                         int64_t B, int64_t N, int C, int H, float eps,
                         sana_dtype dtype, void* workspace, size_t ws_bytes,
                         cudaStream_t stream);

/* How many kernels sana_linattn_forward (and sana_linattn_forward_noalloc) launch
 * for this shape and dtype: 1 (one cluster launch, short problems on the tensor
 * cores), 2 (the two persistent passes) or 3 (the CUDA-core path); 0 for an empty
 * shape (B or N zero); a negative sana_status for an invalid one.  Host only. */
SANA_API int sana_linattn_forward_kernels(int64_t B, int64_t N, int C, int H, sana_dtype dtype);

/* The prefix (causal) form of Eq. (1): the explainer page of the Sana notes
 * describes linear attention as a cumulative prefix sum; here token n sees keys
 * j <= n only:
 *   O_n = phi(Q_n) S_n[:, :D] / (phi(Q_n) S_n[:, D] + eps),
 *   S_n = sum_{j <= n} phi(K_j)^T [V_j | 1].
 * Arguments, dtypes, layouts and errors as for sana_linattn_forward; workspace:
 * at least sana_linattn_workspace_bytes(B, N, C, H, 2) bytes (the states of
 * every 128-token chunk of every (b, h) and their prefixes on the tensor-core path
 * (bf16, C <= 4096, gains 16-byte aligned); one fp32 state per 64-token chunk on
 * the CUDA-core path).  Chunk states are combined in chunk order, so results are
 * reproducible. */
SANA_API int sana_linattn_forward_causal(const void* q, const void* k, const void* v,
                                         const float* gq, const float* gk, void* out,
                                         int64_t B, int64_t N, int C, int H, float eps,
                                         sana_dtype dtype, void* workspace, size_t ws_bytes,
                                         cudaStream_t stream);

/* Gradients of sana_linattn_forward's output for training (the pages define
 * only the forward; the gradients follow from Eq. (1) and the feature map):
 * given dout = dL/dO (B, N, C), writes dq, dk, dv (B, N, C) in `dtype` and, with
 * the norm on, dgq, dgk = dL/dgq, dL/dgk (fp32 [C]; both NULL with the norm off,
 * when gq = gk = NULL).  Recomputes the forward state itself, the way
 * sana_linattn_forward forms it (for bf16 with C <= 4096 on the tensor cores,
 * phi(K) and V as bf16 operands, fp32 sums).  For bf16 with C <= 4096, N >= 128 and
 * gains 16-byte aligned (or none) the whole backward runs on the tensor cores:
 * dnum = dO / (den + eps) is rounded to bf16 as the operand of dphi(Q) and of the
 * gradient state [dS | dz], which pass 1 of the forward forms; otherwise (fp32,
 * shorter sequences, whose key gradients are small differences of O(1) terms, or
 * other gains) CUDA-core kernels with fp32 intermediates run.  All tensors
 * 16-byte aligned (gains and their gradients 4-byte); outputs must not overlap
 * inputs or each other.  workspace: at least
 * sana_linattn_backward_workspace_bytes(B, N, C, H) bytes.  Sums are formed in a
 * fixed order, so results are reproducible.  B == 0 or N == 0 zero-fills
 * dgq, dgk. */
SANA_API size_t sana_linattn_backward_workspace_bytes(int64_t B, int64_t N, int C, int H);
SANA_API int sana_linattn_backward(const void* q, const void* k, const void* v,
                                   const float* gq, const float* gk, const void* dout,
                                   void* dq, void* dk, void* dv, float* dgq, float* dgk,
                                   int64_t B, int64_t N, int C, int H, float eps,
                                   sana_dtype dtype, void* workspace, size_t ws_bytes,
                                   cudaStream_t stream);

/* sana_linattn_backward with the forward's state passed in, as a training step
 * holds it (sana_linattn_kv_state's output for the same k, v, gk, eps: kv (B, H, D,
 * D+1) fp32, 16-byte aligned, read only; it must not overlap the outputs or the
 * workspace).  The state is then not formed again: the same gradients, bit for bit,
 * one pass over k and v fewer.  kv NULL is SANA_EINVAL (for B, N > 0); everything
 * else as for sana_linattn_backward, whose workspace size applies. */
SANA_API int sana_linattn_backward_with_state(const void* q, const void* k, const void* v,
                                              const float* gq, const float* gk,
                                              const float* kv, const void* dout, void* dq,
                                              void* dk, void* dv, float* dgq, float* dgk,
                                              int64_t B, int64_t N, int C, int H, float eps,
                                              sana_dtype dtype, void* workspace,
                                              size_t ws_bytes, cudaStream_t stream);

/* The state half of Eq. (1) (the sums formed once and reused by every query,
 * section 2.1 of the Sana notes): kv (B, H, D, D+1) fp32 receives
 * S_{b,h}[d][e] = sum_n phi(K)[d] V[e] for e < D and S_{b,h}[d][D] =
 * sum_n phi(K)[d].  Because S is a plain sum over tokens, states of disjoint
 * token ranges add up to the state of their union (sequence sharding reduces
 * them with one sum all-reduce).  workspace as for sana_linattn_forward. */
SANA_API int sana_linattn_kv_state(const void* k, const void* v, const float* gk, float* kv,
                          int64_t B, int64_t N, int C, int H, float eps,
                          sana_dtype dtype, void* workspace, size_t ws_bytes,
                          cudaStream_t stream);

/* The two persistent passes of sana_linattn_forward as separate calls; issued
 * one after the other on the same stream they are exactly the forward wherever
 * the forward runs the two passes (same kernels, same plan, bit-identical
 * output), and other work may be enqueued between them.  For the short problems
 * that the forward runs as one cluster launch they still run the two passes; the
 * results then agree with the forward's to rounding (the state's partial sums
 * are added in another order).
 *   sana_linattn_forward_pass1: the split-N partial states of phi(K)^T [V | 1]
 *     (one per contiguous token range of every (b, h), a fixed function of B, N, H
 *     and the device) into `workspace`.
 *   sana_linattn_forward_pass2: sums each (b, h)'s partials in range order and
 *     applies the state to q, writing out.  Reads the partials pass 1 wrote into
 *     the same workspace for the same (B, N, C, H, eps, gains) on the same device.
 * bf16 with C <= 4096 only (the tensor-core path; SANA_EUNSUPPORTED otherwise).
 * workspace: at least sana_linattn_workspace_bytes(B, N, C, H, 0) bytes; not
 * touched by anything else between the two calls. */
SANA_API int sana_linattn_forward_pass1(const void* k, const void* v, const float* gk,
                                        int64_t B, int64_t N, int C, int H, float eps,
                                        void* workspace, size_t ws_bytes, cudaStream_t stream);
SANA_API int sana_linattn_forward_pass2(const void* q, const float* gq, void* out,
                                        int64_t B, int64_t N, int C, int H, float eps,
                                        void* workspace, size_t ws_bytes, cudaStream_t stream);

/* The query half of Eq. (1) with a given state:
 * out = phi(Q) kv[:, :D] / (phi(Q) kv[:, D] + eps).
 * q, out: (B, N, C) in `dtype`; kv: (B, H, D, D+1) fp32; gq: fp32 [C] or NULL
 * (norm off).  Needs no workspace. */
SANA_API int sana_linattn_apply(const void* q, const float* gq, const float* kv, void* out,
                       int64_t B, int64_t N, int C, int H, float eps,
                       sana_dtype dtype, cudaStream_t stream);

/* The variant fused with the QKV projection (section 7 of the Sana notes,
 * on-device deployment: ReLU(K)^T V fused with the QKV projection).
 * x: (B, N, C) bf16; Wqkv: (C, 3C) bf16 row-major, columns [0,C) project to Q,
 * [C,2C) to K and [2C,3C) to V, no bias.  The projected Q, K, V are kept in
 * fp32 until the norm (no intermediate rounding).  out: (B, N, C) bf16.
 * gq, gk: fp32 [C] or both NULL.  workspace: at least
 * sana_linattn_workspace_bytes(B, N, C, H, 1) bytes. */
SANA_API int sana_linattn_qkv_fused(const void* x, const void* Wqkv,
                           const float* gq, const float* gk, void* out,
                           int64_t B, int64_t N, int C, int H, float eps,
                           void* workspace, size_t ws_bytes, cudaStream_t stream);

/* The fused variant with a W8A8 prologue (section 7 of the Sana notes, on-device
 * deployment: linear layers in 8-bit weights and activations, attention in full
 * precision).  The pages leave the scale granularity open; this library uses
 * symmetric int8 with one scale per token of x and one per output channel of
 * Wqkv, as produced by sana_quantize_rows_i8 / sana_quantize_cols_i8:
 *     [Q | K | V][n, c] = (sum_k xq[n, k] Wq[k, c]) * sx[n] * sw[c]
 * with the integer sum exact (int32) and the scaling in fp32; the norm, feature
 * map and Eq. (1) then run exactly as in sana_linattn_qkv_fused.
 * xq: (B, N, C) int8, 16-byte aligned; sx: fp32 [B * N]; Wq: (C, 3C) int8
 * row-major, columns [Q | K | V], 16-byte aligned; sw: fp32 [3C]; gq, gk: fp32
 * [C] or both NULL; out: (B, N, C) bf16.  workspace: at least
 * sana_linattn_workspace_bytes(B, N, C, H, 1) bytes.  Errors as for
 * sana_linattn_qkv_fused; out must not overlap any input. */
SANA_API int sana_linattn_qkv_fused_w8a8(const int8_t* xq, const float* sx,
                                         const int8_t* Wq, const float* sw,
                                         const float* gq, const float* gk, void* out,
                                         int64_t B, int64_t N, int C, int H, float eps,
                                         void* workspace, size_t ws_bytes,
                                         cudaStream_t stream);

/* Symmetric int8 quantisation of each row of x (rows, cols) in `dtype`
 * (row-major, cols % 8 == 0, x 16-byte aligned for bf16 / 32 for fp32, xq
 * 8-byte aligned): scales[r] = max_c |x[r, c]| / 127 (fp32, IEEE division) and
 * xq[r, c] = round_half_even(x[r, c] / scales[r]) in fp32, clamped to
 * [-127, 127]; an all-zero row gets scale 0 and zero codes.  xq and scales are
 * caller-owned device memory and must not overlap x or each other. */
SANA_API int sana_quantize_rows_i8(const void* x, sana_dtype dtype, int8_t* xq,
                                   float* scales, int64_t rows, int cols,
                                   cudaStream_t stream);

/* The same per column of a (K, cols) row-major matrix (e.g. Wqkv with
 * cols = 3C): scales[c] = max_k |w[k, c]| / 127, wq[k, c] = round_half_even(
 * w[k, c] / scales[c]) clamped to [-127, 127]. */
SANA_API int sana_quantize_cols_i8(const void* w, sana_dtype dtype, int8_t* wq,
                                   float* scales, int64_t K, int cols,
                                   cudaStream_t stream);

/* sana_linattn_forward without a caller-provided workspace, for callers that
 * cannot allocate device memory: code running inside a CUDA-graph capture or a
 * framework hook where cudaMalloc is forbidden, allocators that must not be
 * re-entered, or hosts whose memory budget is fixed up front.  The paper has no
 * counterpart; this is a library convenience.
 *
 * Same arguments, kernels, plan and results as sana_linattn_forward, minus the
 * workspace.  Its scratch is a 16 MiB array in the library's own device memory,
 * which every GPU that loads the library holds until the process exits.  The
 * call allocates nothing and frees nothing.
 *   - Problems whose workspace (sana_linattn_workspace_bytes(B, N, C, H, 0))
 *     exceeds 16 MiB return SANA_ESCRATCH; 2048px B=8 and 4096px B=2 at
 *     C = 2240 fit.
 *   - The first call on a device looks up the array's device address with the
 *     device current (cudaGetSymbolAddress) and keeps it for the life of the
 *     process; make that first call before any stream capture.  The kept
 *     address, like the library's other per-device set-up, does not survive
 *     cudaDeviceReset or the teardown of the device's primary context: do not
 *     call the library across one.
 *   - Every call shares the one array and leaves its contents behind; the
 *     forward path writes every scratch byte before reading it, so stale
 *     contents never matter.  Calls that overlap on the GPU (different streams,
 *     no ordering between them) race on the array: serialise them. */
SANA_API int sana_linattn_forward_noalloc(const void* q, const void* k, const void* v,
                                          const float* gq, const float* gk, void* out,
                                          int64_t B, int64_t N, int C, int H, float eps,
                                          sana_dtype dtype, cudaStream_t stream);

/* Device-side error word of the current device.  The tensor-core kernels bound
 * every wait (about 2 s); a wait that gives up records an error code (1 = wait
 * timeout) and the place it gave up (`site`), and the kernel winds down instead
 * of hanging.  Reads the word into *code and *site (either may be NULL) and
 * clears it when `clear` is non-zero.  Synchronous: call it after the work of
 * interest has been synchronised.  Returns SANA_OK or SANA_ECUDA. */
SANA_API int sana_linattn_device_error(int* code, int* site, int clear);

/* Self-test of the bounded waits: enqueues one kernel whose single thread waits
 * on an mbarrier that nothing arrives on.  After `limit_us` microseconds (at most
 * 10 s) the wait gives up and records code 1 (wait timeout) at site 999 in the
 * device error word (see sana_linattn_device_error); the kernel then exits and
 * the context stays usable.  Returns SANA_EINVAL for a limit out of range. */
SANA_API int sana_linattn_selftest_wait_timeout(int64_t limit_us, cudaStream_t stream);

/* Self-test of the launch-error path: enqueues a launch that the CUDA runtime
 * rejects before anything reaches the GPU (one block of 2048 threads, above the
 * per-block limit) and returns the status the library reports for it, SANA_ECUDA,
 * as every entry point does for a failed launch.  The error is not sticky: the
 * context stays usable and later calls succeed. */
SANA_API int sana_linattn_selftest_launch_failure(cudaStream_t stream);

/* Static description of a status code (never NULL). */
SANA_API const char* sana_linattn_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* SANA_LINATTN_H */
