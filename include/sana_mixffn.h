/* C ABI of the Mix-FFN of the Linear DiT block, on sm_100a.
 *
 * "Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
 * Transformers", section 2.2: an inverted residual block, a 3x3 depthwise
 * convolution and a GLU take the place of the MLP FFN; section 2.3: the
 * convolution's zero padding is what carries position (no positional encoding).
 * "SANA 1.5", section "Model architecture": C = 2240, FFN width F = 5600.
 *
 * Tokens n = y * Ws + x of a row-major (Hs, Ws) latent grid, N = Hs * Ws:
 *   U  = X W1 + b1                                 1x1 expand, C -> 2F
 *   Cv[y, x, c] = bdw[c] + sum_{i, j in 0..2} wdw[c][i][j] U[y + i - 1, x + j - 1, c]
 *                                                  (cross-correlation; U is zero
 *                                                  outside the grid)
 *   Hg = Cv[:, :F] * gate(Cv[:, F:])               GLU: value half times the gate of
 *                                                  the second half
 *   Y  = Hg W2 + b2                                1x1 project, F -> C
 * gate(z) = sigmoid(z) = 1 / (1 + exp(-z)) (the GLU's definition) or SiLU, z *
 * sigmoid(z).  Biases are optional (NULL: none).
 *
 * Conventions (as in sana_linattn.h): pointers are caller-owned device memory;
 * the library allocates nothing, does not synchronise and launches on `stream`.
 * Activations are bf16 (B, N, channels) row-major, contiguous, 16-byte aligned;
 * weights of the 1x1 convolutions are bf16 row-major (in, out); the depthwise
 * weights are fp32 [2F][3][3] and all biases fp32.  Every sum accumulates in
 * fp32; U and Hg are stored in bf16 between the kernels.  Results are bitwise
 * reproducible for a fixed shape and device.  Violations return a status and
 * launch nothing; launch failures return SANA_ECUDA; a bounded device-side wait
 * that gives up is reported by sana_linattn_device_error. */
#ifndef SANA_MIXFFN_H
#define SANA_MIXFFN_H

#include "sana_linattn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { SANA_GATE_SIGMOID = 0, SANA_GATE_SILU = 1 } sana_gate;

/* D[M][Nc] = A[M][K] W[K][Nc] (+ bias[Nc]) with bf16 A, W, D and fp32
 * accumulation on the tensor cores (tcgen05 UMMA, TMA-fed, each UMMA spread over a
 * pair of SMs: clusters of two CTAs with 256 x 256 tiles).  Both 1x1
 * convolutions of the Mix-FFN are this call.  K and Nc must be positive
 * multiples of 8 (TMA row pitch), M >= 0 (0: nothing launched), M < 2^31;
 * A, W, D 16-byte aligned, bias 4-byte aligned or NULL; D must not overlap A, W
 * or bias.  SANA_EUNSUPPORTED: shared memory or TMEM not available. */
SANA_API int sana_gemm_bias_bf16(const void* A, const void* W, const float* bias, void* D,
                                 int64_t M, int K, int Nc, cudaStream_t stream);

/* Hg = GLU(depthwise 3x3 convolution of u): u (B, Hs*Ws, 2F) bf16, wdw
 * [2F][3][3] fp32, bdw [2F] fp32 or NULL, h (B, Hs*Ws, F) bf16; gate is a
 * sana_gate.  F must be a positive multiple of 8; B, Hs, Ws >= 0 (any 0: nothing
 * launched), Hs, Ws < 2^24, B <= 65535.  h must not overlap u. */
SANA_API int sana_mixffn_dwconv_glu(const void* u, const float* wdw, const float* bdw, void* h,
                                    int64_t B, int Hs, int Ws, int F, int gate,
                                    cudaStream_t stream);

/* Bytes of device workspace sana_mixffn_forward needs: U (B*N x 2F bf16) then Hg
 * (B*N x F bf16), each 256-byte aligned.  0 for an empty or invalid shape. */
SANA_API size_t sana_mixffn_workspace_bytes(int64_t B, int Hs, int Ws, int C, int F);

/* The whole Mix-FFN: x (B, Hs*Ws, C) bf16 -> y (B, Hs*Ws, C) bf16, with W1 (C, 2F)
 * and W2 (F, C) bf16 row-major, b1 [2F], wdw [2F][3][3], bdw [2F], b2 [C] fp32
 * (biases NULL allowed).  Three launches on `stream`: the expand GEMM into U, the
 * depthwise convolution + GLU into Hg, the project GEMM into y.  C and F positive
 * multiples of 8; the workspace (256-byte aligned, at least
 * sana_mixffn_workspace_bytes) must not overlap any argument; y must not overlap
 * x or the weights. */
SANA_API int sana_mixffn_forward(const void* x, const void* W1, const float* b1,
                                 const float* wdw, const float* bdw, const void* W2,
                                 const float* b2, void* y, int64_t B, int Hs, int Ws, int C,
                                 int F, int gate, void* workspace, size_t ws_bytes,
                                 cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SANA_MIXFFN_H */
