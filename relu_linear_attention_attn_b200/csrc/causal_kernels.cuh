// The prefix (causal) form of Eq. (1) ("Sana: Efficient High-Resolution Image
// Synthesis with Linear Diffusion Transformers": linear attention as a cumulative
// prefix sum, the explainer page's O(N) form), token n seeing keys j <= n:
//     O_n = phi(Q_n) S_n[:, :D] / (phi(Q_n) S_n[:, D] + eps),
//     S_n = sum_{j <= n} phi(K_j)^T [V_j | 1].
// Chunked over L = kCausalChunk tokens (CUDA-core kernels):
//   1. kv_partial_simt with tps = L: the state of each chunk alone,
//   2. causal_scan: an exclusive prefix sum over the chunks of each (b, h), in
//      place and in chunk order (reproducible), so chunk c holds sum_{c' < c},
//   3. causal_apply_simt: per chunk, the prefix state applied to every query plus
//      the masked quadratic form inside the chunk:
//        num_n = phi(Q_n) P_c + sum_{j in chunk, j <= n} (phi(Q_n).phi(K_j)) [V_j | 1].
#pragma once

#include "sana_common.cuh"

namespace sana {

constexpr int kCausalChunk = 128;
constexpr int kRowPad = 36;

// Exclusive prefix over chunks: grid B * H, 256 threads; part[bh][c] becomes
// sum_{c' < c} part[bh][c'] (the first chunk's becomes zero).
__global__ void __launch_bounds__(256)
causal_scan(float* __restrict__ part, int S)
{
    float* p = part + (int64_t)blockIdx.x * S * kStateFloats;
    for (int i = threadIdx.x; i < kStateFloats; i += blockDim.x) {
        float run = 0.f;
        for (int c = 0; c < S; ++c) {
            const float x = p[(int64_t)c * kStateFloats + i];
            p[(int64_t)c * kStateFloats + i] = run;
            run += x;
        }
    }
}

// The feature map of one head's 32 values (fp32 result, not rounded).
__device__ __forceinline__ void phi32(float* x, const float* g, float eps, bool norm) {
    if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < kD; ++i) ss = fmaf(x[i], x[i], ss);
        const float r = rsqrtf(ss * (1.f / kD) + eps);
#pragma unroll
        for (int i = 0; i < kD; ++i) x[i] = fmaxf(__ldg(g + i) * (x[i] * r), 0.f);
    } else {
#pragma unroll
        for (int i = 0; i < kD; ++i) x[i] = fmaxf(x[i], 0.f);
    }
}

// grid (ceil(N / L), H, B), L threads: thread t takes token c*L + t.
template <typename T>
__global__ void __launch_bounds__(kCausalChunk)
causal_apply_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const float* __restrict__ gq, const float* __restrict__ gk,
                  const float* __restrict__ pre, T* __restrict__ out, int64_t N, int H, int S,
                  float eps, int norm)
{
    // phi(K) and V of the chunk; rows padded to 36 floats so they read as float4
    __shared__ __align__(16) float sK[kCausalChunk][kRowPad];
    __shared__ __align__(16) float sV[kCausalChunk][kRowPad];
    __shared__ float sP[kStateFloats];          // prefix state of the chunk
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
    const int64_t n = (int64_t)c * kCausalChunk + t;
    const bool live = n < N;
    const int64_t C = (int64_t)H * kD;
    const float* ps = pre + (((int64_t)b * H + h) * S + c) * kStateFloats;
    for (int i = t; i < kStateFloats; i += kCausalChunk) sP[i] = ps[i];
    float x[kD];
    const int64_t row = ((int64_t)b * N + n) * C + (int64_t)h * kD;
    if (live) {
#pragma unroll
        for (int i = 0; i < kD; i += 8) load8(k + row + i, x + i);
        phi32(x, gk + h * kD, eps, norm != 0);
#pragma unroll
        for (int i = 0; i < kD; ++i) sK[t][i] = x[i];
#pragma unroll
        for (int i = 0; i < kD; i += 8) load8(v + row + i, x + i);
#pragma unroll
        for (int i = 0; i < kD; ++i) sV[t][i] = x[i];
    } else {
#pragma unroll
        for (int i = 0; i < kD; ++i) { sK[t][i] = 0.f; sV[t][i] = 0.f; }
    }
    float fq[kD];
    if (live) {
#pragma unroll
        for (int i = 0; i < kD; i += 8) load8(q + row + i, fq + i);
        phi32(fq, gq + h * kD, eps, norm != 0);
    } else {
#pragma unroll
        for (int i = 0; i < kD; ++i) fq[i] = 0.f;
    }
    __syncthreads();
    float num[kDP];
#pragma unroll
    for (int e = 0; e < kDP; ++e) num[e] = 0.f;
#pragma unroll 4
    for (int d = 0; d < kD; ++d) {
        const float a = fq[d];
#pragma unroll
        for (int e = 0; e < kDP; ++e) num[e] = fmaf(a, sP[d * kDP + e], num[e]);
    }
    for (int j = 0; j <= t; ++j) {               // keys of this chunk up to the query
        const float4* kr = reinterpret_cast<const float4*>(sK[j]);
        const float4* vr = reinterpret_cast<const float4*>(sV[j]);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int d4 = 0; d4 < kD / 4; ++d4) {
            const float4 kk = kr[d4];
            a0 = fmaf(fq[4 * d4 + 0], kk.x, a0);
            a1 = fmaf(fq[4 * d4 + 1], kk.y, a1);
            a0 = fmaf(fq[4 * d4 + 2], kk.z, a0);
            a1 = fmaf(fq[4 * d4 + 3], kk.w, a1);
        }
        const float a = a0 + a1;
#pragma unroll
        for (int e4 = 0; e4 < kD / 4; ++e4) {
            const float4 vv = vr[e4];
            num[4 * e4 + 0] = fmaf(a, vv.x, num[4 * e4 + 0]);
            num[4 * e4 + 1] = fmaf(a, vv.y, num[4 * e4 + 1]);
            num[4 * e4 + 2] = fmaf(a, vv.z, num[4 * e4 + 2]);
            num[4 * e4 + 3] = fmaf(a, vv.w, num[4 * e4 + 3]);
        }
        num[kD] += a;
    }
    if (!live) return;
    const float inv = 1.f / (num[kD] + eps);
    float o[kD];
#pragma unroll
    for (int e = 0; e < kD; ++e) o[e] = num[e] * inv;
#pragma unroll
    for (int i = 0; i < kD; i += 8) store8(out + row + i, o + i);
}

}  // namespace sana
