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
// Per query and head the chunk costs about 1,056 FMA for the prefix state and
// 65 (L + 1) / 2 on average for the quadratic form, so L = 64 balances the two
// against the chunk states' traffic (one 4,224-byte state per chunk and head).
// The inner products run as packed fp32 pairs (fma.rn.f32x2).
#pragma once

#include "f32x2.cuh"
#include "sana_common.cuh"

namespace sana {

constexpr int kCausalChunk = 64;
constexpr int kRowPad = 36;
constexpr int kStateRowPad = 34;     // prefix-state rows padded to an even length

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
    __shared__ __align__(16) float sP[kD][kStateRowPad];   // prefix state of the chunk
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
    const int64_t n = (int64_t)c * kCausalChunk + t;
    const bool live = n < N;
    const int64_t C = (int64_t)H * kD;
    const float* ps = pre + (((int64_t)b * H + h) * S + c) * kStateFloats;
    for (int i = t; i < kStateFloats; i += kCausalChunk) sP[i / kDP][i % kDP] = ps[i];
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
    // num2[i]: value columns 2i, 2i + 1; numz: the normaliser column
    uint64_t num2[kD / 2], fq2[kD / 2];
#pragma unroll
    for (int i = 0; i < kD / 2; ++i) {
        num2[i] = 0ull;
        fq2[i] = pack2(fq[2 * i], fq[2 * i + 1]);
    }
    float numz = 0.f;
#pragma unroll 4
    for (int d = 0; d < kD; ++d) {
        const uint64_t a2 = pack2(fq[d], fq[d]);
        const float2* pr = reinterpret_cast<const float2*>(sP[d]);
#pragma unroll
        for (int i = 0; i < kD / 2; ++i) {
            const float2 pp = pr[i];
            num2[i] = fma2(a2, pack2(pp.x, pp.y), num2[i]);
        }
        numz = fmaf(fq[d], sP[d][kD], numz);
    }
    for (int j = 0; j <= t; ++j) {               // keys of this chunk up to the query
        const float4* kr = reinterpret_cast<const float4*>(sK[j]);
        const float4* vr = reinterpret_cast<const float4*>(sV[j]);
        uint64_t acc = 0ull;                     // even and odd channels of the dot product
#pragma unroll
        for (int d4 = 0; d4 < kD / 4; ++d4) {
            const float4 kk = kr[d4];
            acc = fma2(fq2[2 * d4], pack2(kk.x, kk.y), acc);
            acc = fma2(fq2[2 * d4 + 1], pack2(kk.z, kk.w), acc);
        }
        float a0, a1;
        unpack2(acc, a0, a1);
        const float a = a0 + a1;
        const uint64_t aa = pack2(a, a);
#pragma unroll
        for (int e4 = 0; e4 < kD / 4; ++e4) {
            const float4 vv = vr[e4];
            num2[2 * e4] = fma2(aa, pack2(vv.x, vv.y), num2[2 * e4]);
            num2[2 * e4 + 1] = fma2(aa, pack2(vv.z, vv.w), num2[2 * e4 + 1]);
        }
        numz += a;
    }
    if (!live) return;
    const float inv = 1.f / (numz + eps);
    float o[kD];
#pragma unroll
    for (int i = 0; i < kD / 2; ++i) {
        float lo, hi;
        unpack2(num2[i], lo, hi);
        o[2 * i] = lo * inv;
        o[2 * i + 1] = hi * inv;
    }
#pragma unroll
    for (int i = 0; i < kD; i += 8) store8(out + row + i, o + i);
}

}  // namespace sana
