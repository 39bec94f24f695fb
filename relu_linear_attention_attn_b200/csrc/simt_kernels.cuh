// CUDA-core (FFMA) kernels for the two passes of Eq. (1) ("Sana: Efficient
// High-Resolution Image Synthesis with Linear Diffusion Transformers",
// section 2.1) with the per-head QK-RMSNorm of SANA-1.5 ("Model architecture",
// QK Norm bullet).  They serve the fp32 dtype and bf16 problems with more than
// 128 heads; bf16 up to 128 heads runs the tensor-core kernels.
//
//   pass 1  kv_partial_simt : split-N partial states  phi(K)^T [V | 1]
//   combine kv_combine      : fixed-order sum of the split partials
//   pass 2  apply_simt      : O = phi(Q) S[:, :D] / (phi(Q) S[:, D] + eps)
#pragma once

#include "sana_common.cuh"

namespace sana {

// Pass 1.  grid (S, H, B), 128 threads.  The CTA (s, h, b) reduces tokens
// [s*tps, min(N, (s+1)*tps)) of head h, batch b, into
// part[((b*H + h)*S + s)][D][D+1].
//   load role : thread t loads half (t & 1) of token (t >> 1) of a 64-token chunk,
//               normalises it with its partner (shuffle), applies gain and ReLU
//   FMA role  : thread t owns state row d = t >> 2, columns 8*(t & 3) .. +7, and
//               (for t & 3 == 0) the normaliser column.
template <typename T>
__global__ void __launch_bounds__(128)
kv_partial_simt(const T* __restrict__ k, const T* __restrict__ v,
                const float* __restrict__ gk, float* __restrict__ part,
                int64_t N, int H, int64_t ldk, int64_t ldv, int S, int64_t tps,
                float eps, int norm)
{
    __shared__ float sK[64][kDP];
    __shared__ float sV[64][kDP];
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    const int64_t n0 = (int64_t)s * tps;
    const int64_t n1 = min(N, n0 + tps);

    const int lt = tid >> 1, half = tid & 1;
    float g[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) g[i] = norm ? __ldg(gk + h * kD + half * 16 + i) : 1.f;

    const int d = tid >> 2, e0 = (tid & 3) * 8;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    float ks = 0.f;

    for (int64_t c0 = n0; c0 < n1; c0 += 64) {
        const int64_t n = c0 + lt;
        const bool live = n < n1;
        float kx[16], vx[16];
        if (live) {
            const T* kp = k + ((int64_t)b * N + n) * ldk + h * kD + half * 16;
            const T* vp = v + ((int64_t)b * N + n) * ldv + h * kD + half * 16;
            load8(kp, kx); load8(kp + 8, kx + 8);
            load8(vp, vx); load8(vp + 8, vx + 8);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) { kx[i] = 0.f; vx[i] = 0.f; }
        }
        if (norm) {
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) ss = fmaf(kx[i], kx[i], ss);
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            const float r = rsqrtf(ss * (1.f / kD) + eps);
#pragma unroll
            for (int i = 0; i < 16; ++i) kx[i] = fmaxf(g[i] * (kx[i] * r), 0.f);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) kx[i] = fmaxf(kx[i], 0.f);
        }
        if (!live) {
#pragma unroll
            for (int i = 0; i < 16; ++i) kx[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) { sK[lt][half * 16 + i] = kx[i]; sV[lt][half * 16 + i] = vx[i]; }
        __syncthreads();
        const int cnt = (int)min((int64_t)64, n1 - c0);
        for (int t = 0; t < cnt; ++t) {
            const float a = sK[t][d];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(a, sV[t][e0 + i], acc[i]);
            ks += a;
        }
        __syncthreads();
    }
    float* out = part + (((int64_t)b * H + h) * S + s) * kStateFloats;
#pragma unroll
    for (int i = 0; i < 8; ++i) out[d * kDP + e0 + i] = acc[i];
    if ((tid & 3) == 0) out[d * kDP + kD] = ks;
}

// Combine.  grid (B*H), 256 threads: kv[bh] = sum_{s=0..S-1} part[bh][s] in
// increasing s, so the result does not depend on scheduling.
__global__ void __launch_bounds__(256)
kv_combine(const float* __restrict__ part, float* __restrict__ kv, int S)
{
    const int64_t bh = blockIdx.x;
    const float* p = part + bh * (int64_t)S * kStateFloats;
    for (int i = threadIdx.x; i < kStateFloats; i += blockDim.x) {
        float acc = 0.f;
        for (int j = 0; j < S; ++j) acc += p[(int64_t)j * kStateFloats + i];
        kv[bh * kStateFloats + i] = acc;
    }
}

// Pass 2.  grid (ceil(N/128), H, B), 128 threads, one token per thread.
template <typename TI, typename TO>
__global__ void __launch_bounds__(128)
apply_simt(const TI* __restrict__ q, const float* __restrict__ gq,
           const float* __restrict__ kv, TO* __restrict__ out,
           int64_t N, int H, int64_t ldq, int64_t ldo, float eps, int norm)
{
    __shared__ float sKV[kStateFloats];
    const int h = blockIdx.y, b = blockIdx.z;
    const float* st = kv + ((int64_t)b * H + h) * kStateFloats;
    for (int i = threadIdx.x; i < kStateFloats; i += blockDim.x) sKV[i] = st[i];
    __syncthreads();
    const int64_t n = (int64_t)blockIdx.x * 128 + threadIdx.x;
    if (n >= N) return;

    float x[kD];
    const TI* qp = q + ((int64_t)b * N + n) * ldq + h * kD;
#pragma unroll
    for (int j = 0; j < kD; j += 8) load8(qp + j, x + j);
    if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < kD; ++j) ss = fmaf(x[j], x[j], ss);
        const float r = rsqrtf(ss * (1.f / kD) + eps);
#pragma unroll
        for (int j = 0; j < kD; ++j) x[j] = fmaxf(__ldg(gq + h * kD + j) * (x[j] * r), 0.f);
    } else {
#pragma unroll
        for (int j = 0; j < kD; ++j) x[j] = fmaxf(x[j], 0.f);
    }
    float o[kDP];
#pragma unroll
    for (int e = 0; e < kDP; ++e) o[e] = 0.f;
#pragma unroll
    for (int dd = 0; dd < kD; ++dd) {
        const float a = x[dd];
#pragma unroll
        for (int e = 0; e < kDP; ++e) o[e] = fmaf(a, sKV[dd * kDP + e], o[e]);
    }
    const float den = o[kD] + eps;
#pragma unroll
    for (int e = 0; e < kD; ++e) o[e] = o[e] / den;
    TO* op = out + ((int64_t)b * N + n) * ldo + h * kD;
#pragma unroll
    for (int j = 0; j < kD; j += 8) store8(op + j, o + j);
}

}  // namespace sana
