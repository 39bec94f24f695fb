// Backward of Eq. (1) ("Sana: Efficient High-Resolution Image Synthesis with
// Linear Diffusion Transformers", section 2.1) with the per-head QK-RMSNorm
// feature map; the pages define only the forward, the gradients are derived
// from it.  Per (b, h), with u = g * x * r, r = (mean_d x^2 + eps)^(-1/2),
// phi = ReLU(u), S = sum_j phi(K_j)^T V_j, z = sum_j phi(K_j):
//   den_i = phi(Q_i) . z + eps,   O_i = phi(Q_i) S / den_i
//   dnum_i = dO_i / den_i,        dden_i = -(dO_i . O_i) / den_i
//   dphi(Q_i) = dnum_i S^T + dden_i z
//   dS = sum_i phi(Q_i)^T dnum_i, dz = sum_i phi(Q_i) dden_i
//   dphi(K_j) = dS V_j + dz,      dV_j = phi(K_j) dS
// and through the feature map (du = dphi where u > 0, else 0):
//   dg[d] += du[d] x[d] r,  dx[c] = g[c] r du[c] - (r^3 x[c] / D) sum_d du[d] g[d] x[d].
//
// CUDA-core kernels (first version), all sums in fp32 and in a fixed order:
//   bwd_query_simt   one thread per (query token, head): dQ, [dnum | dden] rows,
//                    the CTA's gain partial
//   outer_partial_simt  split-N partials of phi(Q)^T [dnum | dden] (dS, dz),
//                    combined by kv_combine
//   bwd_key_simt     one thread per (key token, head): dK, dV, gain partial
//   gain_combine     gain partials summed over CTAs in order
// The 32 x 33 products run as packed fp32 pairs (fma.rn.f32x2) on state rows
// staged in shared memory with an even pitch.
#pragma once

#include "f32x2.cuh"
#include "sana_common.cuh"

namespace sana {

constexpr int kBwdTile = 128;      // tokens per CTA of the per-token kernels
constexpr int kGrow = kDP;         // [dnum | dden] floats per token-head
constexpr int kSPitch = kDP + 1;   // shared-memory pitch of a state row (even)

// A (D, D+1) state into shared memory rows of pitch kSPitch.
__device__ __forceinline__ void stage_state(const float* st, float (*sS)[kSPitch], int t,
                                            int nthreads) {
    for (int i = t; i < kStateFloats; i += nthreads) sS[i / kDP][i % kDP] = st[i];
}

// y[e] = sum_d a[d] S[d][e] for e < D (packed pairs), and the normaliser column
// sum_d a[d] S[d][D] (scalar), on a staged state.
__device__ __forceinline__ void vec_state(const float* a, const float (*sS)[kSPitch], float* y,
                                          float& yz) {
    uint64_t y2[kD / 2];
#pragma unroll
    for (int i = 0; i < kD / 2; ++i) y2[i] = 0ull;
    float z = 0.f;
#pragma unroll 4
    for (int d = 0; d < kD; ++d) {
        const uint64_t a2 = pack2(a[d], a[d]);
        const float2* row = reinterpret_cast<const float2*>(sS[d]);
#pragma unroll
        for (int i = 0; i < kD / 2; ++i) {
            const float2 sv = row[i];
            y2[i] = fma2(a2, pack2(sv.x, sv.y), y2[i]);
        }
        z = fmaf(a[d], sS[d][kD], z);
    }
#pragma unroll
    for (int i = 0; i < kD / 2; ++i) unpack2(y2[i], y[2 * i], y[2 * i + 1]);
    yz = z;
}

// y[d] = sum_{e < D} S[d][e] b[e] (packed pairs over e, lanes added at the end).
__device__ __forceinline__ void state_vec(const float (*sS)[kSPitch], const float* b, float* y) {
    uint64_t b2[kD / 2];
#pragma unroll
    for (int i = 0; i < kD / 2; ++i) b2[i] = pack2(b[2 * i], b[2 * i + 1]);
#pragma unroll
    for (int d = 0; d < kD; ++d) {
        const float2* row = reinterpret_cast<const float2*>(sS[d]);
        uint64_t acc = 0ull;
#pragma unroll
        for (int i = 0; i < kD / 2; ++i) {
            const float2 sv = row[i];
            acc = fma2(b2[i], pack2(sv.x, sv.y), acc);
        }
        float lo, hi;
        unpack2(acc, lo, hi);
        y[d] = lo + hi;
    }
}

// u, r and phi of one head's 32 values; returns r (1 with the norm off).
__device__ __forceinline__ float phi_fwd32(const float* x, const float* g, float eps, bool norm,
                                           float* u, float* p) {
    float r = 1.f;
    if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < kD; ++i) ss = fmaf(x[i], x[i], ss);
        r = rsqrtf(ss * (1.f / kD) + eps);
#pragma unroll
        for (int i = 0; i < kD; ++i) u[i] = __ldg(g + i) * (x[i] * r);
    } else {
#pragma unroll
        for (int i = 0; i < kD; ++i) u[i] = x[i];
    }
#pragma unroll
    for (int i = 0; i < kD; ++i) p[i] = fmaxf(u[i], 0.f);
    return r;
}

// dx (in place over dp) and the per-channel gain contribution du * x * r.
__device__ __forceinline__ void phi_bwd32(float* dp, const float* x, const float* u,
                                          const float* g, float r, bool norm, float* dg) {
#pragma unroll
    for (int i = 0; i < kD; ++i) dp[i] = u[i] > 0.f ? dp[i] : 0.f;       // du
    if (!norm) {
#pragma unroll
        for (int i = 0; i < kD; ++i) dg[i] = 0.f;
        return;
    }
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < kD; ++i) {
        const float gi = __ldg(g + i);
        t = fmaf(dp[i] * gi, x[i], t);
        dg[i] = dp[i] * x[i] * r;
    }
    const float c = r * r * r * t * (1.f / kD);
#pragma unroll
    for (int i = 0; i < kD; ++i) dp[i] = __ldg(g + i) * r * dp[i] - c * x[i];
}

// The CTA's 128 tokens' gain contributions summed per channel in a fixed order
// (warp butterfly, then warps in order) into part[row][h * D + c].
__device__ __forceinline__ void gain_partial_store(const float* dg, float* red, float* part,
                                                   int t, int h) {
    float v[kD];
#pragma unroll
    for (int i = 0; i < kD; ++i) v[i] = dg[i];
    const int lane = t & 31, w = t >> 5;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    red[w * kD + lane] = v[0];                    // lane l holds channel l's warp sum
    __syncthreads();
    if (t < kD) {
        float s = 0.f;
        for (int i = 0; i < kBwdTile / 32; ++i) s += red[i * kD + t];
        part[h * kD + t] = s;
    }
}

// grid (ceil(N / 128), H, B), 128 threads.  Sz: forward states (B, H, D, D+1).
template <typename T>
__global__ void __launch_bounds__(kBwdTile)
bwd_query_simt(const T* __restrict__ q, const T* __restrict__ dout,
               const float* __restrict__ gq, const float* __restrict__ Sz,
               T* __restrict__ dq, float* __restrict__ G, float* __restrict__ gpart,
               int64_t N, int H, float eps, int norm)
{
    __shared__ __align__(16) float sS[kD][kSPitch];
    __shared__ float red[kBwdTile];
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
    stage_state(Sz + ((int64_t)b * H + h) * kStateFloats, sS, t, kBwdTile);
    __syncthreads();
    const int64_t n = (int64_t)tile * kBwdTile + t;
    const bool live = n < N;
    const int64_t C = (int64_t)H * kD;
    const int64_t row = ((int64_t)b * N + n) * C + (int64_t)h * kD;
    float x[kD], u[kD], p[kD], dg[kD];
    float r = 1.f;
    if (live) {
#pragma unroll
        for (int i = 0; i < kD; i += 8) load8(q + row + i, x + i);
        r = phi_fwd32(x, gq + h * kD, eps, norm != 0, u, p);
        float num[kD], numz;
        vec_state(p, sS, num, numz);
        const float den = numz + eps;
        float go[kD];
#pragma unroll
        for (int i = 0; i < kD; i += 8) load8(dout + row + i, go + i);
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < kD; ++e) dot = fmaf(go[e], num[e] / den, dot);
        const float dden = -dot / den;
        float* gr = G + (((int64_t)b * N + n) * H + h) * kGrow;
#pragma unroll
        for (int e = 0; e < kD; ++e) {
            go[e] = go[e] / den;                  // dnum
            gr[e] = go[e];
        }
        gr[kD] = dden;
        float dp[kD];
        state_vec(sS, go, dp);                    // dnum S^T
#pragma unroll
        for (int d = 0; d < kD; ++d) dp[d] = fmaf(dden, sS[d][kD], dp[d]);   // + dden z
        phi_bwd32(dp, x, u, gq + h * kD, r, norm != 0, dg);
#pragma unroll
        for (int i = 0; i < kD; i += 8) store8(dq + row + i, dp + i);
    } else {
#pragma unroll
        for (int i = 0; i < kD; ++i) dg[i] = 0.f;
    }
    if (norm)
        gain_partial_store(dg, red, gpart + ((int64_t)b * gridDim.x + tile) * C, t, h);
}

// Split-N partials of phi(X)^T [G] for G rows of 33 floats per token-head:
// grid (S, H, B), 128 threads; part[((b*H + h)*S + s)][d][e], tokens
// [s*tps, min(N, (s+1)*tps)).  Same structure as kv_partial_simt.
template <typename T>
__global__ void __launch_bounds__(128)
outer_partial_simt(const T* __restrict__ x, const float* __restrict__ gx,
                   const float* __restrict__ G, float* __restrict__ part, int64_t N, int H,
                   int S, int64_t tps, float eps, int norm)
{
    __shared__ float sA[64][kDP];
    __shared__ __align__(16) float sB[64][kSPitch];
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int64_t n0 = (int64_t)s * tps, n1 = min(N, n0 + tps);
    const int64_t C = (int64_t)H * kD;
    const int d = tid >> 2, e0 = (tid & 3) * 8;
    uint64_t acc2[4];                 // columns e0 .. e0 + 7 in pairs
    float acc_last = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc2[i] = 0ull;
    for (int64_t c0 = n0; c0 < n1; c0 += 64) {
        // load role: thread t < 64 forms phi of token c0 + t, threads 64..127 copy its G row
        const int lt = tid & 63;
        const int64_t n = c0 + lt;
        const bool live = n < n1;
        if (tid < 64) {
            float xx[kD], u[kD], p[kD];
            if (live) {
                const T* xp = x + ((int64_t)b * N + n) * C + (int64_t)h * kD;
#pragma unroll
                for (int i = 0; i < kD; i += 8) load8(xp + i, xx + i);
                phi_fwd32(xx, gx + h * kD, eps, norm != 0, u, p);
            } else {
#pragma unroll
                for (int i = 0; i < kD; ++i) p[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < kD; ++i) sA[lt][i] = p[i];
        } else if (live) {
            const float* gr = G + (((int64_t)b * N + n) * H + h) * kGrow;
#pragma unroll
            for (int i = 0; i < kGrow; ++i) sB[lt][i] = gr[i];
        } else {
#pragma unroll
            for (int i = 0; i < kGrow; ++i) sB[lt][i] = 0.f;
        }
        __syncthreads();
        const int cnt = (int)min((int64_t)64, n1 - c0);
        for (int tt = 0; tt < cnt; ++tt) {
            const float a = sA[tt][d];
            const uint64_t a2 = pack2(a, a);
            const float2* br = reinterpret_cast<const float2*>(&sB[tt][e0]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 bv = br[i];
                acc2[i] = fma2(a2, pack2(bv.x, bv.y), acc2[i]);
            }
            acc_last = fmaf(a, sB[tt][kD], acc_last);
        }
        __syncthreads();
    }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) unpack2(acc2[i], acc[2 * i], acc[2 * i + 1]);
    float* out = part + (((int64_t)b * H + h) * S + s) * kStateFloats;
#pragma unroll
    for (int i = 0; i < 8; ++i) out[d * kDP + e0 + i] = acc[i];
    if ((tid & 3) == 0) out[d * kDP + kD] = acc_last;
}

// grid (ceil(N / 128), H, B), 128 threads.  dSz: (B, H, D, D+1) = [dS | dz].
template <typename T>
__global__ void __launch_bounds__(kBwdTile)
bwd_key_simt(const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ gk,
             const float* __restrict__ dSz, T* __restrict__ dk, T* __restrict__ dv,
             float* __restrict__ gpart, int64_t N, int H, float eps, int norm)
{
    __shared__ __align__(16) float sS[kD][kSPitch];
    __shared__ float red[kBwdTile];
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
    stage_state(dSz + ((int64_t)b * H + h) * kStateFloats, sS, t, kBwdTile);
    __syncthreads();
    const int64_t n = (int64_t)tile * kBwdTile + t;
    const bool live = n < N;
    const int64_t C = (int64_t)H * kD;
    const int64_t row = ((int64_t)b * N + n) * C + (int64_t)h * kD;
    float dg[kD];
    if (live) {
        float x[kD], u[kD], p[kD], vv[kD];
#pragma unroll
        for (int i = 0; i < kD; i += 8) load8(k + row + i, x + i);
        const float r = phi_fwd32(x, gk + h * kD, eps, norm != 0, u, p);
#pragma unroll
        for (int i = 0; i < kD; i += 8) load8(v + row + i, vv + i);
        float dvv[kD], unused;
        vec_state(p, sS, dvv, unused);            // phi(K) dS
#pragma unroll
        for (int i = 0; i < kD; i += 8) store8(dv + row + i, dvv + i);
        float dp[kD];
        state_vec(sS, vv, dp);                    // dS V
#pragma unroll
        for (int d = 0; d < kD; ++d) dp[d] += sS[d][kD];                      // + dz
        phi_bwd32(dp, x, u, gk + h * kD, r, norm != 0, dg);
#pragma unroll
        for (int i = 0; i < kD; i += 8) store8(dk + row + i, dp + i);
    } else {
#pragma unroll
        for (int i = 0; i < kD; ++i) dg[i] = 0.f;
    }
    if (norm)
        gain_partial_store(dg, red, gpart + ((int64_t)b * gridDim.x + tile) * C, t, h);
}

// dg[c] = sum over the rows of gpart (B * tiles rows of C) in row order.
__global__ void __launch_bounds__(256)
gain_combine(const float* __restrict__ gpart, float* __restrict__ dg, int64_t rows, int C)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    float s = 0.f;
    for (int64_t r = 0; r < rows; ++r) s += gpart[r * C + c];
    dg[c] = s;
}

}  // namespace sana
