// Symmetric int8 quantisation for the W8A8 prologue of the fused variant
// ("Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
// Transformers", section 7, on-device deployment: linear layers with 8-bit
// weights and activations, attention in full precision).  The pages do not fix
// the granularity; here x has one scale per token (row) and Wqkv one per output
// channel (column):
//     scale = max|x| / 127            (fp32, IEEE division)
//     code  = rint(x / scale)         (fp32 IEEE division, round half to even),
//             clamped to [-127, 127]; scale 0 and zero codes for an all-zero slice.
// Both kernels are HBM-bound elementwise passes (read 2 or 4 B, write 1 B).
#pragma once

#include "sana_common.cuh"

namespace sana {

__device__ __forceinline__ int8_t quant_code(float x, float s) {
    if (s == 0.f) return 0;
    int q = __float2int_rn(__fdiv_rn(x, s));
    q = q > 127 ? 127 : (q < -127 ? -127 : q);
    return (int8_t)q;
}

// One warp per row of `cols` elements (cols % 8 == 0, rows 16-byte aligned):
// the row's max |x| by a warp max (order-free, exact), then the codes.
template <typename T>
__global__ void __launch_bounds__(256)
quantize_rows_i8(const T* __restrict__ x, int8_t* __restrict__ q, float* __restrict__ scale,
                 int64_t rows, int cols)
{
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const T* xr = x + row * cols;
    float amax = 0.f;
    for (int c = lane * 8; c < cols; c += 32 * 8) {
        float v[8];
        load8(xr + c, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = __fdiv_rn(amax, 127.f);
    int8_t* qr = q + row * cols;
    for (int c = lane * 8; c < cols; c += 32 * 8) {
        float v[8];
        load8(xr + c, v);
        uint32_t w0 = 0, w1 = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            w0 |= (uint32_t)(uint8_t)quant_code(v[i], s) << (8 * i);
            w1 |= (uint32_t)(uint8_t)quant_code(v[4 + i], s) << (8 * i);
        }
        *reinterpret_cast<uint2*>(qr + c) = make_uint2(w0, w1);
    }
    if (lane == 0) scale[row] = s;
}

// Per column of a (K, cols) row-major matrix: block (32, 8) covers 32 columns;
// thread (x, y) scans rows y, y + 8, ... of column x.
template <typename T>
__global__ void __launch_bounds__(256)
quantize_cols_i8(const T* __restrict__ w, int8_t* __restrict__ q, float* __restrict__ scale,
                 int64_t K, int cols)
{
    __shared__ float red[8][33];
    const int col = blockIdx.x * 32 + threadIdx.x;
    const bool live = col < cols;
    float amax = 0.f;
    if (live)
        for (int64_t r = threadIdx.y; r < K; r += 8) amax = fmaxf(amax, fabsf(to_float(w[r * cols + col])));
    red[threadIdx.y][threadIdx.x] = amax;
    __syncthreads();
    if (threadIdx.y == 0) {
        for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i][threadIdx.x]);
        red[0][threadIdx.x] = amax;
    }
    __syncthreads();
    const float s = __fdiv_rn(red[0][threadIdx.x], 127.f);
    if (live) {
        for (int64_t r = threadIdx.y; r < K; r += 8) q[r * cols + col] = quant_code(to_float(w[r * cols + col]), s);
        if (threadIdx.y == 0) scale[col] = s;
    }
}

}  // namespace sana
