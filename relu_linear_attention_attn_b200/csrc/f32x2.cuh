// Packed fp32 pairs for sm_100a's fma.rn.f32x2: two fp32 lanes in one 64-bit
// register, each lane an IEEE fused multiply-add with round-to-nearest (the same
// result as fmaf on that lane), at twice the scalar FMA rate.
#pragma once

#include <stdint.h>

#include "sana_common.cuh"

namespace sana {

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t p, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// bf16 pair (lo in the low half-word) -> two fp32 lanes; exact.
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t u) {
    return pack2(bf16lo(u), bf16hi(u));
}

}  // namespace sana
