// common.cuh -- small device helpers shared by the libgdn kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#define GDN_DEVICE __device__ __forceinline__

namespace gdn {

// bf16 bits -> float (exact widening)
GDN_DEVICE float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// two packed bf16 (low half first) -> two floats
GDN_DEVICE float2 bf16x2_to_f32x2(uint32_t packed) {
    return make_float2(__uint_as_float(packed << 16), __uint_as_float(packed & 0xFFFF0000u));
}

// float -> bf16 bits, round to nearest even (hardware conversion)
GDN_DEVICE uint32_t f32_to_bf16_bits(float x) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}

// two floats -> packed bf16x2 (x in the low half), round to nearest even
GDN_DEVICE uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// softplus(x) = log(1 + e^x) without overflow
GDN_DEVICE float softplus_f32(float x) {
    return x > 0.f ? x + log1pf(expf(-x)) : log1pf(expf(x));
}

// log(alpha) = -exp(A_log) * softplus(a + dt_bias)
GDN_DEVICE float log_alpha_f32(float a, float A_log, float dt_bias) {
    return -expf(A_log) * softplus_f32(a + dt_bias);
}

GDN_DEVICE float sigmoid_f32(float b) { return 1.f / (1.f + expf(-b)); }

GDN_DEVICE float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

}  // namespace gdn
