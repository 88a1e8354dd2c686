// silu.cuh -- SiLU(g) * u rounded to BF16, shared by the MLP intermediate
// kernel (BF16 inputs) and the gate_up GEMM's fused epilogue (FP32 inputs).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace nvfp4 {

// SiLU(g) * u for g < -80, where e^-g overflows binary32 while the product
// can still be a representable BF16 number.  There SiLU(g) = g e^g / (1 +
// e^g) equals g e^g to a relative 2^-115, and everything stays in FP32 by
// carrying powers of two apart: u = mu 2^eu (|mu| in [1, 2)), e^g = 2^k 2^f
// with n = g log2(e) = k + f (log2(e) in two parts, so n is exact to about
// 2^-40 relative; k = floor), p = 2^f from exp2f, and h = (g mu p) 2^(eu + k)
// scaled in one or two exact power-of-two steps.  The error before the final
// BF16 rounding is near 2^-22 relative (exp2f's and three roundings).
__device__ __forceinline__ uint32_t silu_mul_tail(float g, float u) {
    const uint32_t ub = __float_as_uint(u);
    if ((ub & 0x7F800000u) == 0)           // zero or subnormal u: the product is below BF16's range
        return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__fmul_rn(g, u), 0.0f)));
    const float L1 = 1.44269502162933349609375f;         // log2(e) to 24 bits
    const float L2 = 1.925963033500011e-8f;              // log2(e) - L1
    const float nh = __fmul_rn(g, L1);
    const float nl = __fmaf_rn(g, L2, __fmaf_rn(g, L1, -nh));   // g log2(e) - nh
    const float k = floorf(nh);
    const float p = exp2f(__fadd_rn(__fsub_rn(nh, k), nl));     // 2^f, f within [0, 1) up to nl
    const float mu = __uint_as_float((ub & 0x807FFFFFu) | 0x3F800000u);
    const int e = static_cast<int>((ub >> 23) & 0xFFu) - 127 + static_cast<int>(k);   // <= 11
    float x = __fmul_rn(__fmul_rn(g, mu), p);
    if (e >= -126)
        x = __fmul_rn(x, __uint_as_float(static_cast<uint32_t>(e + 127) << 23));
    else if (e >= -252)
        x = __fmul_rn(__fmul_rn(x, 0x1p-126f), __uint_as_float(static_cast<uint32_t>(e + 253) << 23));
    else
        x = __fmul_rn(x, 0.0f);
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// SiLU(g) * u rounded to BF16: in FP32 as g / (1 + e^-g) times u for
// g >= -80, by silu_mul_tail below.
__device__ __forceinline__ uint32_t silu_mul1(float g, float u) {
    if (g >= -80.0f) {
        const float s = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
        return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(s, u)));
    }
    return silu_mul_tail(g, u);
}

}  // namespace nvfp4
