// silu.cuh -- SiLU(g) * u rounded to BF16, shared by the MLP intermediate
// kernel (BF16 inputs) and the gate_up GEMM's fused epilogue (FP32 inputs).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace nvfp4 {

// SiLU(g) * u rounded to BF16.  In FP32 for g >= -80; below, e^-g overflows
// binary32 while the product is still a representable BF16 number, so those
// (rare) elements are evaluated in FP64 and rounded to BF16 once.
__device__ __forceinline__ uint32_t silu_mul1(float g, float u) {
    if (g >= -80.0f) {
        const float s = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
        return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(s, u)));
    }
    const double gd = g;
    return __bfloat16_as_ushort(__double2bfloat16(gd / (1.0 + exp(-gd)) * static_cast<double>(u)));
}

}  // namespace nvfp4
