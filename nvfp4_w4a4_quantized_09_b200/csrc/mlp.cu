// mlp.cu -- the MLP intermediate between the two W4A4 GEMMs of a SiLU-gated
// MLP: h = SiLU(gate) * up, read from the BF16 gate_up GEMM output and
// written as BF16 for the next global scale + quantization.  Every linear
// layer runs W4A4 (chatpaper.ai abstract), the down projection included.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_common.h"
#include "nvfp4.h"
#include "silu.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// SiLU(g) * u for the two BF16 values in each half of a word pair.
__device__ __forceinline__ uint32_t silu_mul2(uint32_t gw, uint32_t uw) {
    const uint32_t h0 = silu_mul1(__uint_as_float(gw << 16), __uint_as_float(uw << 16));
    const uint32_t h1 = silu_mul1(__uint_as_float(gw & 0xFFFF0000u), __uint_as_float(uw & 0xFFFF0000u));
    return h0 | (h1 << 16);
}

// One thread per 8 outputs; warps walk whole rows (vectors of 8 along f).
__global__ void __launch_bounds__(kThreads)
silu_mul_kernel(const uint8_t* __restrict__ gu, int64_t rows, int64_t vec_per_row,
                int64_t ld_bytes, uint8_t* __restrict__ h, int64_t ldh_bytes, int64_t f_bytes) {
    const int64_t total = rows * vec_per_row;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < total;
         i += stride) {
        const int64_t r = i / vec_per_row;
        const int64_t v = i - r * vec_per_row;
        const uint8_t* row = gu + r * ld_bytes + v * 16;
        const uint4 g = ld_stream16(row);
        const uint4 u = ld_stream16(row + f_bytes);
        uint4 o;
        o.x = silu_mul2(g.x, u.x);
        o.y = silu_mul2(g.y, u.y);
        o.z = silu_mul2(g.z, u.z);
        o.w = silu_mul2(g.w, u.w);
        *reinterpret_cast<uint4*>(h + r * ldh_bytes + v * 16) = o;
    }
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_silu_mul(const void* gate_up, int64_t rows, int64_t f, int64_t ld,
                                       void* h, int64_t ldh, void* stream) {
    if (rows < 0 || f < 0) return NVFP4_ERR_INVALID_ARG;
    if (f % 8 != 0 || ld % 8 != 0 || ldh % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    if (rows == 0 || f == 0) return NVFP4_OK;
    if (!gate_up || !h) return NVFP4_ERR_INVALID_ARG;
    if (extent_too_large(rows, ld, 2) || extent_too_large(rows, ldh, 2))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (f > ld / 2 || ldh < f) return NVFP4_ERR_INVALID_ARG;   // ld >= 2f, ld even
    if (!aligned16(gate_up) || !aligned16(h)) return NVFP4_ERR_ALIGNMENT;
    DeviceInfo dev;
    nvfp4_status st = current_device_info(&dev);
    if (st != NVFP4_OK) return st;
    const int64_t total = rows * (f / 8);
    int64_t blocks = (total + kThreads - 1) / kThreads;
    const int64_t max_blocks = static_cast<int64_t>(dev.sms) * 8;
    if (blocks > max_blocks) blocks = max_blocks;
    silu_mul_kernel<<<static_cast<int>(blocks), kThreads, 0, as_stream(stream)>>>(
        static_cast<const uint8_t*>(gate_up), rows, f / 8, ld * 2, static_cast<uint8_t*>(h),
        ldh * 2, f * 2);
    return cuda_status(cudaGetLastError());
}
