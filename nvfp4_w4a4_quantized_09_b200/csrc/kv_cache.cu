// kv_cache.cu -- FP8 E4M3 KV-cache quantization with a calibrated per-tensor
// scale:  s = fl32(amax / 448),  byte = signed E4M3_RNE_satfinite(fl32(x / s)).
//
// Source: evolve.pub, Key claims under review (calibrated per-tensor FP8
// KV-cache scales, throughput-free).  The formula is the plain reading of a
// per-tensor FP8 scale; the pages give none.
//
// Bandwidth-bound (2 bytes in, 1 byte out per element); each thread keeps four
// 16-byte loads in flight.  Exactness without a
// division per element: with r = RN(1/s), the reals r(1 - 2^-20) and
// r(1 + 2^-20), rounded, bracket 1/s (r is within 2^-24 of 1/s), so x*rlo and
// x*rhi bracket the exact quotient x/s; fl32 rounding and the E4M3 RNE encode
// are both monotone, so when the two bracket codes agree they equal the code
// of fl32(x/s).  Elements whose bracket codes differ (a quotient within 2^-20
// of a rounding boundary) take the IEEE division.  If 1/s is not a normal
// float every element divides.
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_common.h"
#include "nvfp4.h"

namespace nvfp4 {
namespace {

constexpr int kKvThreads = 256;
constexpr int kKvUnroll = 4;      // vectors in flight per thread

struct KvArgs {
    const uint8_t* x;
    int64_t ld_bytes;
    uint8_t* out;
    int64_t ldo;
    int64_t rows;
    uint32_t vec_per_row;    // cols / 8
    const float* scale;
};

// Two signed E4M3 codes (RNE, saturating at 448): low byte from a, high from b.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(b), "f"(a));
    return h;
}

// 16-byte streaming load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Eight BF16 values -> eight signed E4M3 bytes of fl32(x / s).
__device__ __forceinline__ uint2 quantize8(const uint4 w, float s, float rlo, float rhi, bool fast) {
    float x[8];
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(ww[i] << 16);
        x[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
    }
    uint32_t lo[2], hi[2];
    if (fast) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            lo[h] = e4m3x2(__fmul_rn(x[4 * h], rlo), __fmul_rn(x[4 * h + 1], rlo)) |
                    (e4m3x2(__fmul_rn(x[4 * h + 2], rlo), __fmul_rn(x[4 * h + 3], rlo)) << 16);
            hi[h] = e4m3x2(__fmul_rn(x[4 * h], rhi), __fmul_rn(x[4 * h + 1], rhi)) |
                    (e4m3x2(__fmul_rn(x[4 * h + 2], rhi), __fmul_rn(x[4 * h + 3], rhi)) << 16);
        }
    }
    if (!fast || ((lo[0] ^ hi[0]) | (lo[1] ^ hi[1])) != 0) {
        // near a rounding boundary (or no usable reciprocal): divide
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int sh = 8 * j;
                if (!fast || (((lo[h] ^ hi[h]) >> sh) & 0xFFu))
                    word |= (e4m3x2(__fdiv_rn(x[4 * h + j], s), 0.0f) & 0xFFu) << sh;
                else
                    word |= lo[h] & (0xFFu << sh);
            }
            lo[h] = word;
        }
    }
    return make_uint2(lo[0], lo[1]);
}

__global__ void __launch_bounds__(kKvThreads) kv_quantize_kernel(const KvArgs a) {
    const float s = *a.scale;
    const float rs = __fdiv_rn(1.0f, s);
    const float ars = fabsf(rs);
    const bool fast = ars >= 0x1p-125f && ars <= 0x1p125f;
    const float rlo = __fmul_rn(rs, 1.0f - 0x1p-20f);
    const float rhi = __fmul_rn(rs, 1.0f + 0x1p-20f);
    // Walk (row, vector) pairs with carries instead of dividing; each thread
    // keeps kKvUnroll vectors in flight (loads issued before any math).
    const uint32_t vpr = a.vec_per_row;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kKvThreads;
    const uint64_t start = static_cast<uint64_t>(blockIdx.x) * kKvThreads + threadIdx.x;
    int64_t r[kKvUnroll];
    uint32_t v[kKvUnroll];
#pragma unroll
    for (int u = 0; u < kKvUnroll; ++u) {
        const uint64_t e = start + u * stride;
        r[u] = static_cast<int64_t>(e / vpr);
        v[u] = static_cast<uint32_t>(e - static_cast<uint64_t>(r[u]) * vpr);
    }
    const uint64_t big = stride * kKvUnroll;
    const int64_t step_r = static_cast<int64_t>(big / vpr);
    const uint32_t step_v = static_cast<uint32_t>(big - static_cast<uint64_t>(step_r) * vpr);
    while (r[0] < a.rows) {
        uint4 w[kKvUnroll];
#pragma unroll
        for (int u = 0; u < kKvUnroll; ++u)
            if (r[u] < a.rows)
                w[u] = ld_stream16(a.x + r[u] * a.ld_bytes + 16 * static_cast<int64_t>(v[u]));
#pragma unroll
        for (int u = 0; u < kKvUnroll; ++u) {
            if (r[u] < a.rows) {
                const uint2 o = quantize8(w[u], s, rlo, rhi, fast);
                *reinterpret_cast<uint2*>(a.out + r[u] * a.ldo + 8 * static_cast<int64_t>(v[u])) = o;
            }
            r[u] += step_r;
            v[u] += step_v;
            if (v[u] >= vpr) {
                v[u] -= vpr;
                ++r[u];
            }
        }
    }
}

__global__ void kv_scale_kernel(const float* amax, float* scale) {
    const float m = *amax;
    *scale = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
}

}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status nvfp4_kv_scale_from_amax(const float* amax, float* scale, void* stream) {
    using namespace nvfp4;
    if (!amax || !scale) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo dev;
    const nvfp4_status st = current_device_info(&dev);
    if (st != NVFP4_OK) return st;
    kv_scale_kernel<<<1, 1, 0, as_stream(stream)>>>(amax, scale);
    return cuda_status(cudaGetLastError());
}

extern "C" nvfp4_status nvfp4_kv_quantize_e4m3(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                               const float* scale, uint8_t* out, int64_t ldo,
                                               void* stream) {
    using namespace nvfp4;
    if (rows < 0 || cols < 0 || !scale) return NVFP4_ERR_INVALID_ARG;
    if (cols % 8 != 0 || ld % 8 != 0 || ldo % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    if (rows == 0 || cols == 0) return NVFP4_OK;
    if (!x || !out || ld < cols || ldo < cols) return NVFP4_ERR_INVALID_ARG;
    if (extent_too_large(rows, ld, 2) || extent_too_large(rows, ldo, 1))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(out) & 7u) != 0) return NVFP4_ERR_ALIGNMENT;
    // every CTA reads *scale while others write out
    if (overlaps(scale, 4, out, extent_bytes(rows, ldo, cols, 1))) return NVFP4_ERR_INVALID_ARG;
    if (cols / 8 >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo dev;
    const nvfp4_status st = current_device_info(&dev);
    if (st != NVFP4_OK) return st;
    KvArgs a;
    a.x = static_cast<const uint8_t*>(x);
    a.ld_bytes = ld * 2;
    a.out = out;
    a.ldo = ldo;
    a.rows = rows;
    a.vec_per_row = static_cast<uint32_t>(cols / 8);
    a.scale = scale;
    const int64_t vecs = rows * (cols / 8);
    int64_t grid = (vecs + kKvThreads - 1) / kKvThreads;
    const int64_t cap = static_cast<int64_t>(dev.sms) * 8;
    if (grid > cap) grid = cap;
    kv_quantize_kernel<<<static_cast<unsigned>(grid), kKvThreads, 0, as_stream(stream)>>>(a);
    return cuda_status(cudaGetLastError());
}
