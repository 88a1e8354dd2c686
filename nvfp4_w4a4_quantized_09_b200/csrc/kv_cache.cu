// kv_cache.cu -- FP8 E4M3 KV-cache quantization with a calibrated per-tensor
// scale:  s = fl32(amax / 448),  byte = signed E4M3_RNE_satfinite(fl32(x / s)).
//
// Source: evolve.pub, Key claims under review (calibrated per-tensor FP8
// KV-cache scales, throughput-free).  The formula is the plain reading of a
// per-tensor FP8 scale; the pages give none.
//
// Bandwidth-bound (2 bytes in, 1 byte out per element); each thread keeps
// several 16-byte loads in flight.  The quotient fl32(x / s) is exact without
// a division per element: with r = RN(1/s) and q0 = RN(x r), the remainder
// x - q0 s is exact in one FMA and RN(q0 + (x - q0 s) r) is the correctly
// rounded quotient (Markstein's theorem: P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990), provided no step over- or underflows.
//  * s in [2^-92, 2^100] keeps r normal and the remainder exact for every
//    quotient of 2^-11 or more; below that (x subnormal or tiny) the result
//    stays under 2^-11 with the sign of x/s, and every such value encodes to a
//    signed zero, as the exact quotient does.  Other s divide.
//  * The quotient is formed from -x and -r, each step the exact negation image
//    of the textbook one, so that x = -0 gives -0 (byte 0x80) as division does.
//  * A quotient that overflows (x/s >= 2^128, or x infinite) comes out NaN;
//    the NaN byte marks its group of eight, which divides instead.
// One E4M3 pair conversion per two elements (the conversion pipe is narrow).
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_common.h"
#include "nvfp4.h"

namespace nvfp4 {
namespace {

constexpr int kKvThreads = 256;
#ifndef NVFP4_KV_UNROLL
#define NVFP4_KV_UNROLL 4
#endif
#ifndef NVFP4_KV_MINB
#define NVFP4_KV_MINB 4
#endif
constexpr int kKvUnroll = NVFP4_KV_UNROLL;      // vectors in flight per thread
constexpr int kKvCtasPerSm = NVFP4_KV_MINB;     // resident CTAs per SM the grid is sized for

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

// Packed pairs of binary32 values, each operation rounded to nearest even.
__device__ __forceinline__ uint64_t f32x2(uint32_t lo, uint32_t hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(lo), "r"(hi));
    return v;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// 16-byte streaming load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

struct KvConsts {
    float s;
    uint64_t S;      // s in both halves
    uint64_t NR;     // -RN(1/s) in both halves
    bool fast;       // s in [2^-92, 2^100]
};

// Eight BF16 values -> eight signed E4M3 bytes of fl32(x / s).
__device__ __forceinline__ uint2 quantize8(const uint4 w, const KvConsts& K) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    if (K.fast) {
        uint32_t h[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // -x of both elements: the BF16 bits moved into place, sign flipped
            const uint64_t nx = f32x2(ww[i] * 0x10000u + 0x80000000u, (ww[i] & 0xFFFF0000u) ^ 0x80000000u);
            const uint64_t q0 = mul_f32x2(nx, K.NR);
            const uint64_t e = fma_f32x2(q0, K.S, nx);
            const uint64_t q1 = fma_f32x2(e, K.NR, q0);
            h[i] = e4m3x2(__uint_as_float(static_cast<uint32_t>(q1)),
                          __uint_as_float(static_cast<uint32_t>(q1 >> 32)));
        }
        const uint32_t b0 = h[0] | (h[1] << 16), b1 = h[2] | (h[3] << 16);
        // a byte whose low seven bits are all set is the NaN code (no finite
        // quotient converts to it under saturation)
        const uint32_t nan = (((b0 & 0x7F7F7F7Fu) + 0x01010101u) | ((b1 & 0x7F7F7F7Fu) + 0x01010101u)) &
                             0x80808080u;
        if (nan == 0) return make_uint2(b0, b1);
    }
    // out of the fast range, an overflowed quotient or a NaN input: divide
    uint32_t b[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t h = e4m3x2(__fdiv_rn(__uint_as_float(ww[i] << 16), K.s),
                                  __fdiv_rn(__uint_as_float(ww[i] & 0xFFFF0000u), K.s));
        b[i >> 1] |= h << (16 * (i & 1));
    }
    return make_uint2(b[0], b[1]);
}

__global__ void __launch_bounds__(kKvThreads, kKvCtasPerSm) kv_quantize_kernel(const KvArgs a) {
    KvConsts K;
    K.s = *a.scale;
    K.fast = K.s >= 0x1p-92f && K.s <= 0x1p100f;
    const float nr = K.fast ? -__fdiv_rn(1.0f, K.s) : 0.0f;
    K.S = f32x2(__float_as_uint(K.s), __float_as_uint(K.s));
    K.NR = f32x2(__float_as_uint(nr), __float_as_uint(nr));
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
                const uint2 o = quantize8(w[u], K);
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
    const int64_t cap = static_cast<int64_t>(dev.sms) * kKvCtasPerSm;
    if (grid > cap) grid = cap;
    kv_quantize_kernel<<<static_cast<unsigned>(grid), kKvThreads, 0, as_stream(stream)>>>(a);
    return cuda_status(cudaGetLastError());
}
