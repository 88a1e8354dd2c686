// harmonize.cu -- checkpoint-side harmonisation of a fused weight's block
// scales: one common global scale g_c = max_i g_i for all modules, every
// module's scale bytes re-expressed against it, codes untouched:
//
//   s8' = E4M3_RNE_satfinite(fl32(E4M3(s8) * fl32(g_i / g_c))).
//
// Source: chatpaper.ai abstract -- per-module-calibrated checkpoints served by
// fused multi-module GEMMs, the global-scale mismatch and its repair.  The
// largest module scale as the common one is the reading taken here (it never
// saturates a scale); the pages give no formula.
//
// Memory-bound and tiny (N*K/16 bytes, read and written once): a grid-stride
// loop over 16-byte chunks; each thread finds the row of each byte (linear
// or tensor-core scale layout), that row's module, and rescales the byte.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_common.h"
#include "nvfp4.h"

namespace nvfp4 {
namespace {

constexpr int kHarmThreads = 256;

struct HarmArgs {
    uint8_t* sf;
    int64_t nbytes;        // scale bytes of the whole tensor in its layout
    int64_t sfcols;        // K / 16: scales per row (linear layout row length)
    int64_t block_bytes;   // tensor-core layout: bytes per 128-row block
    int layout;
    int nseg;
    int seg_end[NVFP4_MAX_SEGMENTS];
    const float* seg_g[NVFP4_MAX_SEGMENTS];
    float* g_common;
};

// E4M3 byte -> float, exact (every E4M3 value is an FP16 value).  The byte
// fills both halves of the pair, so either half of the result holds it.
__device__ __forceinline__ float e4m3_value_f32(uint32_t byte) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(byte | (byte << 8))));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Non-negative float -> UE4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_encode_rne(float s) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(s));
    return h & 0xFFu;
}

// Row of the scale byte at offset o of the layout.
__device__ __forceinline__ int64_t row_of(int64_t o, const HarmArgs& a) {
    if (a.layout == NVFP4_SF_TCGEN05) {
        // 512-byte atoms of 128 rows x 4 scales: inner offset
        // (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4
        const int64_t blk = o / a.block_bytes;
        const int inner = static_cast<int>(o & 511);
        return blk * 128 + ((inner & 15) >> 2) * 32 + (inner >> 4);
    }
    return o / a.sfcols;
}

__global__ void __launch_bounds__(kHarmThreads) harmonize_kernel(const HarmArgs a) {
    __shared__ float s_ratio[NVFP4_MAX_SEGMENTS];
    __shared__ int s_end[NVFP4_MAX_SEGMENTS];
    if (threadIdx.x == 0) {
        float gc = *a.seg_g[0];
        for (int i = 1; i < a.nseg; ++i) gc = fmaxf(gc, *a.seg_g[i]);
        for (int i = 0; i < NVFP4_MAX_SEGMENTS; ++i) {
            s_ratio[i] = (i < a.nseg) ? __fdiv_rn(*a.seg_g[i], gc) : 1.0f;
            s_end[i] = (i < a.nseg) ? a.seg_end[i] : 0x7FFFFFFF;
        }
        if (blockIdx.x == 0) *a.g_common = gc;
    }
    __syncthreads();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kHarmThreads * 16;
    for (int64_t o = (static_cast<int64_t>(blockIdx.x) * kHarmThreads + threadIdx.x) * 16;
         o < a.nbytes; o += stride) {
        uint8_t v[16];
        const bool whole = o + 16 <= a.nbytes;
        if (whole) {
            *reinterpret_cast<uint4*>(v) = *reinterpret_cast<const uint4*>(a.sf + o);
        } else {
            for (int k = 0; k < 16; ++k) v[k] = (o + k < a.nbytes) ? a.sf[o + k] : 0;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int64_t r = row_of(o + k, a);
            int s = 0;
            while (s < a.nseg - 1 && r >= s_end[s]) ++s;
            // padding rows of the tensor-core layout hold 0 and stay 0
            v[k] = static_cast<uint8_t>(e4m3_encode_rne(__fmul_rn(e4m3_value_f32(v[k]), s_ratio[s])));
        }
        if (whole) {
            *reinterpret_cast<uint4*>(a.sf + o) = *reinterpret_cast<const uint4*>(v);
        } else {
            for (int k = 0; k < 16; ++k)
                if (o + k < a.nbytes) a.sf[o + k] = v[k];
        }
    }
}

}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status nvfp4_harmonize_scales(uint8_t* w_sf, int64_t K, const nvfp4_segment* segs,
                                               int nseg, nvfp4_sf_layout layout, float* g_common,
                                               void* stream) {
    using namespace nvfp4;
    if (!w_sf || !g_common || !segs || nseg < 1 || nseg > NVFP4_MAX_SEGMENTS)
        return NVFP4_ERR_INVALID_ARG;
    if (layout != NVFP4_SF_LINEAR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
    int64_t N = 0;
    for (int s = 0; s < nseg; ++s) {
        if (segs[s].n_offset != N || segs[s].n_size <= 0 || !segs[s].w_gscale)
            return NVFP4_ERR_INVALID_ARG;
        if (segs[s].n_size >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
        // g_common is written while other CTAs still read the module scales
        if (segs[s].w_gscale == g_common) return NVFP4_ERR_INVALID_ARG;
        N += segs[s].n_size;   // at most 16 terms below 2^31: no overflow
    }
    if (K <= 0 || K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (N >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(w_sf)) return NVFP4_ERR_ALIGNMENT;
    size_t nbytes = 0;
    nvfp4_status st = nvfp4_sf_bytes(N, K, layout, &nbytes);
    if (st != NVFP4_OK) return st;
    // the module scales are read, and g_common written, while w_sf is rewritten
    if (overlaps(g_common, 4, w_sf, nbytes)) return NVFP4_ERR_INVALID_ARG;
    for (int s = 0; s < nseg; ++s)
        if (overlaps(segs[s].w_gscale, 4, w_sf, nbytes)) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo dev;
    st = require_sm100(&dev);
    if (st != NVFP4_OK) return st;

    HarmArgs a = {};
    a.sf = w_sf;
    a.nbytes = static_cast<int64_t>(nbytes);
    a.sfcols = K / 16;
    a.block_bytes = 128 * (((K / 16) + 3) / 4 * 4);
    a.layout = layout;
    a.nseg = nseg;
    for (int s = 0; s < nseg; ++s) {
        a.seg_end[s] = static_cast<int>(segs[s].n_offset + segs[s].n_size);
        a.seg_g[s] = segs[s].w_gscale;
    }
    a.g_common = g_common;
    const int64_t chunks = (a.nbytes + 15) / 16;
    int64_t grid = (chunks + kHarmThreads - 1) / kHarmThreads;
    const int64_t cap = static_cast<int64_t>(dev.sms) * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    harmonize_kernel<<<static_cast<unsigned>(grid), kHarmThreads, 0, as_stream(stream)>>>(a);
    return cuda_status(cudaGetLastError());
}
