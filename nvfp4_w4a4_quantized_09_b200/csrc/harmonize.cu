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
// Memory-bound and small (N*K/16 bytes, read and written once): a grid-stride
// loop over 16-byte chunks.  A chunk's rows come from one division per chunk:
// in the tensor-core layout its bytes are four scales of each of four rows
// (32 rows apart), in the linear layout one run of consecutive rows; the
// module of each row is found by walking the segment table forward from the
// previous row's.  Bytes are decoded, rescaled and encoded in pairs.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_common.h"
#include "nvfp4.h"

namespace nvfp4 {
namespace {

constexpr int kHarmThreads = 256;
static_assert(kHarmThreads >= NVFP4_MAX_SEGMENTS, "one thread per module scale");

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

// Two E4M3 bytes (low byte first) -> two floats, exact (every E4M3 value is
// an FP16 value).
__device__ __forceinline__ float2 e4m3x2_values(uint32_t pair) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(pair)));
    return make_float2(__half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu))),
                       __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16))));
}

// Two non-negative floats -> two UE4M3 bytes (lo in the low byte), round to
// nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3x2_encode_rne(float lo, float hi) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
    return h;
}

// Module of row r, walking forward from segment s (rows only grow).
__device__ __forceinline__ int seg_from(int s, int64_t r, int nseg, const int* end) {
    while (s < nseg - 1 && r >= end[s]) ++s;
    return s;
}

__global__ void __launch_bounds__(kHarmThreads) harmonize_kernel(const HarmArgs a) {
    __shared__ float s_g[NVFP4_MAX_SEGMENTS];
    __shared__ float s_ratio[NVFP4_MAX_SEGMENTS];
    __shared__ int s_end[NVFP4_MAX_SEGMENTS];
    // the module scales are read in parallel (one dependent load per CTA, not nseg)
    if (threadIdx.x < a.nseg) s_g[threadIdx.x] = *a.seg_g[threadIdx.x];
    __syncthreads();
    if (threadIdx.x < NVFP4_MAX_SEGMENTS) {
        float gc = s_g[0];
        for (int i = 1; i < a.nseg; ++i) gc = fmaxf(gc, s_g[i]);
        const int i = threadIdx.x;
        s_ratio[i] = (i < a.nseg) ? __fdiv_rn(s_g[i], gc) : 1.0f;
        s_end[i] = (i < a.nseg) ? a.seg_end[i] : 0x7FFFFFFF;
        if (blockIdx.x == 0 && i == 0) *a.g_common = gc;
    }
    __syncthreads();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kHarmThreads * 16;
    for (int64_t o = (static_cast<int64_t>(blockIdx.x) * kHarmThreads + threadIdx.x) * 16;
         o < a.nbytes; o += stride) {
        uint32_t w[4];
        const bool whole = o + 16 <= a.nbytes;
        if (whole) {
            const uint4 q = *reinterpret_cast<const uint4*>(a.sf + o);
            w[0] = q.x, w[1] = q.y, w[2] = q.z, w[3] = q.w;
        } else {
            for (int j = 0; j < 4; ++j) {
                w[j] = 0;
                for (int b = 0; b < 4; ++b)
                    if (o + 4 * j + b < a.nbytes) w[j] |= static_cast<uint32_t>(a.sf[o + 4 * j + b]) << (8 * b);
            }
        }
        // module ratio of every byte of the chunk
        float ratio[16];
        if (a.layout == NVFP4_SF_TCGEN05) {
            // 512-byte atoms of 128 rows x 4 scales, inner offset
            // (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4: word j of the chunk
            // holds the four scales of row 32 j + (inner / 16) of the block
            const int64_t r0 = (o / a.block_bytes) * 128 + ((o & 511) >> 4);
            int s = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                s = seg_from(s, r0 + 32 * j, a.nseg, s_end);   // padding rows hold 0 and stay 0
#pragma unroll
                for (int b = 0; b < 4; ++b) ratio[4 * j + b] = s_ratio[s];
            }
        } else {
            // consecutive bytes of consecutive rows, sfcols per row
            int64_t r = o / a.sfcols;
            int64_t left = (r + 1) * a.sfcols - o;       // bytes of row r from o on
            int s = seg_from(0, r, a.nseg, s_end);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                while (k >= left) {
                    ++r;
                    left += a.sfcols;
                    s = seg_from(s, r, a.nseg, s_end);
                }
                ratio[k] = s_ratio[s];
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 lo = e4m3x2_values(w[j] & 0xFFFFu), hi = e4m3x2_values(w[j] >> 16);
            w[j] = e4m3x2_encode_rne(__fmul_rn(lo.x, ratio[4 * j]), __fmul_rn(lo.y, ratio[4 * j + 1])) |
                   (e4m3x2_encode_rne(__fmul_rn(hi.x, ratio[4 * j + 2]), __fmul_rn(hi.y, ratio[4 * j + 3])) << 16);
        }
        if (whole) {
            *reinterpret_cast<uint4*>(a.sf + o) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
            for (int k = 0; k < 16; ++k)
                if (o + k < a.nbytes) a.sf[o + k] = static_cast<uint8_t>(w[k >> 2] >> (8 * (k & 3)));
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
