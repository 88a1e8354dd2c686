// quantize.cu -- the bandwidth-bound half of the NVFP4 W4A4 layer:
//   nvfp4_global_scale: per-tensor FP32 scale from the absolute maximum,
//   nvfp4_quantize:     16-element block scales (UE4M3) and packed E2M1 codes,
//                       scales written straight into the tensor-core layout.
// Format: evolve.pub review of "Why Gated DeltaNet Survives 4-Bit
// Quantization", Scope & Claims (E2M1 values, E4M3 scale per 16-element
// block); per-module global scales: chatpaper.ai abstract.
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_common.h"
#include "nvfp4.h"

namespace nvfp4 {
namespace {

struct GlobalScaleWorkspace {
    unsigned int amax_bits;  // running max of |x| as float bits (non-negative)
    unsigned int ticket;     // CTAs finished
};

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / 32;
constexpr int kGsUnroll = 4;

// 16-byte streaming load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Max of the BF16 magnitudes (bit patterns with the sign cleared) held in a
// 16-byte vector, folded into a running two-lane unsigned max.
__device__ __forceinline__ uint32_t vmax_mag(uint32_t m, const uint4& v) {
    m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    return m;
}

// ---------------------------------------------------------------------------
// Global scale: every warp walks whole rows with coalesced 16-byte loads and
// keeps the max magnitude as an integer (the BF16 bit order of non-negative
// values is their numeric order, so the max is exact).  One atomic per CTA;
// the last CTA to finish turns the max into g and resets the workspace.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
global_scale_kernel(const uint8_t* __restrict__ x, int64_t rows, int64_t vec_per_row,
                    int64_t ld_bytes, float* __restrict__ g_out, float* __restrict__ amax_out,
                    GlobalScaleWorkspace* ws) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    uint32_t m = 0;
    for (int64_t r = warp; r < rows; r += nwarps) {
        const uint8_t* row = x + r * ld_bytes;
        int64_t c = lane;
        for (; c + 32 * (kGsUnroll - 1) < vec_per_row; c += 32 * kGsUnroll) {
            uint4 v[kGsUnroll];
#pragma unroll
            for (int u = 0; u < kGsUnroll; ++u) v[u] = ld_stream(row + (c + 32 * u) * 16);
#pragma unroll
            for (int u = 0; u < kGsUnroll; ++u) m = vmax_mag(m, v[u]);
        }
        for (; c < vec_per_row; c += 32) m = vmax_mag(m, ld_stream(row + c * 16));
    }
    uint32_t mag = max(m & 0xFFFFu, m >> 16);
    mag = __reduce_max_sync(0xFFFFFFFFu, mag);
    __shared__ uint32_t s_max[kWarpsPerBlock];
    if (lane == 0) s_max[threadIdx.x >> 5] = mag;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
#pragma unroll
        for (int i = 0; i < kWarpsPerBlock; ++i) b = max(b, s_max[i]);
        if (b) atomicMax(&ws->amax_bits, b << 16);
        __threadfence();
        const unsigned int t = atomicAdd(&ws->ticket, 1u);
        if (t == gridDim.x - 1) {
            __threadfence();
            const unsigned int bits = atomicExch(&ws->amax_bits, 0u);
            const float amax = __uint_as_float(bits);
            const float g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
            *g_out = g;
            if (amax_out) *amax_out = amax;
            atomicExch(&ws->ticket, 0u);
        }
    }
}

// ---------------------------------------------------------------------------
// Quantizer.  Work unit = 64 consecutive elements of a row (4 blocks of 16),
// handled by 8 threads with one 16-byte load each; a warp covers 4 units per
// step and a warp task is 16 units of one row (4 loads in flight per thread).
// Each pair of threads owns one 16-block: one shuffle gives the block max,
// both compute the scale, each converts its 8 elements.  The 4 scale bytes of
// a unit land in one 32-bit word of the tensor-core layout.
// ---------------------------------------------------------------------------
struct QuantParams {
    const uint8_t* x;
    int64_t ld_bytes;
    int64_t rows;
    int64_t cols;
    const float* g;
    uint8_t* codes;
    uint8_t* sf;
    int64_t row0;              // first row of this slice in the whole tensor
    uint32_t rows_walk;        // slice rows, plus the layout's padding rows if last
    uint32_t units_per_row;    // ceil(cols / 64)
    uint32_t tasks_per_row;    // ceil(units_per_row / 16)
    uint32_t sf_groups;        // padded scale columns / 4 (tensor-core layout)
    int layout;
};

constexpr int kUnitsPerTask = 16;
constexpr int kStepsPerTask = kUnitsPerTask / 4;

// UE4M3 encode (round to nearest even, saturate at 448) of a non-negative
// float; the hardware conversion is exact RNE.
__device__ __forceinline__ uint32_t e4m3_rne_satfinite(float s) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(s));
    return h & 0xFFu;
}

// UE4M3 decode from the bit fields: bias 7, subnormals m * 2^-9.
__device__ __forceinline__ float e4m3_decode(uint32_t s8) {
    const uint32_t e = (s8 >> 3) & 15u, m = s8 & 7u;
    if (e == 0) return static_cast<float>(m) * 0.001953125f;  // exact: m * 2^-9
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eight E2M1 codes (round to nearest even, saturate at 6) packed into a word,
// element 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8(const float (&t)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(out)
        : "f"(t[0]), "f"(t[1]), "f"(t[2]), "f"(t[3]), "f"(t[4]), "f"(t[5]), "f"(t[6]),
          "f"(t[7]));
    return out;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__global__ void __launch_bounds__(kThreads) quantize_kernel(QuantParams p) {
    const int lane = threadIdx.x & 31;
    const int sub = lane & 7;   // 16-byte slot inside the 64-element unit
    const int oct = lane >> 3;  // unit inside the warp step
    const uint32_t warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;
    const uint32_t total = p.rows_walk * p.tasks_per_row;
    const float g = *p.g;
    const int64_t code_row_bytes = p.cols / 2;
    const int64_t sfcols = p.cols / 16;

    for (uint32_t task = warp; task < total; task += nwarps) {
        const uint32_t rl = task / p.tasks_per_row;      // row inside the slice
        const uint32_t tk = task - rl * p.tasks_per_row;
        const bool row_ok = rl < p.rows;
        const int64_t r = p.row0 + rl;                   // row of the whole tensor
        uint4 v[kStepsPerTask];
#pragma unroll
        for (int s = 0; s < kStepsPerTask; ++s) {
            const uint32_t unit = tk * kUnitsPerTask + s * 4 + oct;
            const int64_t e = static_cast<int64_t>(unit) * 64 + sub * 8;
            v[s] = make_uint4(0, 0, 0, 0);
            if (row_ok && e < p.cols) v[s] = ld_stream(p.x + rl * p.ld_bytes + e * 2);
        }
#pragma unroll
        for (int s = 0; s < kStepsPerTask; ++s) {
            const uint32_t unit = tk * kUnitsPerTask + s * 4 + oct;
            const int64_t e = static_cast<int64_t>(unit) * 64 + sub * 8;
            // block max: this thread's 8 magnitudes, then its pair partner's
            uint32_t m2 = vmax_mag(0u, v[s]);
            uint32_t mag = max(m2 & 0xFFFFu, m2 >> 16);
            mag = max(mag, __shfl_xor_sync(0xFFFFFFFFu, mag, 1));
            const float ab = __uint_as_float(mag << 16);
            const float sfv = __fdiv_rn(__fdiv_rn(ab, 6.0f), g);
            const uint32_t s8 = e4m3_rne_satfinite(sfv);
            const float d = __fmul_rn(e4m3_decode(s8), g);
            uint32_t packed = 0;
            if (d != 0.0f) {
                float f[8];
                unpack_bf16x8(v[s], f);
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __fdiv_rn(f[i], d);
                packed = e2m1x8(f);
            }
            if (row_ok && e < p.cols)
                *reinterpret_cast<uint32_t*>(p.codes + r * code_row_bytes + e / 2) = packed;
            // the unit's four block scales -> one word (block j in byte j)
            uint32_t w = s8 << (8 * (sub >> 1));
            w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
            w |= __shfl_xor_sync(0xFFFFFFFFu, w, 4);
            if (p.layout == NVFP4_SF_TCGEN05) {
                if (sub == 0 && unit < p.sf_groups) {
                    const uint64_t off = (static_cast<uint64_t>(r >> 7) * p.sf_groups + unit) * 512u +
                                         static_cast<uint64_t>(r & 31) * 16u +
                                         static_cast<uint64_t>((r >> 5) & 3) * 4u;
                    *reinterpret_cast<uint32_t*>(p.sf + off) = w;
                }
            } else {
                const int64_t b = static_cast<int64_t>(unit) * 4 + (sub >> 1);
                if ((sub & 1) == 0 && row_ok && b < sfcols)
                    p.sf[r * sfcols + b] = static_cast<uint8_t>(s8);
            }
        }
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
nvfp4_status current_device_info(DeviceInfo* info) {
    static DeviceInfo cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
    if (cache[dev].sms == 0) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        cache[dev] = d;
    }
    *info = cache[dev];
    return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_sf_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout,
                                       size_t* bytes) {
    if (!bytes || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
    if (cols % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t sfcols = cols / 16;
    if (layout == NVFP4_SF_LINEAR) {
        *bytes = static_cast<size_t>(rows * sfcols);
    } else if (layout == NVFP4_SF_TCGEN05) {
        *bytes = static_cast<size_t>(((rows + 127) / 128 * 128) * ((sfcols + 3) / 4 * 4));
    } else {
        return NVFP4_ERR_INVALID_ARG;
    }
    return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_global_scale(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                           float* g_out, float* amax_out, void* workspace,
                                           void* stream) {
    if (!g_out || !workspace || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0 && !x) return NVFP4_ERR_INVALID_ARG;
    if (cols % 8 != 0 || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    if (rows > 0 && ld < cols) return NVFP4_ERR_INVALID_ARG;
    if ((x && !aligned16(x)) || !aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    DeviceInfo dev;
    nvfp4_status st = current_device_info(&dev);
    if (st != NVFP4_OK) return st;
    const int64_t eff_rows = (cols == 0) ? 0 : rows;
    int64_t warps = eff_rows < 1 ? 1 : eff_rows;
    const int64_t max_warps = static_cast<int64_t>(dev.sms) * 64;
    if (warps > max_warps) warps = max_warps;
    const int blocks = static_cast<int>((warps + kWarpsPerBlock - 1) / kWarpsPerBlock);
    global_scale_kernel<<<blocks, kThreads, 0, as_stream(stream)>>>(
        static_cast<const uint8_t*>(x), eff_rows, cols / 8, ld * 2, g_out, amax_out,
        static_cast<GlobalScaleWorkspace*>(workspace));
    return cuda_status(cudaGetLastError());
}

namespace {

nvfp4_status quantize_impl(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* g,
                           uint8_t* codes, uint8_t* sf, nvfp4_sf_layout layout,
                           int64_t row_offset, int64_t total_rows, void* stream) {
    if (rows < 0 || cols < 0 || !g || row_offset < 0 || total_rows < 0)
        return NVFP4_ERR_INVALID_ARG;
    if (row_offset + rows > total_rows) return NVFP4_ERR_INVALID_ARG;
    if (layout != NVFP4_SF_LINEAR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
    if (cols % 32 != 0 || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    const bool last = (row_offset + rows == total_rows);
    const int64_t pad_end = (layout == NVFP4_SF_TCGEN05) ? (total_rows + 127) / 128 * 128 : total_rows;
    const int64_t rows_walk = last ? pad_end - row_offset : rows;
    if (rows_walk == 0 || cols == 0) return NVFP4_OK;
    if (!codes || !sf || (rows > 0 && !x)) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && ld < cols) return NVFP4_ERR_INVALID_ARG;
    if ((x && !aligned16(x)) || !aligned16(codes) || !aligned16(sf)) return NVFP4_ERR_ALIGNMENT;
    QuantParams p;
    p.x = static_cast<const uint8_t*>(x);
    p.ld_bytes = ld * 2;
    p.rows = rows;
    p.cols = cols;
    p.g = g;
    p.codes = codes;
    p.sf = sf;
    p.layout = layout;
    p.row0 = row_offset;
    const int64_t units = (cols + 63) / 64;
    const int64_t tasks_per_row = (units + kUnitsPerTask - 1) / kUnitsPerTask;
    if (rows_walk * tasks_per_row >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    p.rows_walk = static_cast<uint32_t>(rows_walk);
    p.units_per_row = static_cast<uint32_t>(units);
    p.tasks_per_row = static_cast<uint32_t>(tasks_per_row);
    p.sf_groups = static_cast<uint32_t>(units);  // roundup(cols/16, 4) / 4
    DeviceInfo dev;
    nvfp4_status st = current_device_info(&dev);
    if (st != NVFP4_OK) return st;
    const int64_t tasks = rows_walk * tasks_per_row;
    int64_t blocks = (tasks + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t max_blocks = static_cast<int64_t>(dev.sms) * 8;
    if (blocks > max_blocks) blocks = max_blocks;
    quantize_kernel<<<static_cast<int>(blocks), kThreads, 0, as_stream(stream)>>>(p);
    return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                       const float* g, uint8_t* codes, uint8_t* sf,
                                       nvfp4_sf_layout layout, void* stream) {
    return quantize_impl(x, rows, cols, ld, g, codes, sf, layout, 0, rows, stream);
}

extern "C" nvfp4_status nvfp4_quantize_slice(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                             const float* g, uint8_t* codes, uint8_t* sf,
                                             nvfp4_sf_layout layout, int64_t row_offset,
                                             int64_t total_rows, void* stream) {
    return quantize_impl(x, rows, cols, ld, g, codes, sf, layout, row_offset, total_rows, stream);
}
