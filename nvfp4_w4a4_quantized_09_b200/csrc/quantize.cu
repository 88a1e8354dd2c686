// quantize.cu -- the bandwidth-bound half of the NVFP4 W4A4 layer:
//   nvfp4_global_scale: per-tensor FP32 scale from the absolute maximum,
//   nvfp4_quantize:     16-element block scales (UE4M3) and packed E2M1 codes,
//                       scales written straight into the tensor-core layout.
// Format: evolve.pub review of "Why Gated DeltaNet Survives 4-Bit
// Quantization", Scope & Claims (the E2M1 element format, with one E4M3
// scale for every 16 elements); per-module global scales: chatpaper.ai abstract.
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
// Quantizer.  One thread owns one 16-element block (32 bytes of BF16): a warp
// chunk covers 64 consecutive blocks of a row (two 1 KB loads per warp in
// flight), and warps walk (row, chunk) pairs with carries instead of
// divisions.  The block max is a bf16x2 abs-max chain.
//
// No IEEE division on the fast path; every result still equals the binary32
// step sequence exactly:
//  * fl32(ab / 6): ab is BF16, i.e. (1 + m/128) * 2^e, and rounding commutes
//    with scaling by 2^e, so it is a 128-entry table of RN((1 + m/128) / 6)
//    with e added to the exponent (tiny ab, where that would underflow, take
//    the IEEE division).
//  * s8 = E4M3(fl32(u / g)): the products u*RN(1/g)*(1 -+ 2^-20) bracket the
//    correctly rounded quotient and E4M3 rounding is monotone, so when both
//    brackets encode to the same byte that byte is exact; otherwise the IEEE
//    division decides.
//  * code = E2M1(fl32(x / d)): likewise x*RN(1/d)*(1 -+ 2^-20) bracket
//    fl32(x/d) and E2M1 rounding is monotone, so every element whose two
//    bracket codes agree has its exact code.  The brackets disagree only for
//    an x/d within ~2^-20 of a rounding threshold (0.25, 0.75, ..., 5); with
//    g = amax / (21 * 2^7) such near-ties are structural rather than rare
//    (d times a threshold often lands next to a BF16 number), so that single
//    element -- not its block -- is recomputed with the IEEE division.
//    Every lane runs the same instructions except for those few elements.
//
// Scales: four neighbouring threads' E4M3 bytes form one 32-bit word of the
// tensor-core layout (block j of a 64-element group in byte j).
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
    uint32_t chunks_per_row;   // ceil(blocks per row / 64)
    uint32_t sf_groups;        // padded scale columns / 4 (tensor-core layout)
    int layout;
};

constexpr int kBlocksPerStep = 32;   // blocks per warp per load
constexpr int kStepsPerChunk = 2;    // loads in flight per thread
constexpr float kLo = 1.0f - 0x1p-20f;
constexpr float kHi = 1.0f + 0x1p-20f;

// UE4M3 encode (round to nearest even, saturate at 448) of a non-negative
// float; the hardware conversion is exact RNE.
__device__ __forceinline__ uint32_t e4m3_rne_satfinite(float s) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(s));
    return h & 0xFFu;
}

// Two UE4M3 encodes at once: low byte from a, high byte from b.
__device__ __forceinline__ uint32_t e4m3x2_rne_satfinite(float a, float b) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(b), "f"(a));
    return h;
}

// UE4M3 decode from the bit fields: bias 7, subnormals m * 2^-9.
__device__ __forceinline__ float e4m3_decode(uint32_t s8) {
    const uint32_t e = (s8 >> 3) & 15u, m = s8 & 7u;
    if (e == 0) return static_cast<float>(m) * 0.001953125f;  // exact: m * 2^-9
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eight E2M1 codes (round to nearest even, saturate at 6) packed into a word,
// element 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8(const float* t) {
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

// Per-lane max(|a|, |b|) of two bf16 pairs (sign bits are junk).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// (a0, a1) * (r, r), each product rounded to nearest even.
__device__ __forceinline__ void mul_f32x2(float a0, float a1, float r, float& o0, float& o1) {
    uint64_t a, b, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %1};" : "=l"(b) : "f"(r));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(o0), "=f"(o1) : "l"(d));
}

struct Block16 {
    uint32_t w[8];  // 16 BF16 values, element 2i in the low half of w[i]
};

// Per-CTA tables, built from g at kernel start.
struct QuantTables {
    float div6[128];     // RN((1 + m/128) / 6)
    float4 dq[128];      // per scale byte: d = fl32(E4M3 * g), RN(1/d)*(1 -+ 2^-20), usable
};

// Kernel-wide constants derived from g.
struct ScaleConsts {
    float g;
    float rg_lo, rg_hi;   // RN(1/g) * (1 -+ 2^-20)
    bool fast;            // g and 1/g in the normal range: the bracket argument holds
};

__device__ __forceinline__ bool normal_range(float v) {
    const float a = fabsf(v);
    return a >= 0x1p-125f && a <= 0x1p125f;
}

__device__ __forceinline__ uint32_t block_scale(float ab, const QuantTables& T,
                                                const ScaleConsts& K) {
    const uint32_t abits = __float_as_uint(ab);
    if (abits == 0) return 0u;
    if (K.fast && abits >= 0x04000000u) {                 // ab >= 2^-119: exact table path
        const uint32_t e = abits >> 23, m7 = (abits >> 16) & 127u;
        const float u = __uint_as_float(__float_as_uint(T.div6[m7]) + ((e - 127u) << 23));
        const uint32_t both = e4m3x2_rne_satfinite(__fmul_rn(u, K.rg_lo), __fmul_rn(u, K.rg_hi));
        if ((both & 0xFFu) == (both >> 8)) return both & 0xFFu;
        return e4m3_rne_satfinite(__fdiv_rn(u, K.g));
    }
    return e4m3_rne_satfinite(__fdiv_rn(__fdiv_rn(ab, 6.0f), K.g));
}

// One E2M1 code (low nibble) of fl32(x / d) by the IEEE division.
__device__ __forceinline__ uint32_t e2m1_exact(float x, float d) {
    uint16_t h;
    asm("{\n\t.reg .b8 q;\n\tcvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\tcvt.u16.u8 %0, q;\n\t}"
        : "=h"(h)
        : "f"(0.0f), "f"(__fdiv_rn(x, d)));
    return h & 0xFu;
}

// Quantize one block: returns the E4M3 scale byte, writes 16 codes to c[2].
__device__ __forceinline__ uint32_t quantize_block(const Block16& b, const QuantTables& T,
                                                   const ScaleConsts& K, uint32_t (&c)[2]) {
    uint32_t m = absmax_bf16x2(b.w[0], b.w[1]);
#pragma unroll
    for (int i = 2; i < 8; ++i) m = absmax_bf16x2(m, b.w[i]);
    const float ab = __uint_as_float(max(m & 0x7FFFu, (m >> 16) & 0x7FFFu) << 16);
    const uint32_t s8 = block_scale(ab, T, K);
    const float4 q = T.dq[s8];
    const float d = q.x;
    c[0] = c[1] = 0;
    if (d == 0.0f) return s8;
    float x[16], t[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(b.w[i] << 16);
        x[2 * i + 1] = __uint_as_float(b.w[i] & 0xFFFF0000u);
    }
    if (q.w != 0.0f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) mul_f32x2(x[2 * i], x[2 * i + 1], q.y, t[2 * i], t[2 * i + 1]);
        c[0] = e2m1x8(t);
        c[1] = e2m1x8(t + 8);
#pragma unroll
        for (int i = 0; i < 8; ++i) mul_f32x2(x[2 * i], x[2 * i + 1], q.z, t[2 * i], t[2 * i + 1]);
        const uint32_t diff0 = c[0] ^ e2m1x8(t), diff1 = c[1] ^ e2m1x8(t + 8);
        if ((diff0 | diff1) == 0) return s8;
        // near-tie elements only: the IEEE quotient decides
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t sh = 4 * (i & 7);
            uint32_t& ci = c[i >> 3];
            if ((((i < 8) ? diff0 : diff1) >> sh) & 0xFu)
                ci = (ci & ~(0xFu << sh)) | (e2m1_exact(x[i], d) << sh);
        }
        return s8;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) t[i] = __fdiv_rn(x[i], d);
    c[0] = e2m1x8(t);
    c[1] = e2m1x8(t + 8);
    return s8;
}

template <bool kWide>
__device__ __forceinline__ void load_block(const uint8_t* p, Block16& b) {
    if constexpr (kWide) {
        asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(b.w[0]), "=r"(b.w[1]), "=r"(b.w[2]), "=r"(b.w[3]), "=r"(b.w[4]),
                       "=r"(b.w[5]), "=r"(b.w[6]), "=r"(b.w[7])
                     : "l"(p));
    } else {
        const uint4 lo = ld_stream(p), hi = ld_stream(p + 16);
        b.w[0] = lo.x, b.w[1] = lo.y, b.w[2] = lo.z, b.w[3] = lo.w;
        b.w[4] = hi.x, b.w[5] = hi.y, b.w[6] = hi.z, b.w[7] = hi.w;
    }
}

template <bool kWide>
__global__ void __launch_bounds__(kThreads, 4) quantize_kernel(QuantParams p) {
    const int lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;
    const int64_t code_row_bytes = p.cols / 2;
    const int64_t sfcols = p.cols / 16;
    const int64_t nblk = p.cols / 16;

    __shared__ QuantTables T;
    ScaleConsts K;
    K.g = *p.g;
    const float rg = __fdiv_rn(1.0f, K.g);
    K.rg_lo = __fmul_rn(rg, kLo);
    K.rg_hi = __fmul_rn(rg, kHi);
    K.fast = normal_range(rg) && normal_range(K.g);
    for (int i = threadIdx.x; i < 128; i += kThreads) {
        T.div6[i] = __fdiv_rn(1.0f + static_cast<float>(i) * 0.0078125f, 6.0f);
        // per scale byte: d, the two bracketing reciprocals, and whether they
        // are usable (1/d in the normal range); otherwise the block divides
        const float d = __fmul_rn(e4m3_decode(static_cast<uint32_t>(i)), K.g);
        const bool usable = (i != 0) && (i != 127) && d >= 0x1p-120f && d <= 0x1p120f;
        const float rd = usable ? __fdiv_rn(1.0f, d) : 0.0f;
        T.dq[i] = make_float4(d, __fmul_rn(rd, kLo), __fmul_rn(rd, kHi), usable ? 1.0f : 0.0f);
    }
    __syncthreads();

    // Walk (row, chunk) pairs with a stride of nwarps chunks, carrying rows
    // instead of dividing.  Software-pipelined: the next chunk's loads are in
    // flight while the current chunk is quantized.
    const uint32_t cpr = p.chunks_per_row;
    const uint32_t step_r = nwarps / cpr, step_c = nwarps - step_r * cpr;
    uint32_t rl = warp / cpr, ch = warp - rl * cpr;
    Block16 cur[kStepsPerChunk], nxt[kStepsPerChunk];
    auto load_chunk = [&](uint32_t lr, uint32_t lc, Block16 (&dst)[kStepsPerChunk]) {
        const bool ok = lr < p.rows;
        const uint8_t* xrow = p.x + static_cast<int64_t>(lr) * p.ld_bytes;
        const int64_t b0 = static_cast<int64_t>(lc) * (kBlocksPerStep * kStepsPerChunk) + lane;
#pragma unroll
        for (int u = 0; u < kStepsPerChunk; ++u) {
            const int64_t b = b0 + u * kBlocksPerStep;
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[u].w[i] = 0;
            if (ok && b < nblk) load_block<kWide>(xrow + b * 32, dst[u]);
        }
    };
    if (rl < p.rows_walk) load_chunk(rl, ch, cur);
    while (rl < p.rows_walk) {
        uint32_t nr = rl + step_r, nc = ch + step_c;
        if (nc >= cpr) {
            nc -= cpr;
            ++nr;
        }
        if (nr < p.rows_walk) load_chunk(nr, nc, nxt);
        const bool row_ok = rl < p.rows;
        const int64_t r = p.row0 + rl;                               // row of the whole tensor
        const int64_t b0 = static_cast<int64_t>(ch) * (kBlocksPerStep * kStepsPerChunk) + lane;
        uint8_t* crow = p.codes + r * code_row_bytes;
        const uint64_t sf_row = (static_cast<uint64_t>(r >> 7) * p.sf_groups) * 512u +
                                static_cast<uint64_t>(r & 31) * 16u +
                                static_cast<uint64_t>((r >> 5) & 3) * 4u;
#pragma unroll
        for (int u = 0; u < kStepsPerChunk; ++u) {
            const int64_t b = b0 + u * kBlocksPerStep;
            uint32_t c[2];
            const uint32_t s8 = quantize_block(cur[u], T, K, c);
            if (row_ok && b < nblk)
                *reinterpret_cast<uint2*>(crow + b * 8) = make_uint2(c[0], c[1]);
            uint32_t w = s8 << (8 * (lane & 3));
            w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
            w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
            if (p.layout == NVFP4_SF_TCGEN05) {
                const int64_t unit = b >> 2;
                if ((lane & 3) == 0 && unit < p.sf_groups)
                    *reinterpret_cast<uint32_t*>(p.sf + sf_row + unit * 512u) = w;
            } else if (row_ok && b < nblk) {
                p.sf[r * sfcols + b] = static_cast<uint8_t>(s8);
            }
        }
#pragma unroll
        for (int u = 0; u < kStepsPerChunk; ++u) cur[u] = nxt[u];
        rl = nr;
        ch = nc;
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
nvfp4_status current_device_info(DeviceInfo* info) {
    static DeviceInfo cache[kMaxDevices];
    static PerDeviceOnce once;
    int dev = 0;
    nvfp4_status st = current_device(&dev);
    if (st != NVFP4_OK) return st;
    st = once.run(dev, [&] {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        cache[dev] = d;
        return NVFP4_OK;
    });
    if (st != NVFP4_OK) return st;
    *info = cache[dev];
    return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

// ---------------------------------------------------------------------------
// Global scale for callers that cannot allocate: the workspace is a
// file-scope device array (one per device that loads the library), whose
// address host code must obtain with cudaGetSymbolAddress -- the array's name
// in host code is only a host-side stand-in.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES];

// Checks of nvfp4_global_scale's arguments other than the workspace, in the
// order the entry points report them; shared with the no-alloc variant so
// that it too refuses a call before enqueuing anything.
static nvfp4_status global_scale_args(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                      const float* g_out) {
    if (!g_out || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0 && !x) return NVFP4_ERR_INVALID_ARG;
    if (cols % 8 != 0 || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    if (rows > 0 && ld < cols) return NVFP4_ERR_INVALID_ARG;
    if (extent_too_large(rows, ld, 2)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (x && !aligned16(x)) return NVFP4_ERR_ALIGNMENT;
    return NVFP4_OK;
}

static nvfp4_status noalloc_scratch_ptr(void** out) {
    static void* cache[kMaxDevices] = {nullptr};
    static PerDeviceOnce once;
    int dev = 0;
    nvfp4_status st = current_device(&dev);
    if (st != NVFP4_OK) return st;
    st = once.run(dev, [&] {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
        cache[dev] = p;
        return NVFP4_OK;
    });
    if (st != NVFP4_OK) return st;
    *out = cache[dev];
    return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_global_scale_noalloc(const void* x, int64_t rows, int64_t cols,
                                                   int64_t ld, float* g_out, float* amax_out,
                                                   void* stream) {
    static_assert(sizeof(GlobalScaleWorkspace) <= NVFP4_NOALLOC_SCRATCH_BYTES,
                  "scratch array too small for the global-scale workspace");
    if (sizeof(GlobalScaleWorkspace) > NVFP4_NOALLOC_SCRATCH_BYTES) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    // refuse before the memset below is enqueued
    nvfp4_status st = global_scale_args(x, rows, cols, ld, g_out);
    if (st != NVFP4_OK) return st;
    const size_t xbytes = extent_bytes(rows, ld, cols, 2);
    if (overlaps(g_out, 4, x, xbytes) || overlaps(amax_out, 4, x, xbytes)) return NVFP4_ERR_INVALID_ARG;
    void* ws = nullptr;
    st = noalloc_scratch_ptr(&ws);
    if (st != NVFP4_OK) return st;
    // the workspace must start at zero: clear it on the stream (no allocation)
    if (cudaMemsetAsync(ws, 0, sizeof(GlobalScaleWorkspace), as_stream(stream)) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return nvfp4_global_scale(x, rows, cols, ld, g_out, amax_out, ws, stream);
}

extern "C" nvfp4_status nvfp4_sf_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout,
                                       size_t* bytes) {
    if (!bytes || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
    // both below 2^31, so the padded product below cannot overflow
    if (cols % 16 != 0 || rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
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
    if (!workspace) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = global_scale_args(x, rows, cols, ld, g_out);
    if (st != NVFP4_OK) return st;
    if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
    // the last CTA writes the results and then clears the workspace, while
    // other CTAs may still read x
    const size_t xbytes = extent_bytes(rows, ld, cols, 2);
    if (overlaps(g_out, 4, workspace, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES) ||
        overlaps(amax_out, 4, workspace, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES) ||
        overlaps(g_out, 4, x, xbytes) || overlaps(amax_out, 4, x, xbytes))
        return NVFP4_ERR_INVALID_ARG;
    DeviceInfo dev;
    st = current_device_info(&dev);
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
    if (row_offset > total_rows || rows > total_rows - row_offset) return NVFP4_ERR_INVALID_ARG;
    // bounds that keep every size product below inside int64
    if (cols >= (int64_t(1) << 31) || total_rows >= (int64_t(1) << 40) || extent_too_large(rows, ld, 2))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (layout != NVFP4_SF_LINEAR && layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
    if (cols % 32 != 0 || ld % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    const bool last = (row_offset + rows == total_rows);
    const int64_t pad_end = (layout == NVFP4_SF_TCGEN05) ? (total_rows + 127) / 128 * 128 : total_rows;
    const int64_t rows_walk = last ? pad_end - row_offset : rows;
    if (rows_walk == 0 || cols == 0) return NVFP4_OK;
    if (!codes || !sf || (rows > 0 && !x)) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && ld < cols) return NVFP4_ERR_INVALID_ARG;
    if ((x && !aligned16(x)) || !aligned16(codes) || !aligned16(sf)) return NVFP4_ERR_ALIGNMENT;
    // every CTA reads *g while others write codes and scales
    size_t sf_total = 0;
    const nvfp4_status sfst = nvfp4_sf_bytes(total_rows, cols, layout, &sf_total);
    if (sfst != NVFP4_OK) return sfst;
    if (overlaps(g, 4, codes, static_cast<size_t>(total_rows) * static_cast<size_t>(cols / 2)) ||
        overlaps(g, 4, sf, sf_total))
        return NVFP4_ERR_INVALID_ARG;
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
    const int64_t chunks_per_row = (cols / 16 + kBlocksPerStep * kStepsPerChunk - 1) /
                                   (kBlocksPerStep * kStepsPerChunk);
    if (rows_walk * chunks_per_row >= (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    p.rows_walk = static_cast<uint32_t>(rows_walk);
    p.chunks_per_row = static_cast<uint32_t>(chunks_per_row);
    p.sf_groups = static_cast<uint32_t>(units);  // roundup(cols/16, 4) / 4
    DeviceInfo dev;
    nvfp4_status st = current_device_info(&dev);
    if (st != NVFP4_OK) return st;
    const int64_t warps = rows_walk * chunks_per_row;
    int64_t blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t max_blocks = static_cast<int64_t>(dev.sms) * 4;   // one resident wave
    if (blocks > max_blocks) blocks = max_blocks;
    const bool wide = x && (reinterpret_cast<uintptr_t>(x) % 32 == 0) && (ld % 16 == 0);
    if (wide)
        quantize_kernel<true><<<static_cast<int>(blocks), kThreads, 0, as_stream(stream)>>>(p);
    else
        quantize_kernel<false><<<static_cast<int>(blocks), kThreads, 0, as_stream(stream)>>>(p);
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
