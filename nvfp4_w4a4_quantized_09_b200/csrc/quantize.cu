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
// Every result equals the binary32 step sequence exactly, with no IEEE
// division and no per-element branch on the fast path:
//  * fl32(ab / 6): ab is BF16, i.e. (1 + m/128) * 2^e, and rounding commutes
//    with scaling by 2^e, so it is a 128-entry table of RN((1 + m/128) / 6)
//    with e added to the exponent (tiny ab take the IEEE division).
//  * fl32(u / g) and fl32(x / d): with r = RN(1/v) and q0 = RN(a * r), the
//    remainder a - q0 * v is exact in one FMA, and RN(q0 + (a - q0 * v) * r)
//    is the correctly rounded quotient (Markstein's theorem: P. Markstein,
//    "Computation of elementary functions on the IBM RISC System/6000
//    processor", IBM J. Res. Dev. 34(1), 1990) provided no step over- or
//    underflows.  The per-scale-byte table marks the d that keep every step in
//    range; a block whose largest quotient could overflow, and every quotient
//    outside those ranges, takes the IEEE division instead.
//  * The element quotient is formed from -x (one integer operation on the
//    BF16 bits) and -RN(1/d): q0 = (-x)(-r), e = q0 d + (-x), q = q0 + e (-r).
//    Each step is the exact negation image of the textbook sequence, and the
//    signed zeros come out as IEEE division gives them: x = -0 yields -0 (code
//    0x8), x = +0 yields +0.
// The conversions run on a narrow pipe, so each is used once per value: one
// E2M1 pair conversion per two elements, one E4M3 pair conversion per two
// blocks.
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

// Two UE4M3 encodes (round to nearest even, saturate at 448) of non-negative
// floats at once: low byte from a, high byte from b.  The hardware conversion
// is exact RNE.
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

struct Block16 {
    uint32_t w[8];  // 16 BF16 values, element 2i in the low half of w[i]
};

// Per-CTA tables, built from g at kernel start.
struct QuantTables {
    float div6[128];     // RN((1 + m/128) / 6)
    float4 dq[128];      // per scale byte: d = fl32(E4M3 * g), -RN(1/d), the largest block
                         // max the fast path takes (0: never), unused
};

// Kernel-wide constants derived from g.
struct ScaleConsts {
    float g;
    float rg;             // RN(1/g)
    bool fast;            // g and 1/g in the normal range
};

__device__ __forceinline__ bool normal_range(float v) {
    const float a = fabsf(v);
    return a >= 0x1p-125f && a <= 0x1p125f;
}

// fl32(fl32(ab / 6) / g), clamped to 1024 (any value from 464 up encodes to
// 448, so the clamp changes no scale byte and keeps overflow away from the
// encoder).  Fast path: ab >= 2^-97 (so fl32(ab/6) >= 2^-100 and the table
// holds it) and g, 1/g normal; everything else divides.
__device__ __forceinline__ float block_quotient(float ab, const QuantTables& T,
                                                const ScaleConsts& K) {
    const uint32_t abits = __float_as_uint(ab);
    float q;
    if (K.fast && abits >= 0x0F000000u) {
        const uint32_t e = abits >> 23, m7 = (abits >> 16) & 127u;
        const float u = __uint_as_float(__float_as_uint(T.div6[m7]) + ((e - 127u) << 23));
        const float q0 = __fmul_rn(u, K.rg);
        const float r = __fmaf_rn(-q0, K.g, u);
        q = __fmaf_rn(r, K.rg, q0);
    } else {
        if (abits == 0) return 0.0f;
        const float u = abits >= 0x04000000u   // ab >= 2^-119: exact table path
            ? __uint_as_float(__float_as_uint(T.div6[(abits >> 16) & 127u]) + (((abits >> 23) - 127u) << 23))
            : __fdiv_rn(ab, 6.0f);
        q = __fdiv_rn(u, K.g);
    }
    return fminf(q, 1024.0f);
}

// 16 E2M1 codes of fl32(x / d) for one block whose scale byte is s8.
__device__ __forceinline__ void encode_block(const Block16& b, float ab, uint32_t s8,
                                             const QuantTables& T, uint32_t (&c)[2]) {
    const float4 q = T.dq[s8];
    const float d = q.x;
    float t[16];
    if (ab < q.z) {
        // d and 1/d in range and no quotient of the block can overflow
        const uint64_t NR = f32x2(__float_as_uint(q.y), __float_as_uint(q.y));
        const uint64_t D = f32x2(__float_as_uint(d), __float_as_uint(d));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w = b.w[i];
            // -x of both elements: the BF16 bits moved into place, sign flipped
            const uint64_t nx = f32x2(w * 0x10000u + 0x80000000u, (w & 0xFFFF0000u) ^ 0x80000000u);
            const uint64_t q0 = mul_f32x2(nx, NR);
            const uint64_t e = fma_f32x2(q0, D, nx);
            const uint64_t q1 = fma_f32x2(e, NR, q0);
            t[2 * i] = __uint_as_float(static_cast<uint32_t>(q1));
            t[2 * i + 1] = __uint_as_float(static_cast<uint32_t>(q1 >> 32));
        }
    } else if (d == 0.0f) {
        c[0] = c[1] = 0;     // zero block or a scale that underflowed: every code 0
        return;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            t[2 * i] = __fdiv_rn(__uint_as_float(b.w[i] << 16), d);
            t[2 * i + 1] = __fdiv_rn(__uint_as_float(b.w[i] & 0xFFFF0000u), d);
        }
    }
    c[0] = e2m1x8(t);
    c[1] = e2m1x8(t + 8);
}

__device__ __forceinline__ float block_absmax(const Block16& b) {
    uint32_t m = absmax_bf16x2(b.w[0], b.w[1]);
#pragma unroll
    for (int i = 2; i < 8; ++i) m = absmax_bf16x2(m, b.w[i]);
    return __uint_as_float(max(m & 0x7FFFu, (m >> 16) & 0x7FFFu) << 16);
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

#ifndef NVFP4_Q_MINB
#define NVFP4_Q_MINB 3
#endif
// Resident CTAs of the quantizer per SM (one wave of the grid).
constexpr int kQuantCtasPerSm = NVFP4_Q_MINB;

// A warp quantizes chunks of 64 consecutive blocks of one row: lane l holds
// blocks l and 32 + l (each load instruction reads 1 KB of contiguous bytes
// and each code store writes 256).  Warps walk (row, chunk) pairs with the
// grid's warp count as stride, carrying rows instead of dividing, and load
// the next chunk while the current one is quantized.  The row is uniform over
// the warp, so the checks for padding rows are uniform branches.  kFull: the
// blocks per row are a multiple of 64, so no chunk is ragged.
template <bool kWide, bool kFull>
__device__ __forceinline__ void load_chunk(const QuantParams& p, uint32_t rl, uint32_t ch,
                                           int lane, Block16 (&dst)[kStepsPerChunk]) {
    const int64_t nblk = p.cols / 16;
    const uint8_t* xrow = p.x + static_cast<int64_t>(rl) * p.ld_bytes;
    const int64_t b0 = static_cast<int64_t>(ch) * (kBlocksPerStep * kStepsPerChunk) + lane;
    if (kFull && rl < p.rows) {
#pragma unroll
        for (int u = 0; u < kStepsPerChunk; ++u) load_block<kWide>(xrow + (b0 + u * kBlocksPerStep) * 32, dst[u]);
        return;
    }
#pragma unroll
    for (int u = 0; u < kStepsPerChunk; ++u) {
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[u].w[i] = 0;
        const int64_t b = b0 + u * kBlocksPerStep;
        if (rl < p.rows && b < nblk) load_block<kWide>(xrow + b * 32, dst[u]);
    }
}

template <bool kWide, bool kFull>
__global__ void __launch_bounds__(kThreads, kQuantCtasPerSm) quantize_kernel(QuantParams p) {
    const int lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;
    const int64_t code_row_bytes = p.cols / 2;
    const int64_t nblk = p.cols / 16;

    __shared__ QuantTables T;
    ScaleConsts K;
    K.g = *p.g;
    K.rg = __fdiv_rn(1.0f, K.g);
    K.fast = normal_range(K.rg) && normal_range(K.g);
    for (int i = threadIdx.x; i < 128; i += kThreads) {
        T.div6[i] = __fdiv_rn(1.0f + static_cast<float>(i) * 0.0078125f, 6.0f);
        // per scale byte: d, -RN(1/d), and the block max below which the fast
        // path is exact: d in [2^-96, 2^100] and ab * RN(1/d) < 2^126
        const float d = __fmul_rn(e4m3_decode(static_cast<uint32_t>(i)), K.g);
        const bool usable = (i != 0) && (i != 127) && d >= 0x1p-96f && d <= 0x1p100f;
        T.dq[i] = make_float4(d, usable ? -__fdiv_rn(1.0f, d) : 0.0f,
                              usable ? __fmul_rn(d, 0x1p125f) : 0.0f, 0.0f);
    }
    __syncthreads();

    const uint32_t cpr = p.chunks_per_row;
    const uint32_t step_r = nwarps / cpr, step_c = nwarps - step_r * cpr;
    uint32_t rl = warp / cpr, ch = warp - rl * cpr;
    Block16 cur[kStepsPerChunk], nxt[kStepsPerChunk];
    if (rl < p.rows_walk) load_chunk<kWide, kFull>(p, rl, ch, lane, cur);
    while (rl < p.rows_walk) {
        uint32_t nr = rl + step_r, nc = ch + step_c;
        if (nc >= cpr) {
            nc -= cpr;
            ++nr;
        }
        if (nr < p.rows_walk) load_chunk<kWide, kFull>(p, nr, nc, lane, nxt);

        static_assert(kStepsPerChunk == 2, "scale bytes are converted and gathered in pairs");
        const float ab0 = block_absmax(cur[0]), ab1 = block_absmax(cur[1]);
        // s8 of block l (low byte) and of block 32 + l (high byte)
        const uint32_t s8pair = e4m3x2_rne_satfinite(block_quotient(ab0, T, K), block_quotient(ab1, T, K));
        uint32_t c0[2], c1[2];
        encode_block(cur[0], ab0, s8pair & 0xFFu, T, c0);
        encode_block(cur[1], ab1, s8pair >> 8, T, c1);

        const int64_t r = p.row0 + rl;                               // row of the whole tensor
        const int64_t b0 = static_cast<int64_t>(ch) * (kBlocksPerStep * kStepsPerChunk) + lane;
        if (rl < p.rows) {
            uint8_t* crow = p.codes + r * code_row_bytes;
            if (kFull || b0 < nblk) *reinterpret_cast<uint2*>(crow + b0 * 8) = make_uint2(c0[0], c0[1]);
            if (kFull || b0 + kBlocksPerStep < nblk)
                *reinterpret_cast<uint2*>(crow + (b0 + kBlocksPerStep) * 8) = make_uint2(c1[0], c1[1]);
        }
        if (p.layout == NVFP4_SF_TCGEN05) {
            // One word of the tensor-core layout is the scale bytes of four
            // consecutive blocks (lanes 4j..4j+3 of one step).  Both steps'
            // words are gathered with two shuffles: lane 4j stores the step-0
            // word of unit j, lane 4j+2 the step-1 word of unit 8 + j.
            const uint32_t v = (s8pair & 0xFFu) | ((s8pair & 0xFF00u) << 8);   // bytes s0, 0, s1, 0
            uint32_t x = v << (8 * (lane & 1));
            x |= __shfl_xor_sync(0xFFFFFFFFu, x, 1);                       // s0 s0' s1 s1' of a lane pair
            const uint32_t y = __shfl_xor_sync(0xFFFFFFFFu, x, 2);
            const int64_t unit0 = static_cast<int64_t>(ch) * 16 + (lane >> 2);
            const uint64_t sf_row = (static_cast<uint64_t>(r >> 7) * p.sf_groups) * 512u +
                                    static_cast<uint64_t>(r & 31) * 16u +
                                    static_cast<uint64_t>((r >> 5) & 3) * 4u;
            if ((lane & 3) == 0) {
                if (kFull || unit0 < p.sf_groups)
                    *reinterpret_cast<uint32_t*>(p.sf + sf_row + unit0 * 512u) = __byte_perm(x, y, 0x5410);
            } else if ((lane & 3) == 2) {
                if (kFull || unit0 + 8 < p.sf_groups)
                    *reinterpret_cast<uint32_t*>(p.sf + sf_row + (unit0 + 8) * 512u) = __byte_perm(y, x, 0x7632);
            }
        } else if (rl < p.rows) {
            if (kFull || b0 < nblk) p.sf[r * nblk + b0] = static_cast<uint8_t>(s8pair);
            if (kFull || b0 + kBlocksPerStep < nblk)
                p.sf[r * nblk + b0 + kBlocksPerStep] = static_cast<uint8_t>(s8pair >> 8);
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
    const size_t code_total = static_cast<size_t>(total_rows) * static_cast<size_t>(cols / 2);
    if (overlaps(g, 4, codes, code_total) || overlaps(g, 4, sf, sf_total))
        return NVFP4_ERR_INVALID_ARG;
    // CTAs read x while others write codes and scales: outputs may not alias it
    {
        const size_t xbytes = extent_bytes(rows, ld, cols, 2);
        if (overlaps(x, xbytes, codes, code_total) || overlaps(x, xbytes, sf, sf_total))
            return NVFP4_ERR_INVALID_ARG;
    }
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
    const int64_t units = (cols + 63) / 64;                 // = roundup(cols/16, 4) / 4
    const int64_t chunks_per_row = (cols / 16 + kBlocksPerStep * kStepsPerChunk - 1) /
                                   (kBlocksPerStep * kStepsPerChunk);
    if (rows_walk * chunks_per_row >= (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    p.rows_walk = static_cast<uint32_t>(rows_walk);
    p.chunks_per_row = static_cast<uint32_t>(chunks_per_row);
    p.sf_groups = static_cast<uint32_t>(units);
    DeviceInfo dev;
    nvfp4_status st = current_device_info(&dev);
    if (st != NVFP4_OK) return st;
    const int64_t warps = rows_walk * chunks_per_row;
    int64_t blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t max_blocks = static_cast<int64_t>(dev.sms) * kQuantCtasPerSm;   // one resident wave
    if (blocks > max_blocks) blocks = max_blocks;
    const bool wide = x && (reinterpret_cast<uintptr_t>(x) % 32 == 0) && (ld % 16 == 0);
    const bool full = (cols / 16) % (kBlocksPerStep * kStepsPerChunk) == 0;
    const dim3 grid(static_cast<unsigned>(blocks)), block(kThreads);
    cudaStream_t cs = as_stream(stream);
    if (wide && full) quantize_kernel<true, true><<<grid, block, 0, cs>>>(p);
    else if (wide) quantize_kernel<true, false><<<grid, block, 0, cs>>>(p);
    else if (full) quantize_kernel<false, true><<<grid, block, 0, cs>>>(p);
    else quantize_kernel<false, false><<<grid, block, 0, cs>>>(p);
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
