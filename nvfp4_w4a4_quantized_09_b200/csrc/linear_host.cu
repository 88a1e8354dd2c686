// linear_host.cu -- the whole W4A4 linear layer from host buffers: the BF16
// activation is copied in, its global scale and NVFP4 codes computed, the
// fused block-scaled GEMM run against a pre-quantized weight, and the BF16
// output copied back, all enqueued on one stream.  Host-side composition of
// the entry points in quantize.cu and gemm.cu; no kernel of its own.
//
// Source: the serving path of the pages' recipe -- W4A4 on every linear layer
// with per-module global scales in the fused GEMM (chatpaper.ai abstract;
// evolve.pub review, Scope & Claims).
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_common.h"
#include "nvfp4.h"

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_fused_linear_host(const void* x_host, int64_t M, int64_t K,
                                                const uint8_t* w_codes, const uint8_t* w_sf,
                                                const nvfp4_segment* segs, int nseg,
                                                void* y_host, void* x_dev, uint8_t* a_codes,
                                                uint8_t* a_sf, float* a_g, float* a_amax,
                                                void* workspace, void* y_dev, void* stream) {
    // Everything the composed calls check is checked here first, so that a
    // refused call enqueues nothing (not even the copy in).
    if (!segs || nseg < 1 || nseg > NVFP4_MAX_SEGMENTS || M < 0 || K < 0) return NVFP4_ERR_INVALID_ARG;
    int64_t N = 0;
    for (int s = 0; s < nseg; ++s) {
        if (segs[s].n_offset != N || segs[s].n_size <= 0 || !segs[s].w_gscale)
            return NVFP4_ERR_INVALID_ARG;
        if (segs[s].n_size >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
        N += segs[s].n_size;
    }
    if (K % 32 != 0 || K < 32 || M >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) ||
        N >= (int64_t(1) << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (extent_too_large(M, K, 2) || extent_too_large(M, N, 2)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    // the quantizer's bound on its work items (128-row padded rows x
    // 1024-element chunks per row)
    if ((M + 127) / 128 * 128 * ((K / 16 + 63) / 64) >= (int64_t(1) << 30))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return NVFP4_OK;
    if (!x_host || !y_host || !x_dev || !a_codes || !a_sf || !a_g || !workspace || !y_dev ||
        !w_codes || !w_sf)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_dev) || !aligned16(a_codes) || !aligned16(a_sf) || !aligned16(workspace) ||
        !aligned16(y_dev) || !aligned16(w_codes) || !aligned16(w_sf) || N % 8 != 0)
        return NVFP4_ERR_ALIGNMENT;
    const size_t x_bytes = static_cast<size_t>(M) * static_cast<size_t>(K) * 2;
    const size_t y_bytes = static_cast<size_t>(M) * static_cast<size_t>(N) * 2;
    const size_t code_bytes = static_cast<size_t>(M) * static_cast<size_t>(K / 2);
    size_t sf_bytes = 0;
    {
        const nvfp4_status sst = nvfp4_sf_bytes(M, K, NVFP4_SF_TCGEN05, &sf_bytes);
        if (sst != NVFP4_OK) return sst;
    }
    if (overlaps(a_g, 4, workspace, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES) ||
        overlaps(a_amax, 4, workspace, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES) ||
        overlaps(a_g, 4, x_dev, x_bytes) || overlaps(a_amax, 4, x_dev, x_bytes) ||
        overlaps(a_g, 4, a_codes, code_bytes) || overlaps(a_g, 4, a_sf, sf_bytes) ||
        overlaps(a_g, 4, y_dev, y_bytes) || overlaps(x_dev, x_bytes, y_dev, y_bytes))
        return NVFP4_ERR_INVALID_ARG;
    for (int s = 0; s < nseg; ++s)
        if (overlaps(segs[s].w_gscale, 4, y_dev, y_bytes)) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo dev;
    nvfp4_status st = require_sm100(&dev);
    if (st != NVFP4_OK) return st;

    cudaStream_t cs = as_stream(stream);
    if (cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    st = nvfp4_global_scale(x_dev, M, K, K, a_g, a_amax, workspace, stream);
    if (st != NVFP4_OK) return st;
    st = nvfp4_quantize(x_dev, M, K, K, a_g, a_codes, a_sf, NVFP4_SF_TCGEN05, stream);
    if (st != NVFP4_OK) return st;
    st = nvfp4_fused_gemm(a_codes, a_sf, a_g, w_codes, w_sf, segs, nseg, y_dev, N, M, K, stream);
    if (st != NVFP4_OK) return st;
    if (cudaMemcpyAsync(y_host, y_dev, y_bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}
