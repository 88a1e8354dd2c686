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

namespace {

// Sizes of a host-buffer call, filled by linear_host_check.
struct LinearHostPlan {
    int64_t N = 0;
    size_t x_bytes = 0, y_bytes = 0, code_bytes = 0, sf_bytes = 0;
};

// Every check the composed calls make, made first so that a refused call
// enqueues nothing (not even the copy in).  NVFP4_OK with plan->N set; M == 0
// is accepted here and enqueues nothing in the callers.
nvfp4_status linear_host_check(const void* x_host, int64_t M, int64_t K, const uint8_t* w_codes,
                               const uint8_t* w_sf, const nvfp4_segment* segs, int nseg,
                               const void* y_host, const void* x_dev, const uint8_t* a_codes,
                               const uint8_t* a_sf, const float* a_g, const float* a_amax,
                               const void* workspace, const void* y_dev, LinearHostPlan* plan) {
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
    plan->N = N;
    if (M == 0) return NVFP4_OK;
    if (!x_host || !y_host || !x_dev || !a_codes || !a_sf || !a_g || !workspace || !y_dev ||
        !w_codes || !w_sf)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_dev) || !aligned16(a_codes) || !aligned16(a_sf) || !aligned16(workspace) ||
        !aligned16(y_dev) || !aligned16(w_codes) || !aligned16(w_sf) || N % 8 != 0)
        return NVFP4_ERR_ALIGNMENT;
    plan->x_bytes = static_cast<size_t>(M) * static_cast<size_t>(K) * 2;
    plan->y_bytes = static_cast<size_t>(M) * static_cast<size_t>(N) * 2;
    plan->code_bytes = static_cast<size_t>(M) * static_cast<size_t>(K / 2);
    {
        const nvfp4_status sst = nvfp4_sf_bytes(M, K, NVFP4_SF_TCGEN05, &plan->sf_bytes);
        if (sst != NVFP4_OK) return sst;
    }
    const size_t xb = plan->x_bytes, yb = plan->y_bytes;
    if (overlaps(a_g, 4, workspace, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES) ||
        overlaps(a_amax, 4, workspace, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES) ||
        overlaps(a_g, 4, x_dev, xb) || overlaps(a_amax, 4, x_dev, xb) ||
        overlaps(a_g, 4, a_codes, plan->code_bytes) || overlaps(a_g, 4, a_sf, plan->sf_bytes) ||
        overlaps(a_g, 4, y_dev, yb) || overlaps(x_dev, xb, y_dev, yb) ||
        overlaps(x_dev, xb, a_codes, plan->code_bytes) || overlaps(x_dev, xb, a_sf, plan->sf_bytes))
        return NVFP4_ERR_INVALID_ARG;
    for (int s = 0; s < nseg; ++s)
        if (overlaps(segs[s].w_gscale, 4, y_dev, yb)) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo dev;
    return require_sm100(&dev);
}

// Copy in, global scale and quantization of the activation, on `stream`.
nvfp4_status enqueue_input(const void* x_host, int64_t M, int64_t K, size_t x_bytes, void* x_dev,
                           uint8_t* a_codes, uint8_t* a_sf, float* a_g, float* a_amax,
                           void* workspace, void* stream) {
    if (cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, as_stream(stream)) !=
        cudaSuccess)
        return NVFP4_ERR_CUDA;
    nvfp4_status st = nvfp4_global_scale(x_dev, M, K, K, a_g, a_amax, workspace, stream);
    if (st != NVFP4_OK) return st;
    return nvfp4_quantize(x_dev, M, K, K, a_g, a_codes, a_sf, NVFP4_SF_TCGEN05, stream);
}

// Rows of each GEMM slice of the overlapped call: about kOverlapRows, a
// multiple of 256, and never 256 rows or fewer (the GEMM kernel is chosen by
// M alone, so every slice runs the kernel the whole M would, and each output
// is accumulated exactly as in the one-launch GEMM).
constexpr int64_t kOverlapRows = 2048;

}  // namespace

extern "C" nvfp4_status nvfp4_fused_linear_host(const void* x_host, int64_t M, int64_t K,
                                                const uint8_t* w_codes, const uint8_t* w_sf,
                                                const nvfp4_segment* segs, int nseg,
                                                void* y_host, void* x_dev, uint8_t* a_codes,
                                                uint8_t* a_sf, float* a_g, float* a_amax,
                                                void* workspace, void* y_dev, void* stream) {
    LinearHostPlan plan;
    nvfp4_status st = linear_host_check(x_host, M, K, w_codes, w_sf, segs, nseg, y_host, x_dev,
                                        a_codes, a_sf, a_g, a_amax, workspace, y_dev, &plan);
    if (st != NVFP4_OK || M == 0) return st;
    st = enqueue_input(x_host, M, K, plan.x_bytes, x_dev, a_codes, a_sf, a_g, a_amax, workspace,
                       stream);
    if (st != NVFP4_OK) return st;
    st = nvfp4_fused_gemm(a_codes, a_sf, a_g, w_codes, w_sf, segs, nseg, y_dev, plan.N, M, K, stream);
    if (st != NVFP4_OK) return st;
    if (cudaMemcpyAsync(y_host, y_dev, plan.y_bytes, cudaMemcpyDeviceToHost, as_stream(stream)) !=
        cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_fused_linear_host_overlap(
    const void* x_host, int64_t M, int64_t K, const uint8_t* w_codes, const uint8_t* w_sf,
    const nvfp4_segment* segs, int nseg, void* y_host, void* x_dev, uint8_t* a_codes,
    uint8_t* a_sf, float* a_g, float* a_amax, void* workspace, void* y_dev, void* stream,
    void* copy_stream) {
    LinearHostPlan plan;
    nvfp4_status st = linear_host_check(x_host, M, K, w_codes, w_sf, segs, nseg, y_host, x_dev,
                                        a_codes, a_sf, a_g, a_amax, workspace, y_dev, &plan);
    if (st != NVFP4_OK || M == 0) return st;
    cudaEvent_t ev;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return NVFP4_ERR_CUDA;
    cudaStream_t cs = as_stream(stream), co = as_stream(copy_stream);
    st = enqueue_input(x_host, M, K, plan.x_bytes, x_dev, a_codes, a_sf, a_g, a_amax, workspace,
                       stream);
    // y_dev is rewritten below: first let every copy already enqueued on
    // copy_stream (the previous call's output) finish.  Only the GEMM waits;
    // this call's copy in and quantization above overlap those copies.
    if (st == NVFP4_OK &&
        (cudaEventRecord(ev, co) != cudaSuccess || cudaStreamWaitEvent(cs, ev, 0) != cudaSuccess))
        st = NVFP4_ERR_CUDA;
    const int64_t sf_rowblock_bytes = (K / 16 + 3) / 4 * 4 * 128;
    for (int64_t r0 = 0; st == NVFP4_OK && r0 < M;) {
        int64_t mc = M - r0;
        if (mc > kOverlapRows + kOverlapRows / 2) mc = kOverlapRows;   // else: the rest in one slice
        st = nvfp4_fused_gemm(a_codes + r0 * (K / 2), a_sf + (r0 / 128) * sf_rowblock_bytes, a_g,
                              w_codes, w_sf, segs, nseg,
                              static_cast<uint16_t*>(y_dev) + r0 * plan.N, plan.N, mc, K, stream);
        if (st != NVFP4_OK) break;
        // the slice's copy out starts as soon as its GEMM is done, while the
        // next slice computes
        if (cudaEventRecord(ev, cs) != cudaSuccess || cudaStreamWaitEvent(co, ev, 0) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<uint16_t*>(y_host) + r0 * plan.N,
                            static_cast<const uint16_t*>(y_dev) + r0 * plan.N,
                            static_cast<size_t>(mc) * plan.N * 2, cudaMemcpyDeviceToHost, co) !=
                cudaSuccess)
            st = NVFP4_ERR_CUDA;
        r0 += mc;
    }
    // the event may be released now: its pending records and waits complete
    // on their own
    cudaEventDestroy(ev);
    return st;
}
