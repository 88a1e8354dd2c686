/*
 * nvfp4.h -- C ABI of the NVFP4 W4A4 quantized linear layer for B200 (sm_100a).
 *
 * The layer follows the pages on "Why Gated DeltaNet Survives 4-Bit
 * Quantization: NVFP4 W4A4 for the Recurrent Half of a Hybrid 27B LLM":
 *   - every linear layer runs with 4-bit weights AND activations (chatpaper.ai
 *     abstract: the paper quantizes every one of its model's 496 linear
 *     layers this way);
 *   - NVFP4 = 4-bit E2M1 elements, each group of 16 consecutive elements
 *     sharing one E4M3 scale
 *     (evolve.pub review, Scope & Claims; thevalue.engineering, second section);
 *   - the GEMM runs natively on NVFP4-capable hardware (evolve.pub FAQ);
 *   - modules fused into one GEMM keep their own global scales, which is the
 *     global-scale mismatch the paper repairs (chatpaper.ai abstract;
 *     evolve.pub Key claims, fourth bullet).
 *
 * Conventions shared by every entry point:
 *   - Pointers marked (device) are CUDA device pointers on the current device;
 *     (host) pointers are read during the call only -- except the activation
 *     and output of nvfp4_fused_linear_host, which its stream's copies use
 *     until they complete.  The caller allocates and
 *     owns every buffer; the library allocates no device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; nothing synchronizes except
 *     nvfp4_last_device_status().  Global scales stay in device memory, so a
 *     whole layer runs without a host round trip.
 *   - Argument checks happen on the host before anything is enqueued; a
 *     failing check returns an error status and enqueues nothing.  A CUDA
 *     launch error returns NVFP4_ERR_CUDA.  No C++ exception crosses the ABI.
 *     Sizes are bounded before any arithmetic on them: a strided buffer that
 *     would span more than 2^48 bytes, and M, N, K or a segment at or above
 *     2^31, give NVFP4_ERR_UNSUPPORTED_SHAPE.  The library cannot see how
 *     large a buffer is: each entry point states the bytes it reads and
 *     writes, and the caller provides at least that many.
 *   - Every entry point may be called from several host threads; the
 *     per-device state the library caches (device properties, symbol
 *     addresses, kernel attributes) is set up once under a lock.
 *   - BF16 tensors are row-major with a row stride `ld` in elements.
 *   - Packed codes: two E2M1 codes per byte, element 2j in the low nibble of
 *     byte j (sign in bit 3 of each nibble); a [rows, cols] tensor occupies
 *     rows * cols/2 contiguous bytes.
 *   - Block scales: unsigned E4M3 bytes (largest 448 = 0x7E), one per 16
 *     consecutive elements of a row.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum  */
    NVFP4_ERR_ALIGNMENT = 2,         /* pointer or stride not 16-byte aligned  */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 3, /* shape outside what the kernels accept  */
    NVFP4_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed      */
    NVFP4_ERR_TIMEOUT = 5,           /* a bounded device-side wait gave up     */
    NVFP4_ERR_DEVICE = 6             /* current device is not sm_100           */
} nvfp4_status;

typedef enum {
    /* [rows, cols/16] bytes, row-major, no padding. */
    NVFP4_SF_LINEAR = 0,
    /* The block-scaled tensor-core layout the GEMM consumes: rows padded to a
     * multiple of 128, scale columns to a multiple of 4; each 128-row x
     * 4-column group is a 512-byte atom, atoms ordered with the scale-column
     * group fastest; inside an atom, scale (r, c) sits at byte
     * (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4).  Padding bytes are 0. */
    NVFP4_SF_TCGEN05 = 1
} nvfp4_sf_layout;

/* One module of a fused weight: rows [n_offset, n_offset + n_size) of the
 * concatenated weight (= output columns of the GEMM) use the FP32 global
 * scale at w_gscale (device pointer). */
typedef struct {
    int64_t n_offset;
    int64_t n_size;
    const float* w_gscale;
} nvfp4_segment;

#define NVFP4_MAX_SEGMENTS 16

/* Elementwise function a fused GEMM may apply to one segment's outputs after
 * the global scales (see nvfp4_fused_gemm_act). */
typedef enum {
    NVFP4_ACT_NONE = 0,
    /* Gated DeltaNet log-space decay gate, per column c of the segment:
     * g = -exp(a_log[c]) * softplus(y + dt_bias[c]), softplus(z) = log(1 + e^z). */
    NVFP4_ACT_DECAY_GATE = 1,
    /* Gated DeltaNet write strength: beta = 1 / (1 + e^-y). */
    NVFP4_ACT_SIGMOID = 2
} nvfp4_act_kind;

typedef struct {
    int kind;              /* nvfp4_act_kind */
    const float* a_log;    /* NVFP4_ACT_DECAY_GATE: device FP32 [n_size], else unused */
    const float* dt_bias;  /* NVFP4_ACT_DECAY_GATE: device FP32 [n_size], else unused */
} nvfp4_segment_act;
/* Bytes of the zero-initialised workspace nvfp4_global_scale needs. */
#define NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES 256

/* Per-tensor FP32 global scale from the absolute maximum.
 *   amax = max |x| over x[rows, cols] (BF16, row stride ld, device);
 *   g = fl32(amax / 2688) (2688 = 6 * 448, the largest E2M1 value times the
 *   largest E4M3 scale); g = 1 when amax == 0.
 * g_out (device, 1 float) receives g; amax_out (device, 1 float) receives
 * amax, or may be NULL.  workspace (device, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES,
 * 16-byte aligned) must be zero before the first call; every call leaves it
 * zero again.  Calls that share a workspace must not overlap in time, and
 * g_out / amax_out must lie outside it (NVFP4_ERR_INVALID_ARG otherwise).
 * Requirements: cols % 8 == 0, ld % 8 == 0, ld >= cols, x 16-byte aligned.
 * rows == 0 or cols == 0 yields amax = 0, g = 1.
 * Errors: NVFP4_ERR_INVALID_ARG (null g_out or workspace, negative size,
 * ld < cols, a result inside the workspace or inside x), NVFP4_ERR_ALIGNMENT
 * (cols, ld, x or workspace), NVFP4_ERR_UNSUPPORTED_SHAPE (the size bounds),
 * CUDA errors.
 * Source: the per-module global scale behind the fused-GEMM repair
 * (chatpaper.ai abstract); absmax is the dynamic reading of it. */
nvfp4_status nvfp4_global_scale(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                float* g_out, float* amax_out, void* workspace,
                                void* stream);

/* Bytes of the library-owned scratch array behind nvfp4_global_scale_noalloc. */
#define NVFP4_NOALLOC_SCRATCH_BYTES 256

/* nvfp4_global_scale without a caller workspace, for callers that cannot
 * allocate device memory -- for example code plugged into a host framework
 * whose memory pool forbids outside cudaMalloc calls, or a hook that runs
 * where allocation is not permitted -- and so cannot hand over the
 * zero-initialised workspace nvfp4_global_scale needs.  The paper has no
 * counterpart; this is a property of the library, not of the method.
 * The workspace lives instead in a file-scope __device__ array of
 * NVFP4_NOALLOC_SCRATCH_BYTES bytes that every GPU loading the library holds
 * until the process exits; the call needs 8 of those bytes and returns
 * NVFP4_ERR_UNSUPPORTED_SHAPE if its need ever exceeded the array.  The call
 * allocates nothing (no cudaMalloc, no allocating library routine): it
 * clears the part of the array that must start at zero with a
 * cudaMemsetAsync on `stream`, then launches the same kernel as
 * nvfp4_global_scale.  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture.  All calls on a device share the one
 * array, which keeps the last call's contents: calls that overlap on the GPU
 * (different streams, no ordering between them) race and may return a wrong
 * g; serialize them.  Arguments, results, requirements and errors as
 * nvfp4_global_scale, without `workspace`.  No passage of the pages defines
 * this entry point: it exists for callers of the library, not for the method. */
nvfp4_status nvfp4_global_scale_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                        float* g_out, float* amax_out, void* stream);

/* Bytes of the scale buffer for a [rows, cols] tensor in `layout`:
 * LINEAR rows * cols/16; TCGEN05 roundup(rows,128) * roundup(cols/16,4).
 * cols must be a multiple of 16, and rows and cols below 2^31
 * (NVFP4_ERR_UNSUPPORTED_SHAPE otherwise). */
nvfp4_status nvfp4_sf_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout,
                            size_t* bytes);

/* 16-element block quantization of x[rows, cols] (BF16, row stride ld, device)
 * under the global scale *g (device).  Per row and 16-block:
 *   s8 = E4M3_RNE_satfinite(fl32(fl32(blockmax / 6) / g)),
 *   d = fl32(E4M3(s8) * g), code = E2M1_RNE_satfinite(fl32(x / d)),
 *   all codes 0 when d == 0; a negative value that rounds to 0 keeps its
 *   sign (code 8).
 * codes (device, rows * cols/2 bytes) and sf (device, nvfp4_sf_bytes bytes in
 * `layout`) are written completely, padding included.
 * Requirements: cols % 32 == 0, ld % 8 == 0, ld >= cols; x, codes, sf 16-byte
 * aligned.  rows == 0 enqueues nothing.
 * Errors: NVFP4_ERR_INVALID_ARG (null pointer, negative size, ld < cols, bad
 * layout, g inside codes or sf), NVFP4_ERR_ALIGNMENT (cols, ld or a pointer),
 * NVFP4_ERR_UNSUPPORTED_SHAPE (the size bounds), CUDA errors.
 * Source: evolve.pub review, Scope & Claims (the element and scale formats
 * and the 16-element grouping); thevalue.engineering, second section. */
nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                            const float* g, uint8_t* codes, uint8_t* sf,
                            nvfp4_sf_layout layout, void* stream);

/* As nvfp4_quantize, for rows [row_offset, row_offset + rows) of a larger
 * [total_rows, cols] quantized tensor -- one module of a fused weight, which
 * keeps its own global scale *g.  codes and sf point to the start of the WHOLE
 * tensor's buffers (total_rows * cols/2 code bytes; nvfp4_sf_bytes(total_rows,
 * cols, layout) scale bytes); only this slice's rows are written, plus, when
 * row_offset + rows == total_rows, the tensor-core layout's padding rows.
 * Calls for different slices of one tensor may run in any order.
 * Requirements and errors as nvfp4_quantize; 0 <= row_offset, row_offset +
 * rows <= total_rows (NVFP4_ERR_INVALID_ARG otherwise).
 * Source: per-module global scales of a fused GEMM (chatpaper.ai abstract;
 * evolve.pub Key claims, fourth bullet). */
nvfp4_status nvfp4_quantize_slice(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                  const float* g, uint8_t* codes, uint8_t* sf,
                                  nvfp4_sf_layout layout, int64_t row_offset,
                                  int64_t total_rows, void* stream);

/* W4A4 GEMM: y[m, n] = BF16_RNE(fl32(acc[m, n] * fl32(*a_g * *w_g))) with
 * acc[m, n] = sum_k E2M1(a[m,k]) E4M3(sa[m,k/16]) E2M1(w[n,k]) E4M3(sw[n,k/16])
 * accumulated in FP32 on the tensor cores (block-scaled FP4 MMA).
 *   a_codes [M, K/2], w_codes [N, K/2]  (device, packed as above, K-major)
 *   a_sf, w_sf  (device) block scales in NVFP4_SF_TCGEN05 layout
 *   a_g, w_g    (device) FP32 global scales
 *   y [M, N] BF16 (device), row stride ldy elements
 * Weights are [N, K] (the nn.Linear convention) and are quantized with
 * nvfp4_quantize like activations.  No bias.
 * Requirements: K % 32 == 0, K >= 32; ldy >= N, ldy % 8 == 0; all pointers
 * 16-byte aligned.  M == 0 or N == 0 enqueues nothing.
 * Few tokens (M <= 128): the kernel is launched as a programmatic dependent
 * of the previous kernel on the stream.  Its CTAs may start before that
 * kernel has finished, but they read no memory until it has completed, so
 * stream order holds for every operand and for y.  Its FP32 summation order
 * depends on K alone, so a row's result does not depend on N.
 * Errors: NVFP4_ERR_INVALID_ARG (null pointer, negative size, a scale inside
 * y), NVFP4_ERR_ALIGNMENT (ldy or a pointer), NVFP4_ERR_UNSUPPORTED_SHAPE (K,
 * the size bounds), NVFP4_ERR_DEVICE (not sm_100), CUDA errors.  A bounded
 * wait that gives up inside the kernel is reported later by
 * nvfp4_last_device_status as NVFP4_ERR_TIMEOUT.
 * Source: chatpaper.ai abstract (W4A4 on every linear layer); evolve.pub FAQ
 * (native NVFP4 execution). */
nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_g,
                        const uint8_t* w_codes, const uint8_t* w_sf, const float* w_g,
                        void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                        void* stream);

/* Fused multi-module W4A4 GEMM: as nvfp4_gemm, but output column n uses the
 * global scale of the segment containing n:  alpha_n = fl32(*a_g *
 * *segs[i].w_gscale) for n in [segs[i].n_offset, +n_size).  The fused
 * result equals, bit for bit, nvfp4_gemm run per module with that module's
 * scale (the kernel configuration depends on M and K only, and every output
 * element is accumulated in the same K order), which is the repair of the
 * global-scale mismatch.
 *   segs (host, nseg entries, copied during the call): in order, contiguous,
 *   starting at 0, n_size > 0; N = sum of n_size.  1 <= nseg <=
 *   NVFP4_MAX_SEGMENTS.  w_codes/w_sf hold the concatenated [N, K] weight,
 *   each module quantized with its own global scale.
 * Requirements as nvfp4_gemm.  Errors as nvfp4_gemm, and NVFP4_ERR_INVALID_ARG
 * for a segment table that is not contiguous from 0 or has more than
 * NVFP4_MAX_SEGMENTS entries.
 * Source: chatpaper.ai abstract (serving modules calibrated one by one
 * through a single fused GEMM is where the mismatch arises); evolve.pub Key
 * claims, fourth bullet. */
nvfp4_status nvfp4_fused_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_g,
                              const uint8_t* w_codes, const uint8_t* w_sf,
                              const nvfp4_segment* segs, int nseg,
                              void* y, int64_t ldy, int64_t M, int64_t K,
                              void* stream);

/* Fused multi-module GEMM with gate functions in the epilogue: as
 * nvfp4_fused_gemm, then each output of segment i is replaced by
 * f_i(fl32(acc * alpha_n)) evaluated in FP32 (expf, log1pf, IEEE division)
 * and rounded once to BF16, f_i given by acts[i] (nvfp4_act_kind; NONE is the
 * identity).  For the fused Gated DeltaNet input projection this yields the
 * log-space decay gate g (segment a) and the write strength beta (segment b)
 * directly, without a BF16 round trip of the raw gate projections.
 *   acts (host, nseg entries, copied during the call) or NULL (all NONE).
 *        A DECAY_GATE entry needs a_log and dt_bias (device, n_size FP32 each).
 * Errors: as nvfp4_fused_gemm; NVFP4_ERR_INVALID_ARG for an unknown kind or a
 * missing parameter array.
 * Source: evolve.pub, Key claims under review, second bullet, and Report
 * preview, Table 3 (the decay gate, kept in log space through a softplus and an
 * exponential, and the sigmoid write strength); the formulas are the Gated
 * DeltaNet reading -- the pages give none. */
nvfp4_status nvfp4_fused_gemm_act(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_g,
                                  const uint8_t* w_codes, const uint8_t* w_sf,
                                  const nvfp4_segment* segs, const nvfp4_segment_act* acts,
                                  int nseg, void* y, int64_t ldy, int64_t M, int64_t K,
                                  void* stream);

/* gate_up GEMM of a SiLU-gated MLP with the intermediate computed in its
 * epilogue:  h[m, j] = BF16_RNE(fl32(SiLU(gate) * up)), gate = fl32(acc[m,
 * gate row j] * alpha), up = fl32(acc[m, up row j] * alpha), alpha =
 * fl32(*a_g * *w_g), SiLU evaluated as in nvfp4_silu_mul -- so no BF16
 * [M, 2F] gate_up tensor is written or read -- plus the global scale of h
 * for its W4A4 requantization:  *h_g = fl32(max|h| / 2688) (1 if h is all
 * zero), what nvfp4_global_scale(h) returns, and *h_amax = max|h| (if
 * non-null).
 *   w_codes/w_sf: the [2F, K] gate_up weight (one global scale *w_g) with its
 *     rows INTERLEAVED in 128-row blocks: block 2b = gate rows [128b, 128b+128),
 *     block 2b+1 = the matching up rows.  Interleaving the BF16 rows before
 *     quantizing changes neither the rows' codes nor the global scale.
 *   h: device BF16 [M, F], row stride ldh elements.
 *   workspace: as nvfp4_global_scale (NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES,
 *     zero-initialised, left zeroed); h_g, h_amax: device FP32, outside
 *     the workspace (NVFP4_ERR_INVALID_ARG otherwise).
 * Requirements: M > 256 (the CTA-pair prefill kernel; smaller batches use
 * nvfp4_gemm + nvfp4_silu_mul), F a multiple of 128, K as nvfp4_gemm,
 * ldh >= F and a multiple of 8, pointers 16-byte aligned.
 * Errors: NVFP4_ERR_INVALID_ARG, NVFP4_ERR_UNSUPPORTED_SHAPE,
 * NVFP4_ERR_ALIGNMENT, CUDA errors.  Asynchronous on `stream`.
 * Source: W4A4 on every linear layer, the MLP's included (chatpaper.ai
 * abstract); the SiLU-gated MLP is the plain reading of the model's MLP. */
nvfp4_status nvfp4_gemm_silu_mul(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_g,
                                 const uint8_t* w_codes, const uint8_t* w_sf, const float* w_g,
                                 void* h, int64_t ldh, int64_t M, int64_t F, int64_t K,
                                 void* workspace, float* h_g, float* h_amax, void* stream);

/* Checkpoint-side repair of the global-scale mismatch: rewrite the block
 * scales of a fused weight so that ONE global scale serves all its modules.
 *   g_c  = max_i *segs[i].w_gscale                 (written to *g_common)
 *   r_i  = fl32(g_i / g_c)
 *   s8' = E4M3_RNE_satfinite(fl32(E4M3(s8) * r_i)) for every scale byte of
 *          module i's rows; the codes are not touched.
 * Afterwards nvfp4_gemm(..., w_sf, g_common, ...) serves the fused weight
 * with a single scale; E4M3(s8') * g_c equals E4M3(s8) * g_i where that
 * product is an E4M3 value and rounds it otherwise (modules with small
 * scales lose precision in the E4M3 subnormals).  This is the alternative to
 * the per-segment epilogue of nvfp4_fused_gemm.
 *   w_sf     (device, in/out) scale bytes of the fused [N, K] weight in
 *            `layout`, N = sum of n_size (padding bytes of the tensor-core
 *            layout stay 0).  16-byte aligned.
 *   K        multiple of 16 (so cols/16 scales per row).
 *   segs     (host, nseg entries, copied during the call): as for
 *            nvfp4_fused_gemm; the w_gscale pointers are device FP32.
 *   g_common (device) receives g_c; it must not be one of the segments'
 *            scales (it is written while the kernel still reads them).
 * Errors: NVFP4_ERR_INVALID_ARG (null pointer, bad segment table, bad
 * layout, g_common equal to a segment's scale pointer), NVFP4_ERR_UNSUPPORTED_SHAPE (K, or a segment or N at 2^31 or
 * more), NVFP4_ERR_ALIGNMENT, CUDA errors.
 * Asynchronous on `stream`.
 * Source: chatpaper.ai abstract (per-module-calibrated checkpoints, fused
 * multi-module kernels, the global-scale mismatch and its repair); the choice
 * of the largest module scale as the common one is a reading -- the pages
 * give no formula. */
nvfp4_status nvfp4_harmonize_scales(uint8_t* w_sf, int64_t K, const nvfp4_segment* segs, int nseg,
                                    nvfp4_sf_layout layout, float* g_common, void* stream);

/* FP8 E4M3 KV cache with a calibrated per-tensor scale.
 *
 * nvfp4_kv_scale_from_amax: *scale = fl32(*amax / 448), or 1 when *amax is 0
 * (both device FP32; amax as written by nvfp4_global_scale's amax_out over the
 * calibration tensor).  Errors: NVFP4_ERR_INVALID_ARG (null), CUDA errors.
 *
 * nvfp4_kv_quantize_e4m3: out[r, c] = signed E4M3 byte of fl32(x[r, c] /
 * *scale), round to nearest even, saturating at +-448 (the NaN code is never
 * written), bit 7 the sign of the quotient (kept for zero).  Every byte
 * equals the one an IEEE division would give.
 *   x      (device) BF16 [rows, cols], row stride ld elements; 16-byte aligned.
 *   scale  (device) FP32 per-tensor scale, positive and finite.
 *   out    (device) bytes [rows, cols], row stride ldo bytes; 8-byte aligned.
 * Requirements: cols, ld, ldo multiples of 8; ld >= cols, ldo >= cols.
 * Errors: NVFP4_ERR_INVALID_ARG, NVFP4_ERR_ALIGNMENT, NVFP4_ERR_UNSUPPORTED_SHAPE
 * (the size bounds of the conventions above), CUDA errors.  Both calls
 * are asynchronous on `stream`.
 * Source: evolve.pub, Key claims under review (calibrated per-tensor FP8
 * KV-cache scales); the formula is a reading -- the pages give none. */
nvfp4_status nvfp4_kv_scale_from_amax(const float* amax, float* scale, void* stream);
nvfp4_status nvfp4_kv_quantize_e4m3(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                    const float* scale, uint8_t* out, int64_t ldo, void* stream);

/* The whole W4A4 linear layer from host buffers, on one stream: the BF16
 * activation x_host [M, K] is copied into x_dev, its global scale (a_g,
 * a_amax) and NVFP4 codes (a_codes, a_sf in the tensor-core layout)
 * computed, the fused GEMM run against the pre-quantized weight (w_codes,
 * w_sf, segs exactly as nvfp4_fused_gemm), and y_dev [M, N] (row stride N)
 * copied back to y_host -- nvfp4_global_scale, nvfp4_quantize and
 * nvfp4_fused_gemm between two cudaMemcpyAsync calls.
 *   x_host (host) BF16 [M, K], contiguous; y_host (host) BF16 [M, N],
 *            contiguous.  Page-locked memory makes the copies asynchronous:
 *            keep both buffers alive, x_host unchanged and y_host unread
 *            until the stream has passed the copies (synchronize it).
 *            Pageable memory works, but the copies then block the caller.
 *   x_dev (device, M * K * 2 bytes), a_codes (device, M * K/2 bytes), a_sf
 *            (device, nvfp4_sf_bytes(M, K, NVFP4_SF_TCGEN05) bytes), a_g,
 *            a_amax (device FP32; a_amax may be NULL), workspace (device, as
 *            nvfp4_global_scale), y_dev (device, M * N * 2 bytes): scratch
 *            the caller owns; the call allocates nothing.
 * Every check of the three composed calls is made before anything is
 * enqueued, so a refused call enqueues nothing.  Requirements: K % 32 == 0,
 * N % 8 == 0, device pointers 16-byte aligned, no scalar inside an output
 * and x_dev apart from y_dev, a_codes and a_sf.
 * Errors: NVFP4_ERR_INVALID_ARG, NVFP4_ERR_ALIGNMENT,
 * NVFP4_ERR_UNSUPPORTED_SHAPE, NVFP4_ERR_DEVICE, as the composed calls;
 * NVFP4_ERR_CUDA when a copy or a launch fails.  M == 0 enqueues nothing.
 * Source: the pages' serving path, W4A4 on every linear layer with
 * per-module global scales in the fused GEMM (chatpaper.ai abstract;
 * evolve.pub review, Scope & Claims). */
nvfp4_status nvfp4_fused_linear_host(const void* x_host, int64_t M, int64_t K,
                                     const uint8_t* w_codes, const uint8_t* w_sf,
                                     const nvfp4_segment* segs, int nseg, void* y_host,
                                     void* x_dev, uint8_t* a_codes, uint8_t* a_sf, float* a_g,
                                     float* a_amax, void* workspace, void* y_dev, void* stream);

/* nvfp4_fused_linear_host with its copy out on a second stream, so that the
 * PCIe transfers overlap the kernels and each other.  On `stream`: the copy in,
 * the global scale and the quantization; then the GEMM in row slices (about
 * 2048 rows each, a multiple of 256; with M <= 3072 one slice), each slice's
 * copy of y_dev to y_host issued on `copy_stream` as soon as that slice's
 * GEMM is done, while the next slice computes.  Before the first slice
 * rewrites y_dev, `stream` waits for everything already enqueued on
 * copy_stream (the previous call's copy out of y_dev), so consecutive calls
 * may reuse one set of device buffers: call i + 1's copy in and quantization
 * run while call i's output is still being copied out (the link is full
 * duplex).  Every slice runs the GEMM kernel that the whole M selects, so y
 * equals nvfp4_fused_linear_host's output bit for bit.
 *   Buffers, requirements and errors as nvfp4_fused_linear_host.  x_host must
 *   stay unchanged until `stream` has passed the copy in; y_host holds the
 *   output once `copy_stream` has passed this call's copies (synchronize it,
 *   or record an event on it); a caller that rewrites or reads y_host between
 *   calls orders that against copy_stream.  copy_stream may equal stream (the
 *   call then runs in series).  The call creates one CUDA event and releases
 *   it before returning; it allocates no device memory.
 * Source: as nvfp4_fused_linear_host. */
nvfp4_status nvfp4_fused_linear_host_overlap(const void* x_host, int64_t M, int64_t K,
                                             const uint8_t* w_codes, const uint8_t* w_sf,
                                             const nvfp4_segment* segs, int nseg, void* y_host,
                                             void* x_dev, uint8_t* a_codes, uint8_t* a_sf,
                                             float* a_g, float* a_amax, void* workspace,
                                             void* y_dev, void* stream, void* copy_stream);

/* MLP intermediate for the W4A4 down projection: h[r, c] = BF16_RNE(
 * fl32(SiLU(gate) * up)) with gate = gate_up[r, c], up = gate_up[r, f + c]
 * (BF16, row stride ld elements, device) and SiLU(v) = v / (1 + e^-v)
 * evaluated in FP32 (expf, IEEE division); h is BF16 [rows, f], row stride
 * ldh (device).  Within one BF16 ulp of the value rounded once from exact
 * arithmetic.  Requirements: f, ld, ldh multiples of 8; ld >= 2f, ldh >= f;
 * pointers 16-byte aligned.  rows == 0 or f == 0 enqueues nothing.
 * Errors: NVFP4_ERR_INVALID_ARG (null pointer, negative size, ld < 2f,
 * ldh < f), NVFP4_ERR_ALIGNMENT (f, ld, ldh or a pointer),
 * NVFP4_ERR_UNSUPPORTED_SHAPE (the size bounds), CUDA errors.
 * Source: W4A4 on every linear layer, the MLP down projection included
 * (chatpaper.ai abstract); the SiLU-gated MLP is the plain reading of the
 * 27B hybrid's MLP block, which the pages do not describe. */
nvfp4_status nvfp4_silu_mul(const void* gate_up, int64_t rows, int64_t f, int64_t ld, void* h,
                            int64_t ldh, void* stream);

/* Synchronizes `stream`, then reads and clears the library's device status
 * word on the current device: NVFP4_ERR_TIMEOUT if a bounded wait inside a
 * kernel gave up since the last call (that kernel's output is then invalid),
 * NVFP4_ERR_CUDA if the stream reports an error, else NVFP4_OK. */
nvfp4_status nvfp4_last_device_status(void* stream);

/* Diagnostic: launches one CTA whose thread waits on a barrier nothing ever
 * arrives on, bounded by limit_ns (1 .. 10^9).  The wait gives up, sets the
 * device status word and returns, so the next nvfp4_last_device_status()
 * reports NVFP4_ERR_TIMEOUT while the context stays usable.  Exercises the
 * timeout path every kernel's waits share, without faulting the GPU. */
nvfp4_status nvfp4_debug_wait_timeout(int64_t limit_ns, void* stream);

/* Static English description of a status code. */
const char* nvfp4_status_string(nvfp4_status s);

/* ABI version (major * 10000 + minor * 100 + patch). */
int nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
