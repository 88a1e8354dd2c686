// gemm.cu -- block-scaled FP4 x FP4 GEMM with FP32 accumulation in tensor
// memory and a BF16 epilogue that applies the global scales per N-segment.
//
// Y[m, n] = bf16( fl32( acc[m, n] * fl32(gA * gW[seg(n)]) ) ),
// acc[m, n] = sum_k e2m1(a[m,k]) e4m3(sa[m,k/16]) e2m1(w[n,k]) e4m3(sw[n,k/16]).
//
// Sources (pages on "Why Gated DeltaNet Survives 4-Bit Quantization"):
// W4A4 on every linear layer and the fused-module global-scale repair
// (chatpaper.ai abstract); native NVFP4 execution (evolve.pub FAQ).
//
// Three kernels, chosen by M alone (so a fused GEMM and its per-module GEMMs
// accumulate every output identically):
//   M <= 128         nvf4_gemm_decode_kernel (gemm_decode.cuh): operands
//                    swapped, K split over a cluster, persistent.
//   128 < M <= 256   nvf4_gemm_kernel<128, 6, 2>: one CTA per 128 x 128 tile,
//                    described below.
//   M > 256          nvf4_gemm_pair_kernel<5, 128, kSilu>: a CTA pair per 256 x 256
//                    tile (cta_group::2), described above its definition.
// Epilogue variants: the gate functions of the Gated DeltaNet projection on
// chosen segments (any kernel, `apply_gates`), and SiLU(gate) * up with the
// global scale of h for the MLP's gate_up GEMM (pair kernel, kSilu = true).
//
// Design of the one-CTA kernel (sm_100a, one CTA per SM, persistent):
//   warp 0      TMA producer: A/B code tiles by tiled TMA (128-byte swizzle),
//               their scale atoms by 1-D bulk copies (the scales are stored
//               in the tensor-core layout, so one k-step of a 128-row block
//               is 2 KB of contiguous bytes).
//   warp 1      TMEM allocator and MMA issuer (one thread): per k-step it
//               copies the scale atoms shared->TMEM and issues
//               tcgen05.mma.kind::mxf4nvf4.block_scale (M=128, N=BN, K=64).
//   warps 2..9  epilogue: two warps per TMEM lane quarter, each draining half
//               of the tile's columns into registers; the accumulator is
//               released as soon as all of it sits in registers, so the next
//               tile's MMAs overlap the alpha scaling and the BF16 stores.
// Every wait is bounded; a timeout sets the device status word and all roles
// leave their loops, drain in-flight copies and free TMEM.
#include <algorithm>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_common.h"
#include "nvfp4.h"
#include "ptx.cuh"
#include "silu.cuh"

namespace nvfp4 {

__device__ int g_device_status;

namespace {

constexpr int kBM = 128;             // MMA M (rows of A per tile)
constexpr int kBKBytes = 128;        // one k-step: 256 FP4 values = 128 bytes per row
constexpr int kAtom = 512;           // one scale atom: 128 rows x 4 scales
constexpr int kAtomsPerStep = 4;     // 256 values = 16 scales = 4 atoms per row block
constexpr int kEpiWarps = 8;         // two per TMEM lane quarter, each half the columns
constexpr int kThreads = 64 + 32 * kEpiWarps;  // producer, MMA, epilogue warps
constexpr int kPairThreads = kThreads;           // producer, MMA, epilogue warps
constexpr uint64_t kTimeoutNs = 1000000000ull;  // 1 s per wait
#ifndef NVFP4_PAIR_KB
#define NVFP4_PAIR_KB 128
#endif
#ifndef NVFP4_PAIR_STAGES
#define NVFP4_PAIR_STAGES 5
#endif
// CTA-pair kernel pipeline: bytes of every row per stage and stage count
constexpr int kPairKB = NVFP4_PAIR_KB;
constexpr int kPairStages = NVFP4_PAIR_STAGES;

struct GemmArgs {
    const uint8_t* a_sf;
    const uint8_t* w_sf;
    const float* a_g;
    uint16_t* y;
    int64_t ldy;
    int M, N, K;
    int m_tiles, n_tiles, k_steps;
    int atoms_per_rb;     // ceil(K/64): scale atoms per 128-row block
    int w_rowblocks;      // ceil(N/128)
    int group_m;          // raster: tiles visit group_m m-tiles per n sweep
    int nt_first;         // raster: the n sweep starts at this n-tile (the gated columns')
    int nseg;
    int seg_end[NVFP4_MAX_SEGMENTS];
    const float* seg_g[NVFP4_MAX_SEGMENTS];
    int any_act;                                   // some segment has a gate function
    int gate_lo, gate_hi;                          // hull of the gated segments' columns
    unsigned int* h_ws;                            // SiLU epilogue: {amax bits, ticket}, zeroed
    float* h_g;                                    // SiLU epilogue: fl32(amax(h) / 2688)
    float* h_amax;                                 // SiLU epilogue: amax(h) (may be null)
    int seg_kind[NVFP4_MAX_SEGMENTS];              // nvfp4_act_kind per segment
    int seg_goff[NVFP4_MAX_SEGMENTS];              // decay gate: offset in the staged parameters
    const float* seg_p0[NVFP4_MAX_SEGMENTS];       // decay gate: A_log per column
    const float* seg_p1[NVFP4_MAX_SEGMENTS];       // decay gate: dt_bias per column
    uint64_t timeout_ns;
    int* status;
};

// Decay-gate parameters staged in shared memory: at most this many columns
// over all decay-gate segments (the GDN projection has one per head).
constexpr int kMaxGateCols = 256;

// Per-segment epilogue data, copied to shared memory at kernel start.
struct SegTable {
    float alpha[NVFP4_MAX_SEGMENTS];          // fl32(gA * gW[s])
    int end[NVFP4_MAX_SEGMENTS];              // one past the segment's last column
    int kind[NVFP4_MAX_SEGMENTS];             // nvfp4_act_kind
    int goff[NVFP4_MAX_SEGMENTS];             // decay gate: first index in gp0/gp1
    float gp0[kMaxGateCols];                  // decay gate: -exp(A_log) per column
    float gp1[kMaxGateCols];                  // decay gate: dt_bias per column
};

template <int BN>
__host__ __device__ constexpr uint32_t make_idesc() {
    // kind::mxf4nvf4 block-scaled descriptor: A and B E2M1 (format 1), both
    // K-major, UE4M3 scales (bit 23 = 0), dense, N >> 3 at bit 17, M >> 4 at
    // bit 24, scale-factor ids 0.
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
           (static_cast<uint32_t>(kBM >> 4) << 24);
}

template <int BN, int STAGES, int ACC>
struct Cfg {
    static constexpr int A_BYTES = kBM * kBKBytes;
    static constexpr int B_BYTES = BN * kBKBytes;
    static constexpr int SFA_BYTES = kAtomsPerStep * kAtom;
    static constexpr int SFB_BYTES = (BN / 128) * kAtomsPerStep * kAtom;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
    static constexpr int NBAR = 2 * STAGES + 2 * ACC + 1;
    static constexpr int OFF_SEG = OFF_BAR + NBAR * 8;
    static constexpr int OFF_MISC = OFF_SEG + static_cast<int>((sizeof(SegTable) + 15) / 16 * 16);
    static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
    static constexpr int SFA_COL = ACC * BN;
    static constexpr int SFB_COL = SFA_COL + kAtomsPerStep * 4;
    static constexpr int COLS_USED = SFB_COL + kAtomsPerStep * (BN / 32);
    static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64
                                   : COLS_USED <= 128 ? 128 : COLS_USED <= 256 ? 256 : 512;
    static_assert(COLS_USED <= 512, "tensor memory overflow");
    static_assert(SMEM <= 232448, "shared memory overflow");
    // a CTA that takes more than half the TMEM must also take more than half
    // the shared memory, so that no second CTA on its SM waits in the allocator
    static_assert(TMEM_COLS <= 256 || SMEM > 228 * 1024 / 2, "two CTAs per SM would share TMEM");
    static_assert(BN % 128 == 0 && BN <= 256, "BN must be 128 or 256");
};

__device__ __forceinline__ void tile_coords(int t, const GemmArgs& a, int& mt, int& nt) {
    const int group_m = min(a.group_m, a.m_tiles);
    const int per_group = group_m * a.n_tiles;
    const int grp = t / per_group;
    const int first_m = grp * group_m;
    const int gsize = min(group_m, a.m_tiles - first_m);
    const int local = t - grp * per_group;
    mt = first_m + local % gsize;
    nt = local / gsize + a.nt_first;           // rotated sweep: gated tiles early, not in the tail
    if (nt >= a.n_tiles) nt -= a.n_tiles;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

// Fill the table: thread t < NVFP4_MAX_SEGMENTS writes entry t.
__device__ __forceinline__ void fill_seg_table(SegTable& T, const GemmArgs& a, int t) {
    const bool in = t < a.nseg;
    T.alpha[t] = in ? __fmul_rn(*a.a_g, *a.seg_g[t]) : 0.0f;
    T.end[t] = in ? a.seg_end[t] : 0x7FFFFFFF;
    T.kind[t] = in ? a.seg_kind[t] : NVFP4_ACT_NONE;
    T.goff[t] = in ? a.seg_goff[t] : 0;
}

// Stage the decay-gate parameters (all threads of the CTA; before a barrier):
// per column -exp(A_log) (the same binary32 value the gate would compute per
// element) and dt_bias.
__device__ __forceinline__ void stage_gate_params(SegTable& T, const GemmArgs& a, int tid, int nthreads) {
    if (!a.any_act) return;
    for (int s = 0; s < a.nseg; ++s) {
        if (a.seg_kind[s] != NVFP4_ACT_DECAY_GATE) continue;
        const int start = s == 0 ? 0 : a.seg_end[s - 1];
        const int n = a.seg_end[s] - start;
        for (int c = tid; c < n; c += nthreads) {
            T.gp0[a.seg_goff[s] + c] = -expf(a.seg_p0[s][c]);
            T.gp1[a.seg_goff[s] + c] = a.seg_p1[s][c];
        }
    }
}

// Gated DeltaNet gate functions in FP32: the log-space decay gate
// -exp(A_log) * softplus(v + dt_bias) with -exp(A_log) staged per column, and
// the sigmoid.  Both are written so that every intermediate stays in (0, 1]
// and no special value reaches a library routine, whatever the size of v:
//   softplus(z) = max(z, 0) + log1p(t), t = e^-|z|, with log1p(t) taken as t
//   once t < 2^-24 (|z| > 17: the two agree to a relative 2^-25);
//   sigmoid(v) = 1 / (1 + t) for v >= 0 and t / (1 + t) below, t = e^-|v|.
__device__ __forceinline__ float gate_fn(float v, int kind, float neg_exp_alog, float dt_bias) {
    if (kind == NVFP4_ACT_DECAY_GATE) {
        const float z = __fadd_rn(v, dt_bias);
        const float a = fabsf(z);
        const float t = expf(-a);
        const float l = a > 17.0f ? t : log1pf(t);
        return __fmul_rn(neg_exp_alog, __fadd_rn(fmaxf(z, 0.0f), l));
    }
    if (kind == NVFP4_ACT_SIGMOID) {
        const float t = expf(-fabsf(v));
        const float s = __frcp_rn(__fadd_rn(1.0f, t));
        return v >= 0.0f ? s : __fmul_rn(t, s);
    }
    return v;
}

// Apply the segments' gate functions to CNT consecutive scaled outputs
// starting at column n0 (columns at or beyond N are left alone).  Out of line:
// the math functions inlined once per element would bloat every epilogue
// that contains this call (only chunks that meet the gated columns reach it,
// and their values take a trip through local memory).  A chunk inside one
// segment, the usual case, is evaluated eight elements at a time so that the
// exp / log1p chains of different elements overlap.
template <int KIND>
__device__ __forceinline__ void gate_run(float* v, int n0, int N, int cnt, int g0, const SegTable& T) {
#pragma unroll 1
    for (int j0 = 0; j0 < cnt; j0 += 8) {
        float x[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) x[jj] = v[j0 + jj];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            if (n0 + j0 + jj < N) {
                const int g = g0 + j0 + jj;
                x[jj] = KIND == NVFP4_ACT_DECAY_GATE ? gate_fn(x[jj], KIND, T.gp0[g], T.gp1[g])
                                                     : gate_fn(x[jj], KIND, 0.0f, 0.0f);
            }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) v[j0 + jj] = x[jj];
    }
}

template <int CNT>
__device__ __noinline__ void apply_gates(float* v, int n0, int N, int nseg, const SegTable& T) {
    static_assert(CNT % 8 == 0 || CNT < 8, "chunks of eight");
    int s = 0;
    while (s < nseg - 1 && n0 >= T.end[s]) ++s;
    if (CNT % 8 == 0 && (s == nseg - 1 || n0 + CNT <= T.end[s])) {
        const int kind = T.kind[s];
        const int g0 = T.goff[s] + n0 - (s == 0 ? 0 : T.end[s - 1]);
        if (kind == NVFP4_ACT_DECAY_GATE) gate_run<NVFP4_ACT_DECAY_GATE>(v, n0, N, CNT, g0, T);
        else if (kind == NVFP4_ACT_SIGMOID) gate_run<NVFP4_ACT_SIGMOID>(v, n0, N, CNT, 0, T);
        return;
    }
    // a chunk that meets two or more segments: one element at a time
#pragma unroll 1
    for (int j = 0; j < CNT; ++j) {
        const int n = n0 + j;
        while (s < nseg - 1 && n >= T.end[s]) ++s;
        const int kind = T.kind[s];
        if (n < N && kind != NVFP4_ACT_NONE) {
            const int g = T.goff[s] + n - (s == 0 ? 0 : T.end[s - 1]);
            const bool decay = kind == NVFP4_ACT_DECAY_GATE;
            v[j] = gate_fn(v[j], kind, decay ? T.gp0[g] : 0.0f, decay ? T.gp1[g] : 0.0f);
        }
    }
}

// The gated chunk's values go through a local copy, so the caller's array
// never has its address taken and stays in registers on every other chunk.
template <int CNT>
__device__ __forceinline__ void apply_gates_copy(float (&v)[CNT], int n0, int N, int nseg,
                                                 const SegTable& T) {
    float tmp[CNT];
#pragma unroll
    for (int j = 0; j < CNT; ++j) tmp[j] = v[j];
    apply_gates<CNT>(tmp, n0, N, nseg, T);
#pragma unroll
    for (int j = 0; j < CNT; ++j) v[j] = tmp[j];
}

template <int BN, int STAGES, int ACC>
__global__ void __launch_bounds__(kThreads, 1)
nvf4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                 const __grid_constant__ CUtensorMap tmap_b, const GemmArgs args) {
    using C = Cfg<BN, STAGES, ACC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tmem_full = bars + 2 * STAGES;
    uint64_t* tmem_empty = bars + 2 * STAGES + ACC;
    uint64_t* drain = bars + 2 * STAGES + 2 * ACC;
    SegTable& seg_tab = *reinterpret_cast<SegTable*>(smem + C::OFF_SEG);
    const float* s_seg_alpha = seg_tab.alpha;
    const int* s_seg_end = seg_tab.end;
    uint32_t* s_tmem_base = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int total_tiles = args.m_tiles * args.n_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < ACC; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], kEpiWarps);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + NVFP4_MAX_SEGMENTS)
        fill_seg_table(seg_tab, args, threadIdx.x - 64);
    stage_gate_params(seg_tab, args, threadIdx.x, blockDim.x);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            const uint64_t pol = l2_policy_evict_last();   // operands are re-read by many tiles
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_parity = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                int mt, nt;
                tile_coords(t, args, mt, nt);
                for (int kb = 0; kb < args.k_steps; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, args.timeout_ns, s_abort,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    const int natoms = min(kAtomsPerStep, args.atoms_per_rb - kb * kAtomsPerStep);
                    int w_rbs = 0;
                    for (int r = 0; r < BN / 128; ++r)
                        if (nt * (BN / 128) + r < args.w_rowblocks) ++w_rbs;
                    const uint32_t bytes = C::A_BYTES + C::B_BYTES + natoms * kAtom * (1 + w_rbs);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(smem + C::OFF_A + stage * C::A_BYTES, &tmap_a, &full[stage],
                                kb * kBKBytes, mt * kBM, pol);
                    tma_load_2d(smem + C::OFF_B + stage * C::B_BYTES, &tmap_b, &full[stage],
                                kb * kBKBytes, nt * BN, pol);
                    const size_t a_off =
                        (static_cast<size_t>(mt) * args.atoms_per_rb + kb * kAtomsPerStep) * kAtom;
                    bulk_load(smem + C::OFF_SFA + stage * C::SFA_BYTES, args.a_sf + a_off,
                              natoms * kAtom, &full[stage], pol);
                    for (int r = 0; r < w_rbs; ++r) {
                        const size_t w_off = (static_cast<size_t>(nt * (BN / 128) + r) *
                                                  args.atoms_per_rb + kb * kAtomsPerStep) * kAtom;
                        bulk_load(smem + C::OFF_SFB + stage * C::SFB_BYTES + r * kAtomsPerStep * kAtom,
                                  args.w_sf + w_off, natoms * kAtom, &full[stage], pol);
                    }
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // leave no copy in flight: wait (bounded) for every stage issued
                int local_abort = 0;
                for (int s = 0; s < STAGES; ++s)
                    if (issued & (1u << s))
                        mbar_wait_bounded(&full[s], (issued_parity >> s) & 1u, args.timeout_ns,
                                          &local_abort, args.status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t idesc = make_idesc<BN>();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int i = 0;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++i) {
                const int acc = i % ACC;
                const uint32_t acc_phase = (i / ACC) & 1;
                if (!mbar_wait_bounded(&tmem_empty[acc], acc_phase ^ 1u, args.timeout_ns, s_abort,
                                       args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < args.k_steps; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, args.timeout_ns, s_abort,
                                           args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int natoms = min(kAtomsPerStep, args.atoms_per_rb - kb * kAtomsPerStep);
                    const uint32_t sa = smem_u32(smem + C::OFF_A + stage * C::A_BYTES);
                    const uint32_t sb = smem_u32(smem + C::OFF_B + stage * C::B_BYTES);
                    const uint32_t ssfa = smem_u32(smem + C::OFF_SFA + stage * C::SFA_BYTES);
                    const uint32_t ssfb = smem_u32(smem + C::OFF_SFB + stage * C::SFB_BYTES);
                    for (int j = 0; j < natoms; ++j) {
                        tc_copy_scales(tmem_base + C::SFA_COL + j * 4, sdesc_scales(ssfa + j * kAtom));
#pragma unroll
                        for (int r = 0; r < BN / 128; ++r)
                            tc_copy_scales(tmem_base + C::SFB_COL + j * (BN / 32) + r * 4,
                                           sdesc_scales(ssfb + r * kAtomsPerStep * kAtom + j * kAtom));
                    }
                    for (int j = 0; j < natoms; ++j) {
                        tc_mma_nvf4(d_tmem, sdesc_kmajor_sw128(sa + j * 32),
                                    sdesc_kmajor_sw128(sb + j * 32), idesc,
                                    tmem_base + C::SFA_COL + j * 4,
                                    tmem_base + C::SFB_COL + j * (BN / 32), (kb | j) != 0);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) tc_commit(&tmem_full[acc]);
            }
            // every tcgen05 operation issued above has finished before TMEM is freed
            tc_commit(drain);
            int local_abort = 0;
            mbar_wait_bounded(drain, 0, args.timeout_ns, &local_abort, args.status);
        }
    } else {
        // ---------------- epilogue (warps 2..9) ----------------
        // Lane 0 of each warp waits for the accumulator and the result is
        // broadcast, so the warp stays converged for tcgen05.ld and leaves
        // together on an abort.  alpha per column comes from the segment table;
        // a 32-column chunk almost always lies inside one segment.
        constexpr int kHalf = BN / 2;            // columns per epilogue warp
        constexpr int kChunks = kHalf / 32;
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int half = (warp - 2) >> 2;        // which half of the columns
        const int row = q * 32 + lane;
        const uint64_t pol_y = l2_policy_evict_first();
        int i = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++i) {
            int mt, nt;
            tile_coords(t, args, mt, nt);
            const int acc = i % ACC;
            const uint32_t acc_phase = (i / ACC) & 1;
            int ok = 1;
            if (lane == 0)
                ok = mbar_wait_bounded(&tmem_full[acc], acc_phase, args.timeout_ns, s_abort,
                                       args.status);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            uint32_t r[kChunks][32];
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + half * kHalf;
#pragma unroll
            for (int ch = 0; ch < kChunks; ++ch) tmem_ld_32cols(taddr + ch * 32, r[ch]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[acc]);   // accumulator free for the next tile
            const int m = mt * kBM + row;
            uint16_t* yrow = args.y + static_cast<int64_t>(m) * args.ldy;
#pragma unroll
            for (int ch = 0; ch < kChunks; ++ch) {
                const int n0 = nt * BN + half * kHalf + ch * 32;
                int s0 = 0;
                while (s0 < args.nseg - 1 && n0 >= s_seg_end[s0]) ++s0;
                const bool one_seg = (s0 == args.nseg - 1) || (n0 + 31 < s_seg_end[s0]);
                if (m < args.M && n0 < args.N) {
                    float v[32];
                    if (one_seg) {
                        const float al = s_seg_alpha[s0];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(__uint_as_float(r[ch][j]), al);
                    } else {
                        int s = s0;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            while (s < args.nseg - 1 && n0 + j >= s_seg_end[s]) ++s;
                            v[j] = __fmul_rn(__uint_as_float(r[ch][j]), s_seg_alpha[s]);
                        }
                    }
                    if (args.any_act && n0 < args.gate_hi && n0 + 32 > args.gate_lo)
                        apply_gates_copy<32>(v, n0, args.N, args.nseg, seg_tab);
                    uint32_t o[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) o[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                    if (n0 + 32 <= args.N) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            st_global_v4_hint(yrow + n0 + 8 * u, o[4 * u], o[4 * u + 1], o[4 * u + 2],
                                              o[4 * u + 3], pol_y);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (n0 + j < args.N)
                                yrow[n0 + j] = static_cast<uint16_t>((o[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

#include "gemm_decode.cuh"

}  // namespace


// ---------------------------------------------------------------------------
// CTA-pair kernel (cta_group::2): a cluster of two CTAs on two SMs computes a
// 256 x 256 output tile.  Each CTA loads its own 128 rows of A, its 128-row
// half of the tile's B rows, its own A scale atoms and the B scale atoms of
// the whole 256-row N tile; every load is a 2-D TMA whose bytes are counted on
// the even CTA's full barrier.  A stage holds KB bytes of every row (2 KB
// values of K): KB = 64 gives ten 19 KB stages (64-byte swizzle), KB = 128
// five 38 KB stages (128-byte swizzle).  The MMA warp of the even CTA copies a
// stage's scale atoms into that stage's own TMEM region of both CTAs
// (tcgen05.cp, each CTA's shared memory into its own TMEM) and issues
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64) right behind them from
// the same thread, so the copies and the MMAs that read them execute in issue
// order without any handshake.  Feeding the tensor cores is a latency
// problem: a stage is refilled only after its MMAs complete, so the time from
// that commit through the TMA reload to the next MMA on it must fit in the
// MMA time of the other stages; every hop removed from that loop and every
// finer stage raises the sustained rate.  Accumulator rows 0..127 live in the
// even CTA's TMEM and 128..255 in the odd CTA's.  Commits are multicast to
// both CTAs' barriers; both CTAs' epilogue warps release the accumulator on
// the even CTA's barrier.  Per CTA and 256 values of K this moves 38 KB from
// L2 for 128 x 256 x 256 multiply-adds (the single-CTA 128 x 256 tile moves
// 54 KB).
// ---------------------------------------------------------------------------
template <int STAGES, int KB>
struct PairCfg {
    static constexpr int BN = 256;
    static constexpr int ATOMS = KB / 32;                          // scale atoms per 128-row block
    static constexpr int A_BYTES = kBM * KB;                       // own 128 rows of A
    static constexpr int B_BYTES = 128 * KB;                       // own half of the N tile
    static constexpr int SFA_BYTES = ATOMS * kAtom;                // own 128-row block
    static constexpr int SFB_BYTES = 2 * ATOMS * kAtom;            // both 128-row blocks of N
    static constexpr int STAGE_TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_EPI = OFF_SFB + STAGES * SFB_BYTES;  // epilogue staging, one per warp
    static constexpr int EPI_BYTES = 32 * 64;                    // 32 rows x 32 BF16 columns
    static constexpr int OFF_BAR = OFF_EPI + kEpiWarps * EPI_BYTES;
    static constexpr int NBAR = 2 * STAGES + 3;                  // full, empty, tmem_full, tmem_empty, drain
    static constexpr int OFF_SEG = OFF_BAR + NBAR * 8;
    static constexpr int OFF_MISC = OFF_SEG + static_cast<int>((sizeof(SegTable) + 15) / 16 * 16);
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int SF_STRIDE = ATOMS * 12;                 // TMEM columns per stage region
    static constexpr int SFB_COL = ATOMS * 4;                    // B scales after the A scales
    static constexpr int TMEM_COLS = 512;
    static_assert(KB == 64 || KB == 128, "stage row bytes: 64 or 128");
    static_assert(BN + STAGES * SF_STRIDE <= TMEM_COLS, "tensor memory overflow");
    static_assert(SMEM <= 232448, "shared memory overflow");
    static_assert(SMEM > 228 * 1024 / 2, "two CTAs per SM would share TMEM");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzled tiles stay 1024-byte aligned");
};

// kind::mxf4nvf4 descriptor for the pair MMA: M = 256, N = 256.
__host__ __device__ constexpr uint32_t make_idesc_pair() {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(256 >> 3) << 17) |
           (static_cast<uint32_t>(256 >> 4) << 24);
}

// K-major operand descriptor for rows of KB bytes in the matching swizzle.
template <int KB>
__device__ __forceinline__ uint64_t sdesc_kmajor(uint32_t saddr) {
    if constexpr (KB == 128) return sdesc_kmajor_sw128(saddr);
    else return sdesc_kmajor_sw64(saddr);
}

template <int STAGES, int KB, bool kSilu>
__global__ void __launch_bounds__(kPairThreads, 1)
nvf4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                      const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_sfa,
                      const __grid_constant__ CUtensorMap tmap_sfb,
                      const __grid_constant__ CUtensorMap tmap_y, const GemmArgs args) {
    using C = PairCfg<STAGES, KB>;
    constexpr int BN = C::BN;
    constexpr int ATOMS = C::ATOMS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tmem_full = bars + 2 * STAGES;
    uint64_t* tmem_empty = bars + 2 * STAGES + 1;
    uint64_t* drain = bars + 2 * STAGES + 2;
    SegTable& seg_tab = *reinterpret_cast<SegTable*>(smem + C::OFF_SEG);
    const float* s_seg_alpha = seg_tab.alpha;
    const int* s_seg_end = seg_tab.end;
    uint32_t* s_tmem_base = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();             // 0: issues the pair's MMAs
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int total_tiles = args.m_tiles * args.n_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, 2 * kEpiWarps);            // both CTAs' epilogue warps
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        prefetch_tmap(&tmap_sfa);
        prefetch_tmap(&tmap_sfb);
        prefetch_tmap(&tmap_y);
    }
    if (warp == 1) {
        tmem_alloc_pair(s_tmem_base, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + NVFP4_MAX_SEGMENTS)
        fill_seg_table(seg_tab, args, threadIdx.x - 64);
    stage_gate_params(seg_tab, args, threadIdx.x, blockDim.x);
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                      // barriers of both CTAs initialised
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem_base;
    const uint32_t full0_leader = mapa_shared(smem_u32(&full[0]), 0);
    const uint32_t tmem_empty_leader = mapa_shared(smem_u32(tmem_empty), 0);

    // The issuing roles run as whole warps with one elected lane issuing, so
    // ring counters, descriptors and addresses stay warp-uniform; only the
    // last stage of K can carry fewer scale atoms than ATOMS.
    const int last_kb = args.k_steps - 1;
    const int last_natoms = args.atoms_per_rb - last_kb * ATOMS;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        const uint64_t pol = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_parity = 0;   // stages the even CTA expects bytes on
        bool ok = true;
        for (int t = pair; t < total_tiles && ok; t += npairs) {
            int mt, nt;
            tile_coords(t, args, mt, nt);
            for (int kb = 0; kb < args.k_steps; ++kb) {
                if (!mbar_wait_warp_pipe(&empty[stage], phase ^ 1u, args.timeout_ns, s_abort, args.status)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = full0_leader + stage * 8;
                if (elect_one()) {
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_TX);
                    tma_load_2d_pair(smem + C::OFF_A + stage * C::A_BYTES, &tmap_a, fb,
                                     kb * KB, mt * 256 + rank * 128, pol);
                    tma_load_2d_pair(smem + C::OFF_B + stage * C::B_BYTES, &tmap_b, fb,
                                     kb * KB, nt * BN + rank * 128, pol);
                    tma_load_2d_pair(smem + C::OFF_SFA + stage * C::SFA_BYTES, &tmap_sfa, fb,
                                     kb * ATOMS * 64, mt * 2 + rank, pol);
                    tma_load_2d_pair(smem + C::OFF_SFB + stage * C::SFB_BYTES, &tmap_sfb, fb,
                                     kb * ATOMS * 64, nt * 2, pol);
                }
                __syncwarp();
                if (rank == 0) {
                    armed |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && rank == 0 && lane == 0) {
            // leave no copy of either CTA in flight on the stages armed here
            int local_abort = 0;
            for (int s = 0; s < STAGES; ++s)
                if (armed & (1u << s))
                    mbar_wait_bounded(&full[s], (armed_parity >> s) & 1u, args.timeout_ns,
                                      &local_abort, args.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (rank == 0) {
            // ---------------- scale copies + MMA issuer (even CTA) ----------------
            constexpr uint32_t idesc = make_idesc_pair();
            // descriptor start-address fields advance by 2 per 32 bytes of K
            const uint64_t da0 = sdesc_kmajor<KB>(smem_u32(smem + C::OFF_A));
            const uint64_t db0 = sdesc_kmajor<KB>(smem_u32(smem + C::OFF_B));
            const uint32_t ssfa0 = smem_u32(smem + C::OFF_SFA);
            const uint32_t ssfb0 = smem_u32(smem + C::OFF_SFB);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int i = 0;
            for (int t = pair; t < total_tiles && ok; t += npairs, ++i) {
                if (!mbar_wait_warp(tmem_empty, (i & 1) ^ 1u, args.timeout_ns, s_abort, args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < args.k_steps; ++kb) {
                    if (!mbar_wait_warp_pipe(&full[stage], phase, args.timeout_ns, s_abort, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = da0 + static_cast<uint64_t>(stage * (C::A_BYTES / 16));
                    const uint64_t db = db0 + static_cast<uint64_t>(stage * (C::B_BYTES / 16));
                    const uint32_t ssfa = ssfa0 + stage * C::SFA_BYTES;
                    const uint32_t ssfb = ssfb0 + stage * C::SFB_BYTES;
                    const uint32_t sfr = tmem_base + BN + stage * C::SF_STRIDE;
                    const uint32_t first = kb != 0;
                    const int natoms = kb == last_kb ? last_natoms : ATOMS;
                    if (elect_one()) {
                        // scale atoms of this stage into its TMEM region (both CTAs),
                        // then the MMAs that read them: same thread, issue order
#pragma unroll
                        for (int j = 0; j < ATOMS; ++j) {
                            if (j < natoms) {
                                tc_copy_scales_pair(sfr + j * 4, sdesc_scales(ssfa + j * kAtom));
                                tc_copy_scales_pair(sfr + C::SFB_COL + j * 8,
                                                    sdesc_scales(ssfb + j * kAtom));
                                tc_copy_scales_pair(sfr + C::SFB_COL + j * 8 + 4,
                                                    sdesc_scales(ssfb + ATOMS * kAtom + j * kAtom));
                            }
                        }
#pragma unroll
                        for (int j = 0; j < ATOMS; ++j) {
                            if (j < natoms)
                                tc_mma_nvf4_pair(tmem_base, da + 2 * j, db + 2 * j, idesc, sfr + j * 4,
                                                 sfr + C::SFB_COL + j * 8, first | static_cast<uint32_t>(j));
                        }
                        tc_commit_pair(&empty[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok && elect_one()) tc_commit_pair(tmem_full, 0x3);
                __syncwarp();
            }
            if (elect_one()) {
                tc_commit_pair(drain, 0x1);
                int local_abort = 0;
                mbar_wait_bounded(drain, 0, args.timeout_ns, &local_abort, args.status);
            }
            __syncwarp();
        }
    } else {
        // ---------------- epilogue (warps 2..9, both CTAs) ----------------
        if constexpr (kSilu) {
            // The weight interleaves gate and up rows in 128-row blocks, so a
            // 256-column tile holds gate columns [0, 128) and the matching up
            // columns [128, 256).  Warp (q, half) writes h columns
            // [64 half, 64 half + 64) of the tile's 128: h = bf16(SiLU(gate) *
            // up) from the FP32 accumulators, and keeps the max |h| (as BF16
            // magnitude bits) for the requantization's global scale.
            const int q = warp & 3;
            const int half = (warp - 2) >> 2;
            const uint64_t pol_y = l2_policy_evict_first();
            const float al = s_seg_alpha[0];
            uint8_t* stage_y = smem + C::OFF_EPI + (warp - 2) * C::EPI_BYTES;
            const uint32_t sy = smem_u32(stage_y);
            const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);
            uint32_t mag = 0;
            int i = 0;
            for (int t = pair; t < total_tiles; t += npairs, ++i) {
                int mt, nt;
                tile_coords(t, args, mt, nt);
                int ok = 1;
                if (lane == 0)
                    ok = mbar_wait_bounded(tmem_full, i & 1, args.timeout_ns, s_abort, args.status);
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (!ok) break;
                tc_fence_after();
                uint32_t r[4][32];
                const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + half * 64;
                tmem_ld_32cols(tq, r[0]);
                tmem_ld_32cols(tq + 32, r[1]);
                tmem_ld_32cols(tq + 128, r[2]);
                tmem_ld_32cols(tq + 160, r[3]);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_relaxed(tmem_empty_leader);
                // every lane computes (the votes below need the whole warp);
                // only rows inside M count toward the max, and the TMA store
                // clips rows beyond M
                const int m0 = mt * 256 + static_cast<int>(rank) * 128 + q * 32;   // row of lane 0
                const bool row_ok = m0 + lane < args.M;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    const int j0 = nt * (BN / 2) + half * 64 + ch * 32;
                    // branch-free FP32 for every element (fast division: within
                    // 2 ulp, far inside the BF16 result's rounding); the rare
                    // g < -80, where e^-g overflows, is redone by the scaled
                    // form of silu_mul_tail after a vote.
                    uint32_t o[16];
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        bool rare = false;
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            const int j = 4 * q8 + jj;
                            const float g0 = __fmul_rn(__uint_as_float(r[ch][2 * j]), al);
                            const float g1 = __fmul_rn(__uint_as_float(r[ch][2 * j + 1]), al);
                            const float u0 = __fmul_rn(__uint_as_float(r[2 + ch][2 * j]), al);
                            const float u1 = __fmul_rn(__uint_as_float(r[2 + ch][2 * j + 1]), al);
                            rare |= (g0 < -80.0f) | (g1 < -80.0f);
                            const float s0 = __fdividef(g0, __fadd_rn(1.0f, expf(-g0)));
                            const float s1 = __fdividef(g1, __fadd_rn(1.0f, expf(-g1)));
                            o[j] = pack_bf16x2(__fmul_rn(s0, u0), __fmul_rn(s1, u1));
                        }
                        if (__any_sync(0xFFFFFFFFu, rare)) {
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) {
                                const int j = 4 * q8 + jj;
                                const float g0 = __fmul_rn(__uint_as_float(r[ch][2 * j]), al);
                                const float g1 = __fmul_rn(__uint_as_float(r[ch][2 * j + 1]), al);
                                if (g0 < -80.0f)
                                    o[j] = (o[j] & 0xFFFF0000u) |
                                           silu_mul1(g0, __fmul_rn(__uint_as_float(r[2 + ch][2 * j]), al));
                                if (g1 < -80.0f)
                                    o[j] = (o[j] & 0xFFFFu) |
                                           (silu_mul1(g1, __fmul_rn(__uint_as_float(r[2 + ch][2 * j + 1]), al)) << 16);
                            }
                        }
                    }
                    if (row_ok) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) mag = max(mag, max(o[j] & 0x7FFFu, (o[j] >> 16) & 0x7FFFu));
                    }
                    if (m0 < args.M) {                                  // warp-uniform
                        // 32 x 32 tile through the staging buffer, one TMA store
                        if (ch > 0) {
                            if (lane == 0) bulk_wait_read_all();
                            __syncwarp();
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            sts128(sy + lane * 64 + ((static_cast<uint32_t>(u) ^ swz) << 4), o[4 * u],
                                   o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmap_y, stage_y, j0, m0, pol_y);
                            bulk_commit_group();
                        }
                    }
                }
                if (lane == 0) bulk_wait_read_all();
                __syncwarp();
            }
            if (lane == 0) bulk_wait_all();
            __syncwarp();
            mag = __reduce_max_sync(0xFFFFFFFFu, mag);
            if (lane == 0 && mag) atomicMax(&args.h_ws[0], mag << 16);
        } else {
        // Each warp owns TMEM lane quarter q (32 rows) and half of the 256
        // columns -- or, in a tile whose columns end within its first half
        // (the last tile when N % 256 <= 128), every other 32-column chunk of
        // that half, so both warps of a quarter share its work (there the
        // gate segments of the fused GDN projection sit).  Per 32-column chunk: alpha and gates in FP32, BF16 RNE,
        // the 32 x 32 tile written into the warp's staging buffer in the
        // 64-byte swizzle (conflict-free: lane i's row is 64 bytes at
        // 64 i, its 16-byte pieces permuted by (i / 2) % 4), then one TMA store
        // of the tile -- whole 32-byte sectors per row, rows and columns
        // beyond M and N clipped by the tensor map.  A lane-per-row st.global
        // would instead send 32 separate 16-byte pieces per instruction.
        constexpr int kHalf = BN / 2;
        constexpr int kChunks = kHalf / 32;
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const uint64_t pol_y = l2_policy_evict_first();
        uint8_t* stage_y = smem + C::OFF_EPI + (warp - 2) * C::EPI_BYTES;
        const uint32_t sy = smem_u32(stage_y);
        const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);
        int i = 0;
        for (int t = pair; t < total_tiles; t += npairs, ++i) {
            int mt, nt;
            tile_coords(t, args, mt, nt);
            // chunk ch of this warp is column chunk chunk_of(ch) of the tile
            const bool narrow = nt * BN + kHalf >= args.N;
            auto chunk_of = [&](int ch) { return narrow ? half + 2 * ch : half * kChunks + ch; };
            const int nch = narrow ? kChunks / 2 : kChunks;
            int ok = 1;
            if (lane == 0)
                ok = mbar_wait_bounded(tmem_full, i & 1, args.timeout_ns, s_abort, args.status);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            uint32_t r[kChunks][32];
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
            for (int ch = 0; ch < kChunks; ++ch)
                if (ch < nch) tmem_ld_32cols(taddr + chunk_of(ch) * 32, r[ch]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            // the values sit in registers: nothing of this thread is left to
            // order before the release (the loads have completed)
            if (lane == 0) mbar_arrive_cluster_relaxed(tmem_empty_leader);
            const int m0 = mt * 256 + static_cast<int>(rank) * 128 + q * 32;   // row of lane 0
            if (m0 >= args.M) continue;                                        // warp-uniform
#pragma unroll
            for (int ch = 0; ch < kChunks; ++ch) {
                if (ch >= nch) break;                                          // warp-uniform
                const int n0 = nt * BN + chunk_of(ch) * 32;
                if (n0 >= args.N) break;                                       // warp-uniform
                int s0 = 0;
                while (s0 < args.nseg - 1 && n0 >= s_seg_end[s0]) ++s0;
                const bool one_seg = (s0 == args.nseg - 1) || (n0 + 31 < s_seg_end[s0]);
                float v[32];
                if (one_seg) {
                    const float al = s_seg_alpha[s0];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(__uint_as_float(r[ch][j]), al);
                } else {
                    int s = s0;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        while (s < args.nseg - 1 && n0 + j >= s_seg_end[s]) ++s;
                        v[j] = __fmul_rn(__uint_as_float(r[ch][j]), s_seg_alpha[s]);
                    }
                }
                if (args.any_act && n0 < args.gate_hi && n0 + 32 > args.gate_lo)
                    apply_gates_copy<32>(v, n0, args.N, args.nseg, seg_tab);
                uint32_t o[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) o[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                // the previous chunk's store has finished reading the buffer
                if (ch > 0) {
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    sts128(sy + lane * 64 + ((static_cast<uint32_t>(u) ^ swz) << 4), o[4 * u],
                           o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmap_y, stage_y, n0, m0, pol_y);
                    bulk_commit_group();
                }
            }
            // the buffer is reused by the next tile's first chunk
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
        }
        // every store of this warp has completed before the CTA exits
        if (lane == 0) bulk_wait_all();
        __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();                                      // no CTA leaves while its peer may signal it
    tc_fence_after();
    if constexpr (kSilu) {
        // the last CTA to finish turns the max |h| into the global scale of h
        if (threadIdx.x == 0) {
            __threadfence();
            const unsigned int tk = atomicAdd(&args.h_ws[1], 1u);
            if (tk == gridDim.x - 1) {
                __threadfence();
                const unsigned int bits = atomicExch(&args.h_ws[0], 0u);
                const float amax = __uint_as_float(bits);
                *args.h_g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
                if (args.h_amax) *args.h_amax = amax;
                atomicExch(&args.h_ws[1], 0u);
            }
        }
    }
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Bounded-wait self-test: one thread waits on a barrier nothing arrives on.
// The wait must give up after limit_ns and set the device status word; the
// context stays usable.  Lets the timeout path be tested without a fault.
// ---------------------------------------------------------------------------
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns, int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        mbar_wait_bounded(&bar, 0, limit_ns, &abort_flag, status);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once (a thread-safe local static); nullptr when the driver has no
// such entry point, which every tensor-map builder below reports as an error.
EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return nullptr;
    }();
    return fn;
}

// [rows, row_bytes] byte matrix read in boxes of box_bytes (128 or 64) x
// box_rows rows, swizzled to the box width, zero fill out of bounds.
bool make_code_map(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t row_bytes,
                   int box_rows, int box_bytes = kBKBytes) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw =
        box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Scale bytes in the tensor-core layout viewed as [row blocks, atoms * 64]
// 8-byte units: one box of box_atoms * 64 units (box_atoms scale atoms of 512
// bytes) x box_rows row blocks is one stage of K for box_rows 128-row blocks.
// Out-of-range row blocks and k positions read as zero.
bool make_sf_map(CUtensorMap* m, const uint8_t* base, int64_t rowblocks, int64_t atoms_per_rb,
                 int box_rows, int box_atoms = kAtomsPerStep) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(atoms_per_rb * 64),
                          static_cast<cuuint64_t>(rowblocks)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(atoms_per_rb * kAtom)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_atoms * 64), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// BF16 output [rows, cols] with row stride ld elements, written by TMA stores
// of 32 x 32 tiles staged in the 64-byte swizzle; boxes reaching past rows or
// cols are clipped.
bool make_out_map(CUtensorMap* m, const uint16_t* base, int64_t rows, int64_t cols, int64_t ld) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

int* device_status_ptr() {
    static int* cache[kMaxDevices] = {nullptr};
    static PerDeviceOnce once;
    int dev = 0;
    if (current_device(&dev) != NVFP4_OK) return nullptr;
    const nvfp4_status st = once.run(dev, [&] {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
        cache[dev] = static_cast<int*>(p);
        return NVFP4_OK;
    });
    return st == NVFP4_OK ? cache[dev] : nullptr;
}

namespace {

template <int BN, int STAGES, int ACC>
nvfp4_status launch_gemm(const uint8_t* a_codes, const uint8_t* w_codes, GemmArgs& args,
                         const DeviceInfo& dev, cudaStream_t stream) {
    using Cf = Cfg<BN, STAGES, ACC>;
    auto kern = nvf4_gemm_kernel<BN, STAGES, ACC>;
    static PerDeviceOnce attr_once;
    int devid = 0;
    nvfp4_status st = current_device(&devid);
    if (st != NVFP4_OK) return st;
    st = attr_once.run(devid, [&] {
        return cuda_status(
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM));
    });
    if (st != NVFP4_OK) return st;
    CUtensorMap ta, tb;
    if (!make_code_map(&ta, a_codes, args.M, args.K / 2, kBM)) return NVFP4_ERR_CUDA;
    if (!make_code_map(&tb, w_codes, args.N, args.K / 2, BN)) return NVFP4_ERR_CUDA;
    args.m_tiles = (args.M + kBM - 1) / kBM;
    args.n_tiles = (args.N + BN - 1) / BN;
    args.nt_first /= BN;
    const int tiles = args.m_tiles * args.n_tiles;
    const int grid = tiles < dev.sms ? tiles : dev.sms;
    kern<<<grid, kThreads, Cf::SMEM, stream>>>(ta, tb, args);
    return cuda_status(cudaGetLastError());
}

template <int STAGES, int KB, bool kSilu = false>
nvfp4_status launch_gemm_pair(const uint8_t* a_codes, const uint8_t* w_codes, GemmArgs& args,
                              const DeviceInfo& dev, cudaStream_t stream) {
    using Cf = PairCfg<STAGES, KB>;
    auto kern = nvf4_gemm_pair_kernel<STAGES, KB, kSilu>;
    static PerDeviceOnce attr_once;
    int devid = 0;
    nvfp4_status st = current_device(&devid);
    if (st != NVFP4_OK) return st;
    st = attr_once.run(devid, [&] {
        return cuda_status(
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM));
    });
    if (st != NVFP4_OK) return st;
    CUtensorMap ta, tb, tsa, tsb, ty;
    const int64_t a_rb = (args.M + 127) / 128, w_rb = (args.N + 127) / 128;
    if (!make_code_map(&ta, a_codes, args.M, args.K / 2, 128, KB)) return NVFP4_ERR_CUDA;
    if (!make_code_map(&tb, w_codes, args.N, args.K / 2, 128, KB)) return NVFP4_ERR_CUDA;
    if (!make_sf_map(&tsa, args.a_sf, a_rb, args.atoms_per_rb, 1, Cf::ATOMS)) return NVFP4_ERR_CUDA;
    if (!make_sf_map(&tsb, args.w_sf, w_rb, args.atoms_per_rb, 2, Cf::ATOMS)) return NVFP4_ERR_CUDA;
    // the output: y [M, N], or h [M, N / 2] for the SiLU epilogue
    if (!make_out_map(&ty, args.y, args.M, kSilu ? args.N / 2 : args.N, args.ldy)) return NVFP4_ERR_CUDA;
    args.k_steps = (args.K + 2 * KB - 1) / (2 * KB);
    args.m_tiles = (args.M + 255) / 256;
    args.n_tiles = (args.N + Cf::BN - 1) / Cf::BN;
    args.nt_first /= Cf::BN;
    const int tiles = args.m_tiles * args.n_tiles;
    const int max_pairs = dev.sms / 2;
    const int pairs = tiles < max_pairs ? tiles : max_pairs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = Cf::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, tsa, tsb, ty, args);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    return cuda_status(cudaGetLastError());
}

// Few tokens (M <= 128): operands swapped, K split over a cluster.  NT and
// the ring depth depend on M alone, the split on K alone (the largest of 1, 2,
// 4, 8 that leaves each CTA at least 8 k-steps), so a row's result never
// depends on N.  Launched as a programmatic dependent of the previous grid on
// the stream (the kernel waits for it before reading any global memory).
nvfp4_status launch_gemm_decode(const uint8_t* a_codes, const uint8_t* w_codes,
                                GemmArgs& args, cudaStream_t stream) {
    auto kern = nvf4_gemm_decode_kernel;
    static PerDeviceOnce attr_once;
    // resident clusters per [device][split][nt_tok / 16], 0 until measured
    static std::atomic<int> max_clusters[kMaxDevices][kDecMaxSplit + 1][9];
    int devid = 0;
    nvfp4_status st = current_device(&devid);
    if (st != NVFP4_OK) return st;
    st = attr_once.run(devid, [&] {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kDecSmemAttr)) != cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
                cudaSuccess)
            return NVFP4_ERR_CUDA;
        return NVFP4_OK;
    });
    if (st != NVFP4_OK) return st;
    DecodeArgs d;
    d.g = args;
    d.nt_tok = ((args.M + 15) / 16) * 16;
    dec_config(d.nt_tok, &d.stages, &d.nparts, &d.nacc);
    d.split = 1;
    while (d.split < kDecMaxSplit && args.k_steps / (2 * d.split) >= 8) d.split *= 2;
    d.g.m_tiles = 1;
    d.g.n_tiles = (args.N + kBM - 1) / kBM;
    const uint32_t smem = dec_layout(d.nt_tok, d.stages, d.nparts).bytes;

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(d.split);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;            // the occupancy query takes the cluster shape only
    // persistent: as many clusters as can be resident at once
    // (racing threads may both measure; they store the same value)
    std::atomic<int>& cached = max_clusters[devid][d.split][d.nt_tok / 16];
    int slots = cached.load(std::memory_order_relaxed);
    if (slots <= 0) {
        cfg.gridDim = dim3(static_cast<unsigned>(d.split), 1, 1);
        if (cudaOccupancyMaxActiveClusters(&slots, kern, &cfg) != cudaSuccess || slots <= 0)
            return NVFP4_ERR_CUDA;
        cached.store(slots, std::memory_order_relaxed);
    }
    const int clusters = d.g.n_tiles < slots ? d.g.n_tiles : slots;
    cfg.gridDim = dim3(static_cast<unsigned>(clusters * d.split), 1, 1);
    cfg.numAttrs = 2;
    CUtensorMap tw, tx;
    if (!make_code_map(&tw, w_codes, args.N, args.K / 2, kBM)) return NVFP4_ERR_CUDA;
    if (!make_code_map(&tx, a_codes, args.M, args.K / 2, d.nt_tok)) return NVFP4_ERR_CUDA;
    if (cudaLaunchKernelEx(&cfg, kern, tw, tx, d) != cudaSuccess) return NVFP4_ERR_CUDA;
    return cuda_status(cudaGetLastError());
}

nvfp4_status gemm_impl(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_g,
                       const uint8_t* w_codes, const uint8_t* w_sf, const nvfp4_segment* segs,
                       const nvfp4_segment_act* acts, int nseg, void* y, int64_t ldy, int64_t M,
                       int64_t K, void* stream) {
    if (!segs || nseg < 1 || nseg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
    if (acts) {
        for (int s = 0; s < nseg; ++s) {
            const int k = acts[s].kind;
            if (k != NVFP4_ACT_NONE && k != NVFP4_ACT_DECAY_GATE && k != NVFP4_ACT_SIGMOID)
                return NVFP4_ERR_INVALID_ARG;
            if (k == NVFP4_ACT_DECAY_GATE && (!acts[s].a_log || !acts[s].dt_bias))
                return NVFP4_ERR_INVALID_ARG;
        }
    }
    if (M < 0 || K < 0 || !a_g) return NVFP4_ERR_INVALID_ARG;
    int64_t N = 0;
    for (int s = 0; s < nseg; ++s) {
        if (segs[s].n_offset != N || segs[s].n_size <= 0 || !segs[s].w_gscale)
            return NVFP4_ERR_INVALID_ARG;
        if (segs[s].n_size >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
        N += segs[s].n_size;   // at most 16 terms below 2^31: no overflow
    }
    if (K % 32 != 0 || K < 32) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ldy < N || ldy % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    if (extent_too_large(M, ldy, 2)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    // tile indices are 32-bit in the kernels (128 x 128 tiles at the finest),
    // and a persistent CTA adds the grid size to its index
    if (((M + 127) / 128) * ((N + 127) / 128) >= (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return NVFP4_OK;
    if (!a_codes || !a_sf || !w_codes || !w_sf || !y) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(w_codes) || !aligned16(w_sf) ||
        !aligned16(y))
        return NVFP4_ERR_ALIGNMENT;
    // the epilogues read the scales and gate parameters while other CTAs write y
    {
        const size_t ybytes = extent_bytes(M, ldy, N, 2);
        if (overlaps(a_g, 4, y, ybytes)) return NVFP4_ERR_INVALID_ARG;
        for (int s = 0; s < nseg; ++s) {
            const size_t pb = static_cast<size_t>(segs[s].n_size) * 4;
            // the parameter arrays are read only for a decay gate (unused otherwise)
            const bool decay = acts && acts[s].kind == NVFP4_ACT_DECAY_GATE;
            if (overlaps(segs[s].w_gscale, 4, y, ybytes) ||
                (decay && overlaps(acts[s].a_log, pb, y, ybytes)) ||
                (decay && overlaps(acts[s].dt_bias, pb, y, ybytes)))
                return NVFP4_ERR_INVALID_ARG;
        }
    }
    DeviceInfo dev;
    nvfp4_status st = require_sm100(&dev);
    if (st != NVFP4_OK) return st;
    int* status = device_status_ptr();
    if (!status) return NVFP4_ERR_CUDA;

    GemmArgs args = {};
    args.a_sf = a_sf;
    args.w_sf = w_sf;
    args.a_g = a_g;
    args.y = static_cast<uint16_t*>(y);
    args.ldy = ldy;
    args.M = static_cast<int>(M);
    args.N = static_cast<int>(N);
    args.K = static_cast<int>(K);
    args.k_steps = static_cast<int>((K + 255) / 256);
    args.atoms_per_rb = static_cast<int>((K + 63) / 64);
    args.w_rowblocks = static_cast<int>((N + 127) / 128);
    // Raster: when the quantized activation fits comfortably in L2, sweep every
    // M tile for each N tile (the weight then streams from HBM once);
    // otherwise walk bands of 16 M tiles.
    args.group_m = (M * (K / 2) <= (int64_t(48) << 20)) ? 1 << 30 : 16;
    args.nseg = nseg;
    args.any_act = 0;
    args.gate_lo = 0x7FFFFFFF;
    args.gate_hi = 0;
    int gate_cols = 0;
    for (int s = 0; s < nseg; ++s) {
        args.seg_goff[s] = gate_cols;
        if (acts && acts[s].kind == NVFP4_ACT_DECAY_GATE) gate_cols += static_cast<int>(segs[s].n_size);
        args.seg_end[s] = static_cast<int>(segs[s].n_offset + segs[s].n_size);
        args.seg_g[s] = segs[s].w_gscale;
        args.seg_kind[s] = acts ? acts[s].kind : NVFP4_ACT_NONE;
        args.seg_p0[s] = acts ? acts[s].a_log : nullptr;
        args.seg_p1[s] = acts ? acts[s].dt_bias : nullptr;
        if (args.seg_kind[s] != NVFP4_ACT_NONE) {
            args.any_act = 1;
            args.gate_lo = std::min(args.gate_lo, static_cast<int>(segs[s].n_offset));
            args.gate_hi = std::max(args.gate_hi, static_cast<int>(segs[s].n_offset + segs[s].n_size));
        }
    }
    if (gate_cols > kMaxGateCols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    // the n-tile width is the kernel's: the launchers turn this column into
    // the first n-tile of the sweep (0 without gates)
    args.nt_first = args.any_act ? args.gate_lo : 0;
    args.timeout_ns = kTimeoutNs;
    args.status = status;
    cudaStream_t cs = as_stream(stream);
    // The configuration depends on M only, so a fused GEMM and its per-module
    // GEMMs accumulate every output element identically.
    if (M > 256) return launch_gemm_pair<kPairStages, kPairKB>(a_codes, w_codes, args, dev, cs);
    if (M <= kBM) return launch_gemm_decode(a_codes, w_codes, args, cs);
    return launch_gemm<128, 6, 2>(a_codes, w_codes, args, dev, cs);
}

// gate_up GEMM with the SiLU(gate) * up epilogue and the global scale of h.
nvfp4_status gemm_silu_impl(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_g,
                            const uint8_t* w_codes, const uint8_t* w_sf, const float* w_g, void* h,
                            int64_t ldh, int64_t M, int64_t F, int64_t K, void* workspace,
                            float* h_g, float* h_amax, void* stream) {
    if (M < 0 || F <= 0 || K < 0 || !a_g || !w_g || !h_g || !workspace) return NVFP4_ERR_INVALID_ARG;
    if (F % 128 != 0 || K % 32 != 0 || K < 32) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M >= (int64_t(1) << 31) || F >= (int64_t(1) << 30) || K >= (int64_t(1) << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ldh < F || ldh % 8 != 0) return NVFP4_ERR_ALIGNMENT;
    if (extent_too_large(M, ldh, 2)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (((M + 255) / 256) * ((2 * F + 255) / 256) >= (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (M <= 256) return NVFP4_ERR_UNSUPPORTED_SHAPE;      // the CTA-pair (prefill) kernel only
    if (!a_codes || !a_sf || !w_codes || !w_sf || !h) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(w_codes) || !aligned16(w_sf) ||
        !aligned16(h) || !aligned16(workspace))
        return NVFP4_ERR_ALIGNMENT;
    // the last CTA writes the scale of h and then clears the workspace; the
    // epilogues read the input scales while other CTAs write h
    const size_t hbytes = extent_bytes(M, ldh, F, 2);
    if (overlaps(h_g, 4, workspace, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES) ||
        overlaps(h_amax, 4, workspace, NVFP4_GLOBAL_SCALE_WORKSPACE_BYTES) ||
        overlaps(a_g, 4, h, hbytes) || overlaps(w_g, 4, h, hbytes))
        return NVFP4_ERR_INVALID_ARG;
    DeviceInfo dev;
    nvfp4_status st = require_sm100(&dev);
    if (st != NVFP4_OK) return st;
    int* status = device_status_ptr();
    if (!status) return NVFP4_ERR_CUDA;
    const int64_t N = 2 * F;
    GemmArgs args = {};
    args.a_sf = a_sf;
    args.w_sf = w_sf;
    args.a_g = a_g;
    args.y = static_cast<uint16_t*>(h);
    args.ldy = ldh;
    args.M = static_cast<int>(M);
    args.N = static_cast<int>(N);
    args.K = static_cast<int>(K);
    args.k_steps = static_cast<int>((K + 255) / 256);
    args.atoms_per_rb = static_cast<int>((K + 63) / 64);
    args.w_rowblocks = static_cast<int>(N / 128);
    args.group_m = (M * (K / 2) <= (int64_t(48) << 20)) ? 1 << 30 : 16;
    args.nseg = 1;
    args.seg_end[0] = static_cast<int>(N);
    args.seg_g[0] = w_g;
    args.seg_kind[0] = NVFP4_ACT_NONE;
    args.gate_lo = 0x7FFFFFFF;
    args.timeout_ns = kTimeoutNs;
    args.status = status;
    args.h_ws = static_cast<unsigned int*>(workspace);
    args.h_g = h_g;
    args.h_amax = h_amax;
    return launch_gemm_pair<kPairStages, kPairKB, true>(a_codes, w_codes, args, dev, as_stream(stream));
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_gemm_silu_mul(const uint8_t* a_codes, const uint8_t* a_sf,
                                            const float* a_g, const uint8_t* w_codes,
                                            const uint8_t* w_sf, const float* w_g, void* h,
                                            int64_t ldh, int64_t M, int64_t F, int64_t K,
                                            void* workspace, float* h_g, float* h_amax,
                                            void* stream) {
    return gemm_silu_impl(a_codes, a_sf, a_g, w_codes, w_sf, w_g, h, ldh, M, F, K, workspace, h_g,
                          h_amax, stream);
}

extern "C" nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_g,
                                   const uint8_t* w_codes, const uint8_t* w_sf, const float* w_g,
                                   void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                                   void* stream) {
    if (N < 0 || !w_g) return NVFP4_ERR_INVALID_ARG;
    if (N == 0) return (M >= 0 && K >= 0) ? NVFP4_OK : NVFP4_ERR_INVALID_ARG;
    nvfp4_segment seg = {0, N, w_g};
    return gemm_impl(a_codes, a_sf, a_g, w_codes, w_sf, &seg, nullptr, 1, y, ldy, M, K, stream);
}

extern "C" nvfp4_status nvfp4_fused_gemm(const uint8_t* a_codes, const uint8_t* a_sf,
                                         const float* a_g, const uint8_t* w_codes,
                                         const uint8_t* w_sf, const nvfp4_segment* segs, int nseg,
                                         void* y, int64_t ldy, int64_t M, int64_t K,
                                         void* stream) {
    return gemm_impl(a_codes, a_sf, a_g, w_codes, w_sf, segs, nullptr, nseg, y, ldy, M, K, stream);
}

extern "C" nvfp4_status nvfp4_fused_gemm_act(const uint8_t* a_codes, const uint8_t* a_sf,
                                             const float* a_g, const uint8_t* w_codes,
                                             const uint8_t* w_sf, const nvfp4_segment* segs,
                                             const nvfp4_segment_act* acts, int nseg, void* y,
                                             int64_t ldy, int64_t M, int64_t K, void* stream) {
    return gemm_impl(a_codes, a_sf, a_g, w_codes, w_sf, segs, acts, nseg, y, ldy, M, K, stream);
}

extern "C" nvfp4_status nvfp4_last_device_status(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        return NVFP4_ERR_TIMEOUT;
    }
    return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_debug_wait_timeout(int64_t limit_ns, void* stream) {
    if (limit_ns <= 0 || limit_ns > 1000000000) return NVFP4_ERR_INVALID_ARG;
    int* status = device_status_ptr();
    if (!status) return NVFP4_ERR_CUDA;
    wait_timeout_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(limit_ns),
                                                                 status);
    return cuda_status(cudaGetLastError());
}

extern "C" const char* nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_ERR_ALIGNMENT: return "pointer or stride not aligned";
        case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case NVFP4_ERR_CUDA: return "CUDA error";
        case NVFP4_ERR_TIMEOUT: return "device-side wait timed out";
        case NVFP4_ERR_DEVICE: return "device is not sm_100";
    }
    return "unknown status";
}

extern "C" int nvfp4_version(void) { return 100; }
