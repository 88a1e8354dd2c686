// gemm_decode.cuh -- the W4A4 GEMM for few tokens (M <= 128), where the
// weights stream from HBM once and nothing else matters.  Included by gemm.cu
// (shares GemmArgs and the tile constants); same result formula:
//
// Y[m, n] = bf16( fl32( acc[m, n] * fl32(gA * gW[seg(n)]) ) ).
//
// Layout of the work (sm_100a):
//   * Operands swapped: 128 weight rows sit on the MMA's M side and the tokens,
//     padded to NT = 16..128, on its N side, so a tile is 128 outputs wide in n
//     whatever the token count.
//   * K is split over a cluster of S CTAs (S = 1, 2, 4 or 8, chosen from K
//     alone: the largest that leaves every CTA at least 8 k-steps, since
//     each further split costs a partial-sum exchange per tile); each CTA
//     accumulates its fixed K slice of a tile in TMEM.
//   * Persistent: one cluster per scheduling slot; cluster c takes weight
//     tiles c, c + C, c + 2C, ...  The shared-memory ring runs across tiles, so
//     weight loads stay in flight while earlier tiles drain.
//   * Split-K reduction through distributed shared memory: every CTA pushes its
//     FP32 partial of each row (the real tokens' columns only) to the CTA
//     owning that row (128/S rows each);
//     the owner adds the S partials in rank order 0..S-1 (a fixed order: the
//     result depends on neither N nor the segment table nor timing), applies
//     alpha and writes BF16.  Handshakes are mbarriers arrived on across the
//     cluster, so no role waits on a cluster-wide barrier inside the loop.
//   * The block scales go shared -> registers -> TMEM with tcgen05.st from four
//     warps (one per TMEM lane quarter) instead of tcgen05.cp, writing the same
//     replicated layout the copy would: lane l of every quarter holds bytes
//     [16 l, 16 l + 16) of each 512-byte scale atom in four columns.
//   * Start-up: warp 0 sets up the barriers (one lane per ring stage) and
//     starts the weight stream without waiting for the TMEM allocation; the
//     feed-loop waits of the producer and the MMA warp spin on the phase
//     instead of suspending, so the two handshakes of every stage add no
//     wake-up latency.
//   * Launched as a programmatic dependent: each CTA lets the next grid on
//     the stream launch at once, so that grid's CTAs set up on the SMs this
//     one leaves while its last tiles drain; every role that reads global
//     memory first waits for the previous grid (griddepcontrol.wait), so
//     stream order holds for all data.
//
// Roles (14 warps): 0 TMA producer; 1 TMEM owner and MMA issuer; 2..5 scale
// writers; 6..9 pushers (accumulator -> owners' shared memory); 10..13
// reducers (rank-order sum, alpha, BF16 store).  Up to four accumulators and
// four partial buffers keep several tiles in flight between the MMA and the
// store, so the cluster handshakes overlap the weight stream.
// TMEM (512 columns, one CTA per SM): the accumulators in columns 0..255,
// then one 32-column scale slot per ring stage.  Every wait is bounded; on a
// timeout all roles stop, drain what is in flight and meet at the final
// cluster barrier.

constexpr int kDecThreads = 448;
constexpr int kDecSfCol = 256;        // TMEM column of the first scale slot
constexpr int kDecSfSlot = 32;        // columns per stage: 16 weight + 16 token scales
constexpr int kDecTmemCols = 512;
constexpr int kDecMaxSplit = 8;
constexpr int kDecMaxStages = 8;
constexpr int kDecMaxAcc = 4;
constexpr int kDecMaxParts = 4;
constexpr int kDecHeld = 2;           // reduced outputs a reducer holds before its stores
constexpr uint32_t kDecStageBudget = 210 * 1024;   // ring + partial buffers
constexpr uint32_t kDecMinSmem = 116 * 1024;       // > half an SM: one CTA per SM
constexpr uint32_t kDecSmemAttr = kDecStageBudget + 4096;   // dynamic shared memory granted
static_assert(2 * kDecMinSmem > 228 * 1024,
              "two decode CTAs could share an SM (and its 512 TMEM columns)");

struct DecodeArgs {
    GemmArgs g;
    int nt_tok;      // MMA N: tokens padded to a multiple of 16 (16..128)
    int split;       // CTAs per cluster along K
    int stages;      // shared-memory ring depth
    int nparts;      // partial-sum buffers
    int nacc;        // TMEM accumulators (256 / nacc columns apart)
};

struct DecLayout {
    uint32_t off_w, off_x, off_sfw, off_sfx, off_part, off_bar, off_seg, off_misc, bytes;
};

__host__ __device__ constexpr uint32_t dec_stage_bytes(int nt_tok) {
    return kBM * kBKBytes + nt_tok * kBKBytes + 2 * kAtomsPerStep * kAtom;
}

__host__ __device__ constexpr uint32_t dec_part_bytes(int nt_tok) {
    return static_cast<uint32_t>(nt_tok) * kBM * 4;
}

__host__ __device__ constexpr DecLayout dec_layout(int nt_tok, int stages, int nparts) {
    DecLayout L{};
    L.off_w = 0;
    L.off_x = L.off_w + stages * kBM * kBKBytes;
    L.off_sfw = L.off_x + stages * nt_tok * kBKBytes;
    L.off_sfx = L.off_sfw + stages * kAtomsPerStep * kAtom;
    L.off_part = L.off_sfx + stages * kAtomsPerStep * kAtom;
    L.off_bar = L.off_part + nparts * dec_part_bytes(nt_tok);
    // full, empty, sf_ready per stage; tmem_full, tmem_empty per accumulator;
    // part_full, part_free per partial buffer; drain
    L.off_seg = L.off_bar + (3 * stages + 2 * kDecMaxAcc + 2 * nparts + 1) * 8;
    L.off_misc = L.off_seg + static_cast<uint32_t>((sizeof(SegTable) + 15) / 16 * 16);
    uint32_t bytes = L.off_misc + 16 + 1024;   // + slack for 1024-byte alignment
    L.bytes = bytes < kDecMinSmem ? kDecMinSmem : bytes;
    return L;
}

// Accumulators, partial buffers and ring depth for a token width.
__host__ __device__ constexpr void dec_config(int nt_tok, int* stages, int* nparts, int* nacc) {
    // four partial buffers only where they still leave the ring its eight
    // stages (width 16); from width 32 two, so the ring keeps seven stages
    const int np = nt_tok <= 16 ? 4 : (nt_tok <= 64 ? 2 : 1);
    int st = static_cast<int>((kDecStageBudget - np * dec_part_bytes(nt_tok)) / dec_stage_bytes(nt_tok));
    st = st > kDecMaxStages ? kDecMaxStages : st;
    *stages = st < 2 ? 2 : st;
    *nparts = np;
    *nacc = nt_tok <= 64 ? 4 : 2;
}

// Every configuration the launcher can pick (token widths 16..128) fits the
// hardware: ring and partial buffers within the shared memory the kernel is
// granted (and the 227 KB a CTA may have), 2..8 stages, the scale slots of
// all stages within the 512 TMEM columns, each accumulator's NT columns
// within its share of columns 0..255, and the operand tiles on the 1024-byte
// boundaries their 128-byte swizzle needs (scales and partials on 16 bytes,
// barriers on 8, the segment table and the two status words, all read as
// 4-byte scalars, on 4).
constexpr bool dec_configs_fit() {
    for (int nt = 16; nt <= 128; nt += 16) {
        int st = 0, np = 0, na = 0;
        dec_config(nt, &st, &np, &na);
        const DecLayout L = dec_layout(nt, st, np);
        if (L.bytes > kDecSmemAttr || L.bytes > 227 * 1024) return false;
        if (st < 2 || st > kDecMaxStages || np < 1 || np > kDecMaxParts || na < 1 || na > kDecMaxAcc)
            return false;
        if (kDecSfCol + st * kDecSfSlot > kDecTmemCols || nt > 256 / na) return false;
        if (L.off_x % 1024 != 0 || L.off_sfw % 16 != 0 || L.off_sfx % 16 != 0 ||
            L.off_part % 16 != 0 || L.off_bar % 8 != 0 || L.off_seg % 4 != 0 || L.off_misc % 4 != 0)
            return false;
    }
    return true;
}
static_assert(dec_configs_fit(), "a decode configuration exceeds a hardware limit");

__device__ __forceinline__ uint32_t make_idesc_dec(int nt_tok) {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nt_tok >> 3) << 17) |
           (static_cast<uint32_t>(kBM >> 4) << 24);
}

__global__ void __launch_bounds__(kDecThreads, 1)
nvf4_gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w,
                        const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ DecodeArgs dargs) {
    const GemmArgs& args = dargs.g;
    const int NT = dargs.nt_tok;
    const int S = dargs.split;
    const int STAGES = dargs.stages;
    const int NPART = dargs.nparts;
    const int NACC = dargs.nacc;
    const int ACC_STRIDE = 256 / NACC;
    const DecLayout L = dec_layout(NT, STAGES, NPART);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.off_bar);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* sf_ready = bars + 2 * STAGES;
    uint64_t* tmem_full = bars + 3 * STAGES;          // [kDecMaxAcc]
    uint64_t* tmem_empty = tmem_full + kDecMaxAcc;    // [kDecMaxAcc]
    uint64_t* part_full = tmem_empty + kDecMaxAcc;    // [NPART]: partials of my rows landed
    uint64_t* part_free = part_full + NPART;          // [NPART]: every owner done with a buffer
    uint64_t* drain = part_free + NPART;
    SegTable& seg_tab = *reinterpret_cast<SegTable*>(smem + L.off_seg);
    const float* s_seg_alpha = seg_tab.alpha;
    const int* s_seg_end = seg_tab.end;
    uint32_t* s_tmem_base = reinterpret_cast<uint32_t*>(smem + L.off_misc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L.off_misc + 4);
    float* part = reinterpret_cast<float*>(smem + L.off_part);   // [NPART][S][NT][128/S]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    grid_launch_dependents();
    const int rank = static_cast<int>(cluster_ctarank());
    const int cluster_id = blockIdx.x / S;
    const int num_clusters = gridDim.x / S;
    const int k_begin = (rank * args.k_steps) / S;
    const int k_end = ((rank + 1) * args.k_steps) / S;
    const int R = kBM / S;                  // rows of a tile owned by each CTA

    if (warp == 0) {
        // lane i sets up the barriers of ring stage i, accumulator i and
        // partial buffer i; the warp then goes straight to the weight stream
        // (named barrier 2: arrive only), the others wait for the set-up and
        // the TMEM allocation
        if (lane < STAGES) {
            mbar_init(&full[lane], 1);
            mbar_init(&empty[lane], 1);
            mbar_init(&sf_ready[lane], 4);
        }
        if (lane < kDecMaxAcc) {
            mbar_init(&tmem_full[lane], 1);
            mbar_init(&tmem_empty[lane], 4);      // the four pusher warps
        }
        if (lane < NPART) {
            mbar_init(&part_full[lane], kBM);     // R rows from each of the S CTAs
            mbar_init(&part_free[lane], 4 * S);   // the 4 reducer warps of each of the S CTAs
        }
        if (lane == 0) {
            mbar_init(drain, 1);
            *s_abort = 0;
            prefetch_tmap(&tmap_w);
            prefetch_tmap(&tmap_x);
        }
        fence_mbar_init();
        __syncwarp();
        named_barrier_arrive(2, kDecThreads);
    } else {
        if (warp == 1) {
            tmem_alloc(s_tmem_base, kDecTmemCols);
            tmem_relinquish();
        }
        tc_fence_before();
        named_barrier_sync(2, kDecThreads);
        tc_fence_after();
    }
    const uint32_t tmem_base = warp == 0 ? 0u : *s_tmem_base;   // the producer needs none
    // Cross-CTA set-up without holding up the weight stream: every thread
    // arrives on the cluster barrier now; the roles that touch a peer's
    // shared memory or barriers (pushers, reducers) wait on it before their
    // first remote access, the others only at the end.  The producer and the
    // MMA warp use local barriers only, so the first weight loads leave at once.
    cluster_arrive();

    // Loop-invariant step data.  Every role walks the same (tile, k-step)
    // sequence with incremental ring counters -- no division in the loops;
    // only the last k-step of K can carry fewer than four scale atoms.
    const int last_kb = args.k_steps - 1;
    const int last_natoms = args.atoms_per_rb - last_kb * kAtomsPerStep;
    const uint32_t s_w0 = smem_u32(smem + L.off_w);
    const uint32_t s_x0 = smem_u32(smem + L.off_x);
    const uint32_t s_sfw0 = smem_u32(smem + L.off_sfw);
    const uint32_t s_sfx0 = smem_u32(smem + L.off_sfx);
    const uint32_t x_stride = static_cast<uint32_t>(NT) * kBKBytes;

    if (warp == 0) {
        // ---------------- TMA producer (whole warp; one elected lane issues) ----------------
        grid_dependency_wait();     // weights, tokens and scales may come from the previous grid
        const uint64_t pol_w = l2_policy_evict_first();   // each weight byte is read once
        const uint64_t pol_x = l2_policy_evict_last();    // tokens are read by every tile
        const uint32_t full_bytes = kBM * kBKBytes + NT * kBKBytes + 2 * kAtomsPerStep * kAtom;
        const uint32_t last_bytes = kBM * kBKBytes + NT * kBKBytes + 2 * last_natoms * kAtom;
        uint32_t issued = 0, issued_parity = 0;
        bool ok = true;
        int stage = 0;
        uint32_t phase = 0;
        for (int nt = cluster_id; nt < args.n_tiles && ok; nt += num_clusters) {
            const uint8_t* wsf = args.w_sf + (static_cast<size_t>(nt) * args.atoms_per_rb +
                                              static_cast<size_t>(k_begin) * kAtomsPerStep) * kAtom;
            const uint8_t* xsf = args.a_sf + static_cast<size_t>(k_begin) * kAtomsPerStep * kAtom;
            for (int kb = k_begin; kb < k_end; ++kb) {
                if (!mbar_spin_warp(&empty[stage], phase ^ 1u, args.timeout_ns, s_abort, args.status)) {
                    ok = false;
                    break;
                }
                const bool last = kb == last_kb;
                const uint32_t sf_bytes = (last ? last_natoms : kAtomsPerStep) * kAtom;
                uint64_t* fb = &full[stage];
                if (elect_one()) {
                    mbar_arrive_expect_tx(fb, last ? last_bytes : full_bytes);
                    tma_load_2d(smem + L.off_w + stage * (kBM * kBKBytes), &tmap_w, fb,
                                kb * kBKBytes, nt * kBM, pol_w);
                    tma_load_2d(smem + L.off_x + stage * x_stride, &tmap_x, fb, kb * kBKBytes, 0, pol_x);
                    bulk_load(smem + L.off_sfw + stage * (kAtomsPerStep * kAtom), wsf, sf_bytes, fb, pol_w);
                    bulk_load(smem + L.off_sfx + stage * (kAtomsPerStep * kAtom), xsf, sf_bytes, fb, pol_x);
                }
                __syncwarp();
                wsf += kAtomsPerStep * kAtom;
                xsf += kAtomsPerStep * kAtom;
                issued |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            // leave no copy in flight: wait (bounded) for every stage issued
            int local_abort = 0;
            for (int st = 0; st < STAGES; ++st)
                if (issued & (1u << st))
                    mbar_wait_bounded(&full[st], (issued_parity >> st) & 1u, args.timeout_ns,
                                      &local_abort, args.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
        const uint32_t idesc = make_idesc_dec(NT);
        // descriptor start-address fields advance by 2 per 32 bytes of K
        const uint64_t dw0 = sdesc_kmajor_sw128(s_w0);
        const uint64_t dx0 = sdesc_kmajor_sw128(s_x0);
        const uint32_t sf0 = tmem_base + kDecSfCol;
        bool ok = true;
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        for (int nt = cluster_id; nt < args.n_tiles && ok; nt += num_clusters) {
            if (!mbar_spin_warp(&tmem_empty[acc], acc_phase ^ 1u, args.timeout_ns, s_abort,
                                args.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + acc * ACC_STRIDE;
            for (int kb = k_begin; kb < k_end; ++kb) {
                if (!mbar_spin_warp(&sf_ready[stage], phase, args.timeout_ns, s_abort, args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t dw = dw0 + static_cast<uint64_t>(stage * (kBM * kBKBytes / 16));
                const uint64_t dx = dx0 + static_cast<uint64_t>(stage * (x_stride / 16));
                const uint32_t sf = sf0 + stage * kDecSfSlot;
                const uint32_t first = kb != k_begin;
                const int natoms = kb == last_kb ? last_natoms : kAtomsPerStep;
                if (elect_one()) {
                    if (natoms == kAtomsPerStep) {
#pragma unroll
                        for (int j = 0; j < kAtomsPerStep; ++j)
                            tc_mma_nvf4(d_tmem, dw + 2 * j, dx + 2 * j, idesc, sf + j * 4,
                                        sf + 16 + j * 4, first | static_cast<uint32_t>(j));
                    } else {
                        for (int j = 0; j < natoms; ++j)
                            tc_mma_nvf4(d_tmem, dw + 2 * j, dx + 2 * j, idesc, sf + j * 4,
                                        sf + 16 + j * 4, first | static_cast<uint32_t>(j));
                    }
                    tc_commit(&empty[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok && elect_one()) tc_commit(&tmem_full[acc]);
            __syncwarp();
            if (++acc == NACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        // every tcgen05 operation issued above has finished before TMEM is freed
        if (elect_one()) {
            tc_commit(drain);
            int local_abort = 0;
            mbar_wait_bounded(drain, 0, args.timeout_ns, &local_abort, args.status);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ---------------- scale writers (warps 2..5) ----------------
        const int q = warp & 3;                   // TMEM lane quarter of this warp
        const uint32_t sf0 = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kDecSfCol;
        const uint32_t lane_off = lane * 16;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int nt = cluster_id; nt < args.n_tiles && ok; nt += num_clusters) {
            for (int kb = k_begin; kb < k_end; ++kb) {
                int got = 1;
                if (lane == 0)
                    got = mbar_wait_bounded(&full[stage], phase, args.timeout_ns, s_abort,
                                            args.status);
                got = __shfl_sync(0xFFFFFFFFu, got, 0);
                if (!got) {
                    ok = false;
                    break;
                }
                tc_fence_after();   // the MMAs that last read this scale slot have completed
                const int natoms = kb == last_kb ? last_natoms : kAtomsPerStep;
                const uint32_t sfw = s_sfw0 + stage * (kAtomsPerStep * kAtom) + lane_off;
                const uint32_t sfx = s_sfx0 + stage * (kAtomsPerStep * kAtom) + lane_off;
                uint32_t rw[16], rx[16];
#pragma unroll
                for (int j = 0; j < kAtomsPerStep; ++j) {
                    uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
                    if (j < natoms) {
                        a = lds128(sfw + j * kAtom);
                        b = lds128(sfx + j * kAtom);
                    }
                    rw[4 * j] = a.x; rw[4 * j + 1] = a.y; rw[4 * j + 2] = a.z; rw[4 * j + 3] = a.w;
                    rx[4 * j] = b.x; rx[4 * j + 1] = b.y; rx[4 * j + 2] = b.z; rx[4 * j + 3] = b.w;
                }
                const uint32_t sf = sf0 + stage * kDecSfSlot;
                tmem_st_16cols(sf, rw);
                tmem_st_16cols(sf + 16, rx);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp < 10) {
        // ---------------- pushers (warps 6..9) ----------------
        // accumulator row `row` (this thread's TMEM lane) -> slot [rank][t][rr]
        // of the CTA that owns the row, then one arrival on the owner's part_full
        const int q = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const int row = q * 32 + lane;
        const int owner = row / R;
        const int rr = row - owner * R;
        const uint32_t part_owner = mapa_shared(smem_u32(part), static_cast<uint32_t>(owner));
        const uint32_t full_owner0 = mapa_shared(smem_u32(part_full), static_cast<uint32_t>(owner));
        cluster_wait();                     // the owners' barriers are initialised
        int i = 0;
        for (int nt = cluster_id; nt < args.n_tiles; nt += num_clusters, ++i) {
            const int acc = i % NACC;
            const int pb = i % NPART;
            const int puse = i / NPART;
            int got = 1;
            if (lane == 0)
                got = mbar_wait_bounded(&tmem_full[acc], (i / NACC) & 1u, args.timeout_ns, s_abort,
                                        args.status);
            if (puse > 0 && got && lane == 0)
                got = mbar_wait_cluster_bounded(&part_free[pb], (puse - 1) & 1u, args.timeout_ns,
                                                s_abort, args.status);
            got = __shfl_sync(0xFFFFFFFFu, got, 0);
            if (!got) break;
            tc_fence_after();
            const uint32_t dst = part_owner + static_cast<uint32_t>(
                pb * dec_part_bytes(NT) + ((rank * NT) * R + rr) * 4);
            for (int c = 0; c < args.M; c += 16) {      // the columns of real tokens only
                uint32_t r[16];
                tmem_ld_16cols(tmem_base + lane_base + acc * ACC_STRIDE + c, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c + j < args.M)
                        st_shared_cluster_f32(dst + static_cast<uint32_t>((c + j) * R * 4),
                                              __uint_as_float(r[j]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[acc]);       // the MMA may reuse it
            mbar_arrive_cluster(full_owner0 + pb * 8);          // my row's partial has landed
        }
    } else {
        // ---------------- reducers (warps 10..13) ----------------
        // thread -> 4 consecutive owned rows (alpha looked up once per tile) and
        // every (4 S)-th token; partials read as float4, sums in rank order.
        // The results stay in registers until this warp has released the
        // partial buffer, so that release never waits on the global stores.
        const int red_tid = threadIdx.x - 10 * 32;
        grid_dependency_wait();     // the activation scale may come from the previous grid
        // the segment table and gate parameters are the reducers' alone
        if (red_tid < NVFP4_MAX_SEGMENTS) fill_seg_table(seg_tab, args, red_tid);
        stage_gate_params(seg_tab, args, red_tid, 128);
        named_barrier_sync(1, 128);
        cluster_wait();                     // the peers' barriers are initialised
        const int ngroups = R / 4;
        const int rg = red_tid % ngroups;
        const int tstep = 128 / ngroups;
        const int t_first = red_tid / ngroups;
        int sg_first = 0;           // segment of this thread's first row: rows only grow from tile to tile
        int i = 0;
        for (int nt = cluster_id; nt < args.n_tiles; nt += num_clusters, ++i) {
            const int pb = i % NPART;
            const int puse = i / NPART;
            const int got = mbar_wait_cluster_bounded(&part_full[pb], puse & 1u, args.timeout_ns,
                                                      s_abort, args.status);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            const float* pbuf = part + pb * (dec_part_bytes(NT) / 4);
            const int n0 = nt * kBM + rank * R + 4 * rg;
            while (sg_first < args.nseg - 1 && n0 >= s_seg_end[sg_first]) ++sg_first;
            float al[4];
            int sgi = sg_first;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                while (sgi < args.nseg - 1 && n0 + u >= s_seg_end[sgi]) ++sgi;
                al[u] = s_seg_alpha[sgi];
            }
            const bool full4 = n0 + 3 < args.N;
            const int t_end = NT < args.M ? NT : args.M;
            const int niter = t_first < t_end ? (t_end - t_first + tstep - 1) / tstep : 0;
            const int slot_stride = NT * R;          // floats between the partials of two ranks
            auto reduce_one = [&](int t) -> uint2 {
                // all S partials are loaded before the rank-ordered adds
                const float* p0 = pbuf + t * R + 4 * rg;
                float4 p[kDecMaxSplit];
#pragma unroll
                for (int qq = 0; qq < kDecMaxSplit; ++qq)
                    if (qq < S) p[qq] = *reinterpret_cast<const float4*>(p0 + qq * slot_stride);
                float4 sum = p[0];
#pragma unroll
                for (int qq = 1; qq < kDecMaxSplit; ++qq) {
                    if (qq < S) {
                        sum.x = __fadd_rn(sum.x, p[qq].x);
                        sum.y = __fadd_rn(sum.y, p[qq].y);
                        sum.z = __fadd_rn(sum.z, p[qq].z);
                        sum.w = __fadd_rn(sum.w, p[qq].w);
                    }
                }
                float o4[4] = {__fmul_rn(sum.x, al[0]), __fmul_rn(sum.y, al[1]),
                               __fmul_rn(sum.z, al[2]), __fmul_rn(sum.w, al[3])};
                if (args.any_act && n0 < args.gate_hi && n0 + 4 > args.gate_lo)
                    apply_gates_copy<4>(o4, n0, args.N, args.nseg, seg_tab);
                return make_uint2(pack_bf16x2(o4[0], o4[1]), pack_bf16x2(o4[2], o4[3]));
            };
            auto store_one = [&](int t, uint2 o) {
                uint16_t* yp = args.y + static_cast<int64_t>(t) * args.ldy + n0;
                if (full4) {
                    *reinterpret_cast<uint2*>(yp) = o;
                } else {
                    const uint16_t v[4] = {static_cast<uint16_t>(o.x & 0xFFFFu), static_cast<uint16_t>(o.x >> 16),
                                           static_cast<uint16_t>(o.y & 0xFFFFu), static_cast<uint16_t>(o.y >> 16)};
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (n0 + u < args.N) yp[u] = v[u];
                }
            };
            uint2 held[kDecHeld];
#pragma unroll
            for (int h = 0; h < kDecHeld; ++h)
                if (h < niter) held[h] = reduce_one(t_first + h * tstep);
            // more outputs than registers hold (one-CTA clusters with wide token
            // counts): those are stored before the release
            for (int h = kDecHeld; h < niter; ++h) store_one(t_first + h * tstep, reduce_one(t_first + h * tstep));
            __syncwarp();
            // this warp is done reading buffer pb: tell every CTA of the cluster.
            // Relaxed: every partial read above was consumed before this point
            // (in-order issue), and a release would wait for the global stores
            // of the previous tile.
            if (lane < S)
                mbar_arrive_cluster_relaxed(
                    mapa_shared(smem_u32(&part_free[pb]), static_cast<uint32_t>(lane)));
#pragma unroll
            for (int h = 0; h < kDecHeld; ++h)
                if (h < niter) store_one(t_first + h * tstep, held[h]);
        }
    }

    // no CTA leaves while a peer may still write into its shared memory or
    // arrive on its barriers
    tc_fence_before();
    __syncwarp();
    if (warp < 6) cluster_wait();           // the roles that did not wait above
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kDecTmemCols);
}
