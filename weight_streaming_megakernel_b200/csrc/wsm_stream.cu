// wsm_stream.cu -- weight-streaming decode GEMM for M <= 8 on the fp32 FMA
// pipes: the weight stream lands in shared memory through TMA and each output
// is a dot product finished by a warp-shuffle reduction.  Persistent, one CTA
// per SM; same work units, partials and chain readiness as the tcgen05 path
// (wsm_internal.cuh).
//
// The three techniques of the FlyDSL article ("AMD: ROCm Low-Latency-GEMM-
// Kernel ... MI355X"), as they land on B200:
//   1. inter-CTA split-K      -> work units of a tile's K range, claimed by
//                                any CTA, reduced in unit order;
//   2. intra-CTA K-slicing    -> KW consumer warps own disjoint 256-wide K
//                                slices of every stage, lanes own 8-wide
//                                pieces; slices are summed once per unit;
//   3. multi-stage LDS pipe   -> a ring of TMA stages with mbarriers, filled
//                                by one producer warp while 8 warps compute.
//
// Stage layout (one pipeline stage = T_N rows of W x T_K columns, plus the
// matching X slice): KW boxes of W [T_N][256] then KW boxes of X [MMAX][256],
// bf16, 512-byte rows.  A lane reads 16 bytes per row, so each LDS.128 of a
// warp covers 512 contiguous bytes (no bank conflicts).
//
// Consumer warp (kw, rg): K slice kw, rows rg*RW .. rg*RW+RW-1.  Per stage a
// lane converts its 8 X values of every row m once and reuses them for RW
// rows of W: RW*8*MMAX FMAs per RW+MMAX shared loads.
#include "wsm_internal.cuh"

namespace wsm {

namespace {

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&f)[8]) {
    // a bf16 value is the upper half of a binary32 value
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xFFFF0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xFFFF0000u);
    f[4] = __uint_as_float(u.z << 16);
    f[5] = __uint_as_float(u.z & 0xFFFF0000u);
    f[6] = __uint_as_float(u.w << 16);
    f[7] = __uint_as_float(u.w & 0xFFFF0000u);
}

constexpr int kConsBar = 1;

// Epilogue of one output (row n of W, X row m): plain, residual add, or
// SiLU*mul (the up value of gate row n comes from the thread owning row n + 8,
// lane ^ 8: every lane of the warp calls this), then one rounding to bf16.
__device__ __forceinline__ void emit_one(const EpiOut &e, int n, int m, bool live, float y) {
    size_t o;
    if (e.epi == kEpiSiluMul) {
        const float up = __shfl_xor_sync(0xffffffffu, y, 8);
        if (!live || (n & 8)) return;
        y = y / (1.f + expf(-y)) * up;
        o = (size_t)m * e.y_cols + ((n >> 4) << 3) + (n & 7);
    } else {
        if (!live) return;
        o = (size_t)m * e.N + n;
        if (e.epi == kEpiResidual) y += __bfloat162float(e.R[o]);
    }
    e.Y[o] = __float2bfloat16_rn(y);
    if (e.Yf32) e.Yf32[o] = y;
}

// Barrier among the consumer warps that also ORs a predicate over them.
__device__ __forceinline__ bool vote_or(bool v, int id, int n) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pc, pr;\n\t"
        "setp.ne.u32 pc, %1, 0;\n\t"
        "bar.red.or.pred pr, %2, %3, pc;\n\t"
        "selp.u32 %0, 1, 0, pr;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Transposed butterfly reduction over the 32 lanes of V values per lane.
// While more than one value is left, each step hands half of them to the
// partner lane (the half the partner keeps) and adds the half it receives, so
// the whole reduction costs about V shuffles instead of 5V.  On return each
// lane holds `V >> h` sums (h = min(5, log2 V) halving steps) starting at
// index base(lane); when V < 32 the lanes with equal halving bits hold equal
// copies.
template <int V>
struct LaneReduce {
    static constexpr int H = (V >= 32) ? 5 : (V >= 16 ? 4 : (V >= 8 ? 3 : (V >= 4 ? 2 : (V >= 2 ? 1 : 0))));
    static constexpr int OUT = V >> H;

    __device__ __forceinline__ static int run(float (&v)[V], int lane) {
        int base = 0;
        int cnt = V;
#pragma unroll
        for (int step = 0; step < 5; ++step) {
            const int o = 16 >> step;
            if (step < H) {
                const int half = cnt >> 1;
                const bool upper = (lane & o) != 0;
#pragma unroll
                for (int i = 0; i < V / 2; ++i) {
                    if (i < half) {
                        const float send = upper ? v[i] : v[i + half];
                        const float keep = upper ? v[i + half] : v[i];
                        const float recv = __shfl_xor_sync(0xffffffffu, send, o);
                        v[i] = keep + recv;
                    }
                }
                if (upper) base += half;
                cnt = half;
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
            }
        }
        return base;
    }
};

}  // namespace

// L2 prefetch of the W of the units this CTA would own in a round-robin (c,
// c + G, ...), p.prefetch_stages stages at most, in each unit's stream order,
// skipping the first `skip` stages of each first-round unit (its claimer's
// ring already holds them).  Out of line: it runs at most once per task.
static __device__ __noinline__ void prefetch_w_l2(const KParams &p, const TaskDev &T, int skip, int KW, int TN) {
    int budget = p.prefetch_stages;
    for (int uu = blockIdx.x; uu < T.n_units && budget > 0; uu += gridDim.x) {
        const UnitSpan ps = unit_span(T, uu);
        const int k_len = ps.k_end - ps.k_begin;
        const int k_rot = unit_k_rot(p, T, ps);
        for (int i = (uu < (int)gridDim.x ? skip : 0); i < k_len && budget > 0; ++i, --budget) {
            const int kk = ps.k_begin + (i + k_rot) % k_len;
            for (int kw = 0; kw < KW; ++kw)
                tma_prefetch_l2_2d(&T.tmW, kk * (KW * kStreamBoxK) + kw * kStreamBoxK, ps.tile * TN);
        }
    }
}

// MMAX: largest M handled (register arrays); RW rows per warp; RG row groups;
// KW K-slices.  Consumer warps = RG*KW = 8; T_N = RG*RW; T_K = KW*256.
template <int MMAX, int RW, int RG, int KW>
__global__ void __launch_bounds__(32 * (1 + RG * KW), 1) wsm_stream_kernel(const __grid_constant__ KParams p) {
    constexpr int NCW = RG * KW;
    constexpr int NCT = NCW * 32;
    constexpr int TN = RG * RW;
    constexpr int V = RW * MMAX;
    using LR = LaneReduce<V>;
    static_assert(NCW == 8, "eight consumer warps");

    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ int stage_meta[kMaxStages][3];   // {task, unit, flags}, written by the producer
    __shared__ float red[2][RG][KW][V];
    __shared__ volatile int abort_flag;
    __shared__ int last_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = p.stages;
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NCW);
        }
        abort_flag = 0;
        fence_mbar_init();
        if (p.independent) pdl_launch_dependents();  // other calls trigger once past their grid wait (consumers)
    }
    __syncthreads();
    const unsigned long long wlim = p.wait_timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_x = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            long long issued = 0;
            bool aborted = false;
            bool slot_ok = false;  // the wait for ring slot s has already succeeded
            bool grid_dep_ok = p.pdl != 2 || p.independent;  // an independent call never waits here
            if (p.pdl == 1 && !p.independent) pdl_wait();
            if (p.debug_stall_ns && blockIdx.x == 0) {
                // test hook: after the previous kernel (whose exit clears the launch error flag), wait on a
                // flag nothing sets until the limit passes, then abandon all of this CTA's work
                if (!grid_dep_ok || p.independent) {
                    pdl_wait();
                    grid_dep_ok = true;
                }
                debug_stall(p, &abort_flag);
                aborted = abort_flag != 0;
            }
            for (int t = 0; t < p.n_tasks && !aborted; ++t) {
                const TaskDev &T = task_at(p, t);
                prefetch_tmap(&T.tmW);
                prefetch_tmap(&T.tmX);
                const uint64_t pol_w = T.w_evict_first ? policy_evict_first() : policy_evict_normal();
                const bool col_dep = T.dep >= 0 && T.dep_col_cnt != nullptr;
                // nothing of X before the dependency is met (per column: the first chunks; after that the
                // chunk mask decides stage by stage)
                bool dep_ok = T.dep < 0 && grid_dep_ok;
                int pend_s[kMaxStages], pend_k[kMaxStages];
                int np = 0;
                // Per-column dependency: each stage's X waits only for the kColChunk-column chunks it
                // reads (seen-complete chunks are cached in chunk_mask).
                unsigned long long chunk_mask = 0;
                unsigned int run_no = 0;
                auto stage_chunks = [&](int k0, int &c0, int &c1) {
                    c0 = k0 / kColChunk;
                    c1 = (min(k0 + KW * kStreamBoxK, T.K) - 1) / kColChunk;
                };
                auto x_now = [&](int k0) -> bool {  // may this stage's X load go out now?
                    if (!dep_ok) return false;
                    if (!col_dep) return true;
                    int c0, c1;
                    stage_chunks(k0, c0, c1);
                    for (int c = c0; c <= c1; ++c)
                        if (c >= 64 || !((chunk_mask >> c) & 1ull)) return false;
                    return true;
                };
                // While this CTA waits (for the previous kernel or a dependency) HBM would idle: prefetch
                // into L2 the W of the units it would own in a round-robin (c, c + G, ...), except the
                // first ring-full of each first-round unit (some CTA's ring already holds it).
                bool prefetched = p.prefetch_stages <= 0;
                auto prefetch_l2 = [&]() {
                    if (prefetched) return;
                    prefetched = true;
                    prefetch_w_l2(p, T, (T.dep >= 0 && p.dep_ring_stages > 0) ? min(S, p.dep_ring_stages) : S, KW, TN);
                };
                auto flush = [&]() {
                    if (!grid_dep_ok) {
                        prefetch_l2();
                        pdl_wait();
                        grid_dep_ok = true;
                    }
                    if (T.dep >= 0 && !col_dep) {
                        if (!prefetched && !dependency_met(p, task_at(p, T.dep))) prefetch_l2();
                        wait_dependency(p, task_at(p, T.dep), t, p.status);
                    }
                    if (col_dep && run_no == 0) run_no = ld_acquire_gpu(&p.run_ctl[0]) + 1u;
                    if (!dep_ok) trace_stamp(p, t, 1, globaltimer());
                    for (int i = 0; i < np; ++i) {
                        if (col_dep) {
                            int c0, c1;
                            stage_chunks(pend_k[i], c0, c1);
                            wait_chunks(p, T, c0, c1, run_no, chunk_mask, t, p.status);
                        }
                        uint8_t *xs = ring + (size_t)pend_s[i] * p.stage_bytes + p.x_off;
#pragma unroll
                        for (int kw = 0; kw < KW; ++kw)
                            tma_load_2d(xs + kw * MMAX * 512, &T.tmX, &full_bar[pend_s[i]],
                                        pend_k[i] + kw * kStreamBoxK, 0, pol_x);
                    }
                    np = 0;
                    dep_ok = true;
                };
                // Wait for ring slot s.  W loads may run ahead of the dependency until the ring is full;
                // then the pending X loads go out first (every issued stage must be able to complete).
                auto take_slot = [&]() -> bool {
                    if (slot_ok) return true;
                    // a dependent task streams at most dep_ring_stages stages of W ahead of its dependency:
                    // more only queues in front of the round trips that end the previous task
                    if (np > 0 && T.dep >= 0 && p.dep_ring_stages > 0 && np >= p.dep_ring_stages) flush();
                    if (np > 0 && !mbar_test(&empty_bar[s], ph ^ 1)) flush();
                    if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1, &abort_flag, wlim, p.status, t, kSiteEmpty)) {
                        if (np > 0) flush();
                        aborted = true;
                        return false;
                    }
                    slot_ok = true;
                    return true;
                };
                bool first_unit = true;
                // The kernel's first task hands unit c to CTA c (no atomic, and it can stream before the
                // grid dependency); later tasks hand out every unit by claim, so the CTAs that finish the
                // previous task first take the next task's work.
                // (with two-level readiness a CTA works only on its group's tiles, all claimed)
                const ClaimRange cr = claim_range(T);
                const bool static_first = t == 0 && T.n_groups <= 1;
                const int n_static = static_first ? min((int)gridDim.x, T.n_units) : 0;
                int u;
                if (static_first) {
                    u = (int)blockIdx.x < T.n_units ? (int)blockIdx.x : T.n_units;
                } else {
                    if (!grid_dep_ok) {
                        pdl_wait();
                        grid_dep_ok = true;
                        dep_ok = T.dep < 0;
                    }
                    u = cr.lo + claim_unit(cr);
                }
                while (u < cr.hi) {
                    if (first_unit) {
                        trace_stamp(p, t, 0, globaltimer());
                        trace_stamp(p, t, 3, smid());
                        first_unit = false;
                    }
                    const UnitSpan us = unit_span(T, u);
                    const int g = us.tile;
                    const int k_begin = us.k_begin;
                    const int k_end = us.k_end;
                    const int k_len = k_end - k_begin;
                    const int k_rot = unit_k_rot(p, T, us);
                    int next_u = cr.hi - cr.lo - n_static;
                    bool claimed = false;
                    for (int kk = k_begin; kk < k_end; ++kk) {
                        if (!take_slot()) break;
                        slot_ok = false;
                        uint8_t *st = ring + (size_t)s * p.stage_bytes;
                        stage_meta[s][0] = t;
                        stage_meta[s][1] = u;
                        stage_meta[s][2] = (kk == k_begin ? kMetaFirst : 0) | (kk == k_end - 1 ? kMetaLast : 0);
                        mbar_arrive_expect_tx(&full_bar[s], T.tx_bytes);
                        // the stage this iteration loads (rotated within the unit when k_rotate)
                        const int kr = k_rot ? k_begin + (kk - k_begin + k_rot) % k_len : kk;
                        const int k0 = kr * (KW * kStreamBoxK);
#pragma unroll
                        for (int kw = 0; kw < KW; ++kw)
                            tma_load_2d(st + kw * TN * 512, &T.tmW, &full_bar[s], k0 + kw * kStreamBoxK, g * TN,
                                        pol_w);
                        if (x_now(k0)) {
#pragma unroll
                            for (int kw = 0; kw < KW; ++kw)
                                tma_load_2d(st + p.x_off + kw * MMAX * 512, &T.tmX, &full_bar[s],
                                            k0 + kw * kStreamBoxK, 0, pol_x);
                        } else {
                            pend_s[np] = s;
                            pend_k[np] = k0;
                            ++np;
                        }
                        ++issued;
                        if (++s == S) {
                            s = 0;
                            ph ^= 1;
                        }
                        // claim the next unit kClaimLead stages before this one ends: early enough to
                        // hide the claim's round trip, late enough not to hold work a faster CTA could
                        // take -- and never while this task's dependency is unmet, when every CTA would
                        // hold a second unit it cannot start (the claim counters belong to the previous
                        // kernel until the grid dependency is resolved)
                        if (!claimed && !p.independent && dep_ok && k_end - kk <= kClaimLead) {
                            next_u = claim_unit(cr);
                            claimed = true;
                        }
                    }
                    if (aborted) break;
                    if (!claimed && !p.independent) {
                        // the unit streamed completely before its dependencies were resolved
                        if (!dep_ok) flush();
                        next_u = claim_unit(cr);
                    }
                    // whatever comes next needs a free slot: wait for it before the claim's result is used,
                    // so the claim's round trip overlaps the wait
                    if (!take_slot()) break;
                    u = p.independent ? u + (int)gridDim.x : cr.lo + next_u + n_static;
                }
                if (np > 0) flush();
                if (aborted) break;
                if (T.dep < 0 && !first_unit) trace_stamp(p, t, 1, globaltimer());
            }
            if (!p.run_ctl && !p.independent) {
                // every CTA counts the end of its claims, aborted or not (after the grid dependency: until
                // then the claim counters belong to the previous kernel)
                if (!grid_dep_ok) {
                    pdl_wait();
                    grid_dep_ok = true;
                }
                claims_finished(p.single, gridDim.x);
            }
            if (!grid_dep_ok) pdl_wait();
            // copies in flight must land before exit (checked before the end marker below advances one of
            // these barriers again)
            drain_issued(full_bar, S, issued, wlim, p.status);
            // end-of-work marker for the consumers (a stage with no data)
            if (!aborted && (slot_ok || mbar_wait_bounded(&empty_bar[s], ph ^ 1, &abort_flag, wlim, p.status, -1,
                                                          kSiteEmpty))) {
                stage_meta[s][0] = 0;
                stage_meta[s][1] = 0;
                stage_meta[s][2] = kMetaDone;
                mbar_arrive(&full_bar[s]);
            }
        }
    } else {
        // ------------------------------------------------------------ consumers
        const int cw = warp - 1;
        const int kw = cw % KW;
        const int rg = cw / KW;
        const int ctid = threadIdx.x - 32;
        const bool leader = (ctid == 0);
        // thread ctid < TN*MMAX owns output (row, m) of a tile
        const int o_m = ctid / TN;
        const int o_row = ctid - o_m * TN;
        const bool owner = ctid < TN * MMAX;
        if (p.pdl && !p.independent) {
            pdl_wait();  // Y and the scratch may still be in use by the previous kernel
            // the next kernel may launch once every CTA has seen this one's predecessor complete: so at most
            // this kernel and the independent calls queued after it can still run when one of those starts
            if (leader) pdl_launch_dependents();
        }
        if (!p.run_ctl && !p.independent && cw == 0) {
            // a single call: the tile counters a failed call before it left mid-count are repaired first
            if (blockIdx.x == 0) repair_after_failure(p, lane);
            else if (leader) wait_repaired(p);
        }
        const unsigned int run_no = p.run_ctl ? ld_acquire_gpu(&p.run_ctl[0]) + 1u : 0u;  // this chain run
        int s = 0;
        uint32_t ph = 0;
        uint32_t unit_i = 0;
        // Accumulators.  At MMAX = 2 and 4 each (row, m) output keeps two partial sums, of the even and
        // the odd K positions of every 8, updated by Blackwell's packed fp32 FMA (two FMAs per
        // instruction, each rounded as fmaf): measured 5-10 % faster there.  MMAX = 1 gains nothing (it
        // is bound by the stream, not the FMA pipe) and at MMAX = 8 the doubled accumulators would not
        // fit: scalar FMAs.
        constexpr bool kPaired = MMAX == 2 || MMAX == 4;
        float acc[RW][MMAX];
        float2 acc2[kPaired ? RW : 1][kPaired ? MMAX : 1];
        for (;;) {
            bool ab = !mbar_wait_bounded(&full_bar[s], ph, &abort_flag, wlim, p.status, -1, kSiteFull);
            ab = __any_sync(0xffffffffu, ab);
            const int flags = ab ? kMetaDone : stage_meta[s][2];
            if (ab || (flags & kMetaDone)) {
                // every consumer warp leaves at the same point (end marker, or an abort anywhere)
                vote_or(ab, kConsBar, NCT);
                break;
            }
            const int t = stage_meta[s][0];
            const int u = stage_meta[s][1];
            const TaskDev &T = task_at(p, t);
            const int M = T.M;
            if (flags & kMetaFirst) {
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int m = 0; m < MMAX; ++m) {
                        if constexpr (kPaired) acc2[r][m] = make_float2(0.f, 0.f);
                        else acc[r][m] = 0.f;
                    }
            }
            {
                const uint8_t *st = ring + (size_t)s * p.stage_bytes;
                const uint8_t *xs = st + p.x_off + kw * MMAX * 512 + lane * 16;
                const uint8_t *ws = st + kw * TN * 512 + (rg * RW) * 512 + lane * 16;
                float xv[MMAX][8];
#pragma unroll
                for (int m = 0; m < MMAX; ++m) {
                    if (m < M) {
                        const uint4 q = *reinterpret_cast<const uint4 *>(xs + m * 512);
                        bf16x8_to_f32(q, xv[m]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) xv[m][j] = 0.f;
                    }
                }
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    const uint4 q = *reinterpret_cast<const uint4 *>(ws + r * 512);
                    float wf[8];
                    bf16x8_to_f32(q, wf);
#pragma unroll
                    for (int m = 0; m < MMAX; ++m) {
                        if constexpr (kPaired) {
#pragma unroll
                            for (int j = 0; j < 8; j += 2)
                                acc2[r][m] = __ffma2_rn(make_float2(wf[j], wf[j + 1]),
                                                        make_float2(xv[m][j], xv[m][j + 1]), acc2[r][m]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j) acc[r][m] = fmaf(wf[j], xv[m][j], acc[r][m]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[s]);
            if (++s == S) {
                s = 0;
                ph ^= 1;
            }
            if (!(flags & kMetaLast)) continue;

            // ---- end of unit: lanes -> warps -> tile outputs
            float v[V];
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int m = 0; m < MMAX; ++m) {
                    if constexpr (kPaired) v[r * MMAX + m] = acc2[r][m].x + acc2[r][m].y;
                    else v[r * MMAX + m] = acc[r][m];
                }
            const int base = LR::run(v, lane);
            const int rb = unit_i & 1;
            ++unit_i;
            constexpr int lane_mask = (V >= 32) ? 0 : (31 >> LR::H);
            if ((lane & lane_mask) == 0) {
#pragma unroll
                for (int i = 0; i < LR::OUT; ++i) red[rb][rg][kw][base + i] = v[i];
            }
            if (vote_or(false, kConsBar, NCT)) break;  // an abort elsewhere: stop with the others
            float val = 0.f;
            if (owner) {
                const int org = o_row / RW, orr = o_row - org * RW;
#pragma unroll
                for (int k = 0; k < KW; ++k) {
                    const float x = red[rb][org][k][orr * MMAX + o_m];
                    val = (k == 0) ? x : val + x;
                }
            }
            const UnitSpan us = unit_span(T, u);
            const int g = us.tile;
            const int n = g * TN + o_row;
            const bool live = owner && o_m < M && n < T.N;
            UnitOut uo = unit_out(T);  // no task-table reads after the first store below
            unit_out_group(uo, T, g);
            if (us.nu == 1) {
                emit_one(uo.e, n, o_m, live, val);
                if (uo.done || uo.col_cnt) {
                    named_bar_sync(kConsBar, NCT);
                    if (leader) tile_finished(uo, g, TN, run_no);  // release covers the CTA's stores (bar.sync before)
                }
            } else {
                if (owner) uo.part[(size_t)u * uo.slot_elems + ctid] = val;
                named_bar_sync(kConsBar, NCT);
                if (leader) {
                    // acq_rel: releases this CTA's partial (stored before the barrier) and acquires the
                    // others' for the last arriver
                    const unsigned int old = atom_add_acqrel_gpu(&uo.tile_cnt[g], 1u);
                    last_flag = (old == (unsigned int)(us.nu - 1)) ? 1 : 0;
                }
                named_bar_sync(kConsBar, NCT);
                if (last_flag) {
                    // the leader's acquire + the barrier order these loads after every partial
                    float sum[1] = {0.f};
                    if (owner)
                        ordered_unit_sums<1, 8>(uo.part + (size_t)us.u0 * uo.slot_elems,
                                                us.slot_stride * uo.slot_elems, 0, ctid, 0, 1, us.nu, sum);
                    emit_one(uo.e, n, o_m, live, sum[0]);
                    named_bar_sync(kConsBar, NCT);
                    if (leader) {
                        uo.tile_cnt[g] = 0u;
                        tile_finished(uo, g, TN, run_no);
                    }
                }
            }
            if (leader) trace_stamp(p, t, 2, globaltimer());
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (p.run_ctl) chain_run_done(p);
        // an independent call completes only after the kernel before it (later kernels rely on stream
        // order): one CTA waits for it, the others leave their SMs to the calls beside this one
        else if (p.independent && blockIdx.x == 0 && p.pdl) pdl_wait();
    }
}

// Kernel for a register width and a tile height, 8 rows per warp either way:
// 16-row tiles are 2 row groups x 4 K-slices (T_K = 1024, W boxes of
// [16 x 256], 8 KB), 32-row tiles 4 row groups x 2 K-slices (T_K = 512, boxes
// of [32 x 256], 16 KB).  Measured on B200: one SM streams at most ~36 GB/s
// with the 8 KB boxes and ~50 GB/s with the 16 KB ones (the same 32 KB per
// stage); the wide stage of the 16-row tiles beats 4 x 4 x 2 (T_K = 512) at
// M = 1 and 2.  Must agree with stream_geo() in wsm_api.cu.
const void *stream_kernel_ptr(int mmax, int tile_rows) {
    if (tile_rows == 32) {
        switch (mmax) {
            case 1: return reinterpret_cast<const void *>(&wsm_stream_kernel<1, 8, 4, 2>);
            case 2: return reinterpret_cast<const void *>(&wsm_stream_kernel<2, 8, 4, 2>);
            case 4: return reinterpret_cast<const void *>(&wsm_stream_kernel<4, 8, 4, 2>);
            case 8: return reinterpret_cast<const void *>(&wsm_stream_kernel<8, 8, 4, 2>);
            default: return nullptr;
        }
    }
    switch (mmax) {
        case 1: return reinterpret_cast<const void *>(&wsm_stream_kernel<1, 8, 2, 4>);
        case 2: return reinterpret_cast<const void *>(&wsm_stream_kernel<2, 8, 2, 4>);
        case 4: return reinterpret_cast<const void *>(&wsm_stream_kernel<4, 8, 2, 4>);
        case 8: return reinterpret_cast<const void *>(&wsm_stream_kernel<8, 8, 2, 4>);
        default: return nullptr;
    }
}

}  // namespace wsm
