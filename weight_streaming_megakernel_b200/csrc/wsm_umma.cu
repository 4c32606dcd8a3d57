// wsm_umma.cu -- weight-streaming decode GEMM on the 5th-generation tensor
// cores (tcgen05 MMA, accumulators in tensor memory), persistent, one CTA per
// SM.  Handles one GEMM (skinny_gemm) or a chain of GEMMs with readiness
// counters (gemm_chain) in the same code.
//
// The product is computed transposed ("swap AB", as the GC-MoE operator does
// on Blackwell: the weight is the 128-row MMA operand):
//     D[128 x n] = W_tile[128 x 64] . X_tile[n x 64]^T,   n = MMA N = X rows (16..64)
// so the wide weight fills the MMA's M = 128 rows and the few X rows its N
// columns.  D lives in tensor memory (TMEM), fp32.
//
// Warp roles (192 threads):
//   warp 0     TMA producer: W tile and X tile of each stage into a ring of
//              shared-memory stages (128-byte swizzle, mbarrier completion).
//              W is read from HBM exactly once per call and its L2 policy is
//              evict-first unless several M-tiles share it; X is evict-last.
//              In a chain it issues a task's W loads before the task's
//              dependency is met and only holds back the X loads.
//   warp 1     TMEM allocation + the single MMA-issuing thread.
//   warps 2-5  epilogue: tcgen05.ld of the accumulator, bf16 rounding, stores,
//              split-K partials and the in-order reduction (see wsm_internal.cuh).
//
// Fleet's per-XCD scheduler workgroup ("Fleet ..." reading notes, section 2)
// has no counterpart: the static stream-K split needs no dispatcher, and the
// dependency wait sits in the producer warp of every CTA.
#include "wsm_internal.cuh"

namespace wsm {

namespace {

// --- tcgen05 wrappers ------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[smem desc] . B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z)
        : "memory");
}

// 32 lanes x 16 consecutive fp32 columns -> 16 registers per thread.  The
// registers are written asynchronously: nothing may read them before
// tmem_ld_wait16() on the same array.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Wait for this thread's outstanding tcgen05.ld; the array is a read-write
// operand so the compiler cannot touch it before the wait has executed.
__device__ __forceinline__ void tmem_ld_wait16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), Blackwell
// descriptor version 1.  Start address in 16-byte units.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);        // [0,14)  start address
    d |= (uint64_t)1 << 16;                           // [16,30) leading byte offset (unused with swizzle) = 16 B
    d |= (uint64_t)(1024u >> 4) << 32;                // [32,46) stride byte offset = 1024 B
    d |= (uint64_t)1 << 46;                           // [46,48) version = 1
    d |= (uint64_t)2 << 61;                           // [61,64) layout = SWIZZLE_128B
    return d;
}

constexpr int kThreads = 192;
constexpr int kEpiWarp0 = 2;
constexpr int kEpiThreads = 128;
constexpr int kEpiBar = 1;          // named barrier id of the epilogue warps
constexpr uint32_t kTmemCols = 2 * kUmmaMaxN;   // two accumulator buffers

__device__ __forceinline__ void epi_bar() { named_bar_sync(kEpiBar, kEpiThreads); }

__device__ __forceinline__ const TaskDev &task_at(const KParams &p, int t) {
    return p.tasks ? p.tasks[t] : p.single;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) wsm_umma_kernel(const __grid_constant__ KParams p) {
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[2];
    __shared__ __align__(8) uint64_t acce_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_flag;
    __shared__ int last_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int c = blockIdx.x;
    const int S = p.stages;
    // 1024-byte aligned ring (required by the 128-byte swizzle pattern)
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf_bar[b], 1);
            mbar_init(&acce_bar[b], kEpiThreads / 32);
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base_sh, kTmemCols);
    if (threadIdx.x == 0) pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const unsigned long long wlim = p.wait_timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_x = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            long long issued = 0;
            bool aborted = false;
            bool grid_dep_ok = p.pdl != 2;  // mode 2 streams W before the previous kernel completes
            if (p.pdl == 1) pdl_wait();
            for (int t = 0; t < p.n_tasks && !aborted; ++t) {
                const TaskDev &T = task_at(p, t);
                const long long Tt = (long long)T.n_g * T.n_mt * T.kb;
                const long long lo = range_lo(Tt, c, G), hi = range_lo(Tt, c + 1, G);
                if (lo >= hi) continue;
                prefetch_tmap(&T.tmW);
                prefetch_tmap(&T.tmX);
                const uint64_t pol_w = T.w_evict_first ? policy_evict_first() : policy_evict_normal();
                bool dep_ok = T.dep < 0 && grid_dep_ok;
                int pend_s[kMaxStages], pend_k[kMaxStages], pend_y[kMaxStages];
                int np = 0;
                if (p.trace) {
                    p.trace[((size_t)c * p.n_tasks + t) * 4 + 0] = globaltimer();
                    uint32_t smid;
                    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
                    p.trace[((size_t)c * p.n_tasks + t) * 4 + 3] = smid;
                }
                auto flush = [&]() {
                    if (!grid_dep_ok) {
                        pdl_wait();
                        grid_dep_ok = true;
                    }
                    if (T.dep >= 0) wait_dependency(p, task_at(p, T.dep), t, p.status);
                    if (p.trace) p.trace[((size_t)c * p.n_tasks + t) * 4 + 1] = globaltimer();
                    for (int i = 0; i < np; ++i)
                        for (int j = 0; j < p.kps; ++j)
                            tma_load_2d(ring + (size_t)pend_s[i] * p.stage_bytes + p.x_off + j * p.x_stride, &T.tmX,
                                        &full_bar[pend_s[i]], pend_k[i] + j * kUmmaBK, pend_y[i], pol_x);
                    np = 0;
                    dep_ok = true;
                };
                IterWalk w;
                w.start(T, lo);
                for (long long it = lo; it < hi; ++it, w.next(T)) {
                    const int kk = w.kk, g = w.g, mt = w.mt;
                    // W loads may run ahead of the dependency until the ring is full
                    if (np > 0 && !mbar_test(&empty_bar[s], ph ^ 1)) flush();
                    if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1, &abort_flag, wlim, p.status, t, kSiteEmpty)) {
                        if (np > 0) flush();  // every issued stage must be able to complete
                        aborted = true;
                        break;
                    }
                    uint8_t *st = ring + (size_t)s * p.stage_bytes;
                    mbar_arrive_expect_tx(&full_bar[s], T.tx_bytes);
                    const int k0 = kk * p.kps * kUmmaBK;
                    for (int j = 0; j < p.kps; ++j)
                        tma_load_2d(st + j * (kUmmaRows * kUmmaBK * 2), &T.tmW, &full_bar[s], k0 + j * kUmmaBK,
                                    g * kUmmaRows, pol_w);
                    const int xy = mt * T.t_m;
                    if (dep_ok) {
                        for (int j = 0; j < p.kps; ++j)
                            tma_load_2d(st + p.x_off + j * p.x_stride, &T.tmX, &full_bar[s], k0 + j * kUmmaBK, xy,
                                        pol_x);
                    } else {
                        pend_s[np] = s;
                        pend_k[np] = k0;
                        pend_y[np] = xy;
                        ++np;
                    }
                    ++issued;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (np > 0) flush();
                if (p.trace && T.dep < 0) p.trace[((size_t)c * p.n_tasks + t) * 4 + 1] = globaltimer();
            }
            if (!grid_dep_ok) pdl_wait();  // a CTA with no work still orders itself after the previous kernel
            // Drain: every stage this thread issued must have landed before the
            // CTA may exit (bounded; in a healthy run these already completed).
            // copies in flight must land before exit, abort or not
            drain_issued(full_bar, S, issued, wlim, p.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t seg = 0;
            bool aborted = false;
            bool any_mma = false;
            for (int t = 0; t < p.n_tasks && !aborted; ++t) {
                const TaskDev &T = task_at(p, t);
                const long long Tt = (long long)T.n_g * T.n_mt * T.kb;
                const long long lo = range_lo(Tt, c, G), hi = range_lo(Tt, c + 1, G);
                const uint32_t idesc = T.idesc;
                long long it = lo;
                int tile = (int)(lo / T.kb);
                for (; it < hi && !aborted; ++tile) {
                    const long long seg_start = it;
                    const long long seg_end = ((long long)tile + 1) * T.kb < hi ? ((long long)tile + 1) * T.kb : hi;
                    const int buf = seg & 1;
                    const uint32_t aph = (seg >> 1) & 1;
                    if (!mbar_wait_bounded(&acce_bar[buf], aph ^ 1, &abort_flag, wlim, p.status, t, kSiteAcc)) {
                        aborted = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(buf * kUmmaMaxN);
                    for (; it < seg_end; ++it) {
                        if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, wlim, p.status, t, kSiteFull)) {
                            aborted = true;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t st0 = smem_u32(ring + (size_t)s * p.stage_bytes);
                        const bool first_stage = (it == seg_start);
                        for (int j = 0; j < p.kps; ++j) {
                            const uint32_t a0 = st0 + (uint32_t)(j * kUmmaRows * kUmmaBK * 2);
                            const uint32_t b0 = st0 + (uint32_t)(p.x_off + j * p.x_stride);
#pragma unroll
                            for (int k = 0; k < kUmmaBK / 16; ++k) {
                                // advancing K by 16 bf16 = 32 bytes inside the swizzle atom
                                tc_mma(d_tmem, sw128_desc(a0 + 32u * k), sw128_desc(b0 + 32u * k), idesc,
                                       (first_stage && j == 0 && k == 0) ? 0u : 1u);
                            }
                        }
                        any_mma = true;
                        tc_commit(&empty_bar[s]);  // frees the stage once these MMAs have read it
                        if (++s == S) {
                            s = 0;
                            ph ^= 1;
                        }
                    }
                    if (aborted) break;
                    tc_commit(&accf_bar[buf]);     // accumulator ready for the epilogue
                    ++seg;
                }
            }
            if (any_mma) {
                // all MMAs of this CTA complete before TMEM can be released
                tc_commit(&drain_bar);
                volatile int never = 0;
                mbar_wait_bounded(&drain_bar, 0, &never, wlim, p.status, -1, kSiteDrain);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quadrant this warp may access
        const int row = q * 32 + lane;          // row of the 128-row tile = TMEM lane
        const int etid = threadIdx.x - kEpiWarp0 * 32;
        const bool leader = (etid == 0);
        if (p.pdl) pdl_wait();                  // Y and the scratch may still be in use by the previous kernel
        uint32_t seg = 0;
        bool aborted = false;
        for (int t = 0; t < p.n_tasks; ++t) {
            const TaskDev &T = task_at(p, t);
            const long long Tt = (long long)T.n_g * T.n_mt * T.kb;
            const long long lo = range_lo(Tt, c, G), hi = range_lo(Tt, c + 1, G);
            long long it = lo;
            bool wrote_any = false;
            for (int tile = (int)(lo / T.kb); it < hi; ++tile) {
                const long long tile_lo = (long long)tile * T.kb, tile_hi = tile_lo + T.kb;
                const long long seg_start = it;
                const long long seg_end = tile_hi < hi ? tile_hi : hi;
                it = seg_end;
                const int buf = seg & 1;
                const uint32_t aph = (seg >> 1) & 1;
                ++seg;
                float acc[kUmmaMaxN];
#pragma unroll
                for (int i = 0; i < kUmmaMaxN; ++i) acc[i] = 0.f;
                if (!aborted) {
                    if (!mbar_wait_bounded(&accf_bar[buf], aph, &abort_flag, wlim, p.status, t, kSiteAcc))
                        aborted = true;
                }
                // warp-uniform abort decision (tcgen05.ld is warp-collective)
                aborted = __any_sync(0xffffffffu, aborted);
                if (!aborted) {
                    tc_fence_after();
                    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kUmmaMaxN);
                    uint32_t r[kUmmaMaxN / 16][16];
#pragma unroll
                    for (int c16 = 0; c16 < kUmmaMaxN / 16; ++c16) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) r[c16][i] = 0u;
                        if (c16 * 16 < T.t_mpad) tmem_ld16(taddr + (uint32_t)(c16 * 16), r[c16]);
                    }
#pragma unroll
                    for (int c16 = 0; c16 < kUmmaMaxN / 16; ++c16) tmem_ld_wait16(r[c16]);
#pragma unroll
                    for (int c16 = 0; c16 < kUmmaMaxN / 16; ++c16)
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc[c16 * 16 + i] = __uint_as_float(r[c16][i]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && !aborted) mbar_arrive(&acce_bar[buf]);

                int g, mt;
                tile_coords(T, tile, g, mt);
                const int n = g * kUmmaRows + row;
                const int m0 = mt * T.t_m;
                const int mrows = min(T.t_m, T.M - m0);
                const bool full_tile = (seg_start == tile_lo) && (seg_end == tile_hi);
                if (full_tile) {
                    if (!aborted && n < T.N) {
#pragma unroll
                        for (int m = 0; m < kUmmaMaxN; ++m) {
                            if (m < mrows) {
                                const size_t o = (size_t)(m0 + m) * T.N + n;
                                T.Y[o] = __float2bfloat16_rn(acc[m]);
                                if (T.Yf32) T.Yf32[o] = acc[m];
                            }
                        }
                    }
                    if (T.notify) {
                        epi_bar();
                        if (leader && !aborted) red_release_gpu_add(T.done, 1u);  // release covers the CTA's stores (bar.sync before)
                    }
                } else {
                    // split tile: write this CTA's partial, then the last arriver reduces
                    int c_first, c_last;
                    const int n_c = tile_contributors(tile_lo, tile_hi, Tt, G, c_first, c_last);
                    const int my_slot = partial_slot(c, seg_start, lo);
                    float *pslot = T.part + (size_t)my_slot * T.slot_elems;
                    if (!aborted) {
#pragma unroll
                        for (int m = 0; m < kUmmaMaxN; ++m)
                            if (m < mrows) pslot[m * kUmmaRows + row] = acc[m];
                    }
                    epi_bar();
                    if (leader) {
                        int last = 0;
                        if (!aborted) {
                            // acq_rel: releases the partials this CTA stored before the barrier, and
                            // acquires the others' partials for the last arriver
                            const unsigned int old = atom_add_acqrel_gpu(&T.tile_cnt[tile], 1u);
                            last = (old == (unsigned int)(n_c - 1)) ? 1 : 0;
                        }
                        last_flag = last;
                    }
                    epi_bar();
                    if (last_flag) {
                        // the leader's acquire + the barrier order these loads after every partial
                        const int first_slot = (range_lo(Tt, c_first, G) < tile_lo) ? 2 * c_first + 1 : 2 * c_first;
                        for (int mb = 0; mb < mrows; mb += 8) {
                            float sum[8];
                            ordered_partial_sums<8, 4>(T.part, T.slot_elems, kUmmaRows, row, mb, mrows, c_first,
                                                       c_last, first_slot, Tt, G, sum);
                            if (n < T.N) {
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    if (mb + i < mrows) {
                                        const size_t o = (size_t)(m0 + mb + i) * T.N + n;
                                        T.Y[o] = __float2bfloat16_rn(sum[i]);
                                        if (T.Yf32) T.Yf32[o] = sum[i];
                                    }
                                }
                            }
                        }
                        epi_bar();
                        if (leader) {
                            T.tile_cnt[tile] = 0u;  // ready for the next call
                            if (T.notify) red_release_gpu_add(T.done, 1u);
                        }
                    }
                }
                wrote_any = true;
            }
            if (p.trace && wrote_any && leader) p.trace[((size_t)c * p.n_tasks + t) * 4 + 2] = globaltimer();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace wsm
