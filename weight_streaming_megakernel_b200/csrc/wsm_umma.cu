// wsm_umma.cu -- weight-streaming decode GEMM on the 5th-generation tensor
// cores (tcgen05 MMA, accumulators in tensor memory), persistent, one CTA per
// SM.  Handles one GEMM (skinny_gemm) or a chain of GEMMs with readiness
// counters (gemm_chain) in the same code.
//
// The product is computed transposed ("swap AB", as the GC-MoE operator does
// on Blackwell: the weight is the 128-row MMA operand):
//     D[128 x n] = W_tile[128 x 64k] . X_tile[n x 64k]^T,   n = MMA N = X rows (16..64)
// so the wide weight fills the MMA's M = 128 rows and the few X rows its N
// columns.  D lives in tensor memory (TMEM), fp32.
//
// Warp roles (320 threads):
//   warp 0     producer: claims work units (wsm_internal.cuh) and loads, per
//              stage, kps boxes of W [128 rows x 64 k] and of X with TMA into
//              a ring of shared-memory stages (128-byte swizzle, mbarrier
//              completion).  W is read from HBM once per call (L2 evict-first
//              unless several M-tiles share it); X is evict-last.  In a chain
//              it issues a task's W loads before the task's dependency is met
//              (at most dep_ring_stages of them) and holds back only the X
//              loads.
//   warp 1     TMEM allocation + the single MMA-issuing thread; four
//              accumulator buffers, so the MMA runs up to three units ahead
//              of the epilogue.
//   warps 2-9  epilogue, two sets of four warps that take alternate units:
//              tcgen05.ld of the accumulator, the fused epilogue (plain,
//              residual, SiLU*mul), bf16 rounding, stores, split-K partials
//              and the in-order reduction.
//
// Fleet's per-XCD scheduler workgroup ("Fleet ..." reading notes, section 2)
// has no counterpart: one atomic counter per task hands out the units, and the
// dependency wait sits in the producer of every CTA.
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

// Barrier among the epilogue warps that also ORs a predicate over them, so
// every decision to stop is taken by all four warps together.
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

constexpr int kEpiWarp0 = 2;
constexpr int kEpiSets = 2;         // two independent epilogue warp sets (units alternate between them)
constexpr int kEpiThreads = 128;    // per set: four warps, one per TMEM lane quadrant
constexpr int kThreads = 64 + kEpiSets * kEpiThreads;
constexpr int kAccBufs = 4;         // accumulators in TMEM: the MMA can run up to three units ahead
constexpr uint32_t kTmemCols = kAccBufs * kUmmaMaxN;   // 128-row tiles
constexpr uint32_t kTmemColsWide = 2 * kTmemCols;        // wide tiles: two accumulators per buffer (all of TMEM)

__device__ __forceinline__ void epi_bar(int set) { named_bar_sync(1 + set, kEpiThreads); }

// Epilogue of one thread's outputs: row n of W (output column n), X rows
// m0 .. m0 + cnt - 1, fp32 values v.  Plain, residual add, or SiLU*mul, then
// one rounding to bf16.  For SiLU*mul the up value of gate row n comes from
// the thread of row n + 8 (lane ^ 8): every lane of the warp calls this with
// the same cnt.  The epilogue kind is branched on once, outside the loops.
template <int MB>
__device__ __forceinline__ void emit_outputs(const EpiOut &e, int n, int m0, int cnt, const float (&v)[MB]) {
    if (e.epi == kEpiSiluMul) {
        const bool writer = !(n & 8) && n < e.N;
        const size_t col = ((size_t)(n >> 4) << 3) + (n & 7);
#pragma unroll
        for (int i = 0; i < MB; ++i) {
            if (i >= cnt) break;  // uniform across the warp
            const float up = __shfl_xor_sync(0xffffffffu, v[i], 8);
            if (writer) {
                const float y = v[i] / (1.f + expf(-v[i])) * up;
                const size_t o = (size_t)(m0 + i) * e.y_cols + col;
                e.Y[o] = __float2bfloat16_rn(y);
                if (e.Yf32) e.Yf32[o] = y;
            }
        }
        return;
    }
    if (n >= e.N) return;
    // residual: all of the thread's R loads go out before its first store (Y may alias R as far as
    // the compiler knows, so loads interleaved with the stores would each wait a round trip)
    float r[MB];
#pragma unroll
    for (int i = 0; i < MB; ++i)
        r[i] = (e.epi == kEpiResidual && i < cnt) ? __bfloat162float(e.R[(size_t)(m0 + i) * e.N + n]) : 0.f;
#pragma unroll
    for (int i = 0; i < MB; ++i) {
        if (i >= cnt) break;
        const size_t o = (size_t)(m0 + i) * e.N + n;
        const float y = e.epi == kEpiResidual ? v[i] + r[i] : v[i];
        e.Y[o] = __float2bfloat16_rn(y);
        if (e.Yf32) e.Yf32[o] = y;
    }
}

// The last unit of a split tile adds the tile's nu partials (slots u0 +
// j * stride, j = 0 .. nu - 1) for its row, in unit order (= K order), and
// writes the outputs.  Partial slots are [128 rows][t_mpad] floats, so a
// thread's values are contiguous: 16-byte loads, CB units x MB rows in flight.
template <int MB, int CB>
__device__ __forceinline__ void reduce_row_partials(const UnitOut &uo, const UnitSpan &us, int row, int mrows,
                                                    int m0, int n) {
    const int nu = us.nu;
    const size_t step = (size_t)us.slot_stride * uo.slot_elems;
    const float *base = uo.part + (size_t)us.u0 * uo.slot_elems + (size_t)row * uo.t_mpad;
    const EpiOut &e = uo.e;
    for (int mb = 0; mb < mrows; mb += MB) {
        float sum[MB];
#pragma unroll
        for (int i = 0; i < MB; ++i) sum[i] = 0.f;
        for (int jb = 0; jb < nu; jb += CB) {
            float4 v[CB][MB / 4];
#pragma unroll
            for (int u = 0; u < CB; ++u) {
                const float4 *q = reinterpret_cast<const float4 *>(base + (size_t)(jb + u) * step + mb);
#pragma unroll
                for (int i = 0; i < MB / 4; ++i)
                    v[u][i] = (jb + u < nu && mb + 4 * i < mrows) ? __ldcg(q + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < CB; ++u) {
                if (jb + u < nu) {
#pragma unroll
                    for (int i = 0; i < MB / 4; ++i) {
                        if (jb + u == 0) {
                            sum[4 * i] = v[u][i].x; sum[4 * i + 1] = v[u][i].y;
                            sum[4 * i + 2] = v[u][i].z; sum[4 * i + 3] = v[u][i].w;
                        } else {
                            sum[4 * i] += v[u][i].x; sum[4 * i + 1] += v[u][i].y;
                            sum[4 * i + 2] += v[u][i].z; sum[4 * i + 3] += v[u][i].w;
                        }
                    }
                }
            }
        }
        emit_outputs<MB>(e, n, m0 + mb, min(MB, mrows - mb), sum);
    }
}

// Exchange buffer (cluster mode): for each quadrant a CTA reduces, one slot per other unit of the tile,
// each slot 32 rows (one per lane) of p.xrow floats: the partial's t_mpad values, then a flag word.  The
// row stride is the chain's widest X tile + 4 floats (so 16-byte accesses of 8 consecutive lanes fall in
// distinct banks) and the flag sits at the same place in every task.
__device__ __forceinline__ void st_release_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.release.cluster.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_cluster_u32(const void *p) {
    uint32_t v;
    asm volatile("ld.acquire.cluster.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

// Bounded wait (per lane) until the flags of this lane's row in `nslots` slots reach `seq`.  Gives up when
// this CTA aborted, when another CTA recorded an error in this launch, or after `limit_ns` (recording a
// time-out).
static __device__ __noinline__ bool xchg_wait(const float *row0, int slot_floats, int nslots, int flag_at,
                                              uint32_t seq, volatile int *abort_flag, unsigned long long limit_ns,
                                              int *status, int task) {
    const unsigned long long t0 = globaltimer();
    for (int sl = 0; sl < nslots; ++sl) {
        const float *f = row0 + (size_t)sl * slot_floats + flag_at;
        for (uint32_t spin = 0;; ++spin) {
            if (ld_acquire_cluster_u32(f) - seq < 0x80000000u) break;  // flag >= seq
            if ((spin & 63u) == 63u) {
                if (*abort_flag || launch_failed(status)) return false;
                if (globaltimer() - t0 > limit_ns) {
                    record_error(status, kCodeTimeout, task, kSiteXchg);
                    *abort_flag = 1;
                    return false;
                }
            }
        }
    }
    return true;
}

// Epilogue of a split tile whose nu units (nu = 2 or 4) run on consecutive CTAs of one cluster: a
// reduce-scatter through distributed shared memory instead of partials in global memory.  The tile's 128
// rows are four 32-row quadrants (one per epilogue warp, TMEM lane quadrant q); quadrant q is reduced by
// the tile's CTA of index q % nu.  Every other CTA of the tile writes that quadrant's rows of its partial
// into the reducing CTA's exchange buffer, each lane its own row followed by a release store of the row's
// flag (the task's index + 1: every CTA takes part in at most one exchange per task, in task order).  The
// reducing lane acquires the flags of its own row only, adds the nu partials in unit order (= K order, the
// order of the global-memory reduction: the same bits), applies the epilogue and stores the outputs; the
// CTA then counts its reduced quadrants toward the task's readiness.  No counted arrivals are involved, so
// a failed launch, whose tasks are no longer ordered once its waits give up, can mix data but cannot put
// any barrier in an undefined state.
static __device__ __noinline__ void xchg_epilogue(const KParams &p, const UnitOut &uo, const UnitSpan &us, int t,
                                                  int u, uint32_t taddr, int q, int lane, int n, int m0, int mrows,
                                                  int set, bool leader, float *xbuf, uint64_t *acce,
                                                  volatile int *abort_flag) {
    const int nu = us.nu;
    const int pj = u - us.u0;                 // this unit's index in its tile
    const int base = (int)cluster_ctarank() - pj;  // cluster rank of the tile's unit 0
    const int owner = q % nu;                 // the tile's CTA that reduces quadrant q
    const int jq = q / nu;                    // which of the owner's quadrants it is
    const int rowf = p.xrow;
    const int slot_floats = 32 * rowf;
    const int flag_at = rowf - 4;
    const uint32_t seq = (uint32_t)t + 1u;
    tc_fence_after();
    if (owner != pj) {
        const int sl = pj < owner ? pj : pj - 1;
        const uint32_t dst = map_to_rank(smem_u32(xbuf + (size_t)(jq * (nu - 1) + sl) * slot_floats + lane * rowf),
                                         (uint32_t)(base + owner));
#pragma unroll 1
        for (int c = 0; c < mrows; c += 16) {
            uint32_t r[16];
            tmem_ld16(taddr + (uint32_t)c, r);
            tmem_ld_wait16(r);
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                st_cluster_v4(dst + (uint32_t)(c + i) * 4u, __uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                              __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
        }
        st_release_cluster_u32(dst + (uint32_t)flag_at * 4u, seq);
    } else {
        const float *rx = xbuf + (size_t)jq * (nu - 1) * slot_floats + lane * rowf;
        const bool ok = __all_sync(0xffffffffu, xchg_wait(rx, slot_floats, nu - 1, flag_at, seq, abort_flag,
                                                          p.wait_timeout_ns, p.status, t));
        if (ok) {
#pragma unroll 1
            for (int c = 0; c < mrows; c += 16) {
                uint32_t r[16];
                tmem_ld16(taddr + (uint32_t)c, r);
                tmem_ld_wait16(r);
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0.f;
                for (int j = 0; j < nu; ++j) {
                    float w[16];
                    if (j == pj) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) w[i] = __uint_as_float(r[i]);
                    } else {
                        const float4 *src = reinterpret_cast<const float4 *>(rx + (size_t)(j < pj ? j : j - 1) *
                                                                                       slot_floats + c);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float4 f = src[i];
                            w[4 * i] = f.x; w[4 * i + 1] = f.y; w[4 * i + 2] = f.z; w[4 * i + 3] = f.w;
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = (j == 0) ? w[i] : v[i] + w[i];
                }
                emit_outputs<16>(uo.e, n, m0 + c, min(16, mrows - c), v);
            }
        }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce);
    epi_bar(set);  // the set's reducing warps have stored their outputs
    if (leader) {
        trace_stamp(p, t, 6, globaltimer());
        if (uo.done) red_release_gpu_add(uo.done, (unsigned int)(kDonePerTile / nu));
        trace_stamp(p, t, 2, globaltimer());
    }
}

}  // namespace

// L2 prefetch of the W of the units this CTA would own in a round-robin (c,
// c + G, ...), p.prefetch_stages stages at most, in each unit's stream order,
// skipping the first `skip` stages of each first-round unit (its claimer's
// ring already holds them).  Out of line: it runs at most once per task.
template <bool kExt>
static __device__ __noinline__ void prefetch_w_l2(const KParams &p, const TaskDev &T, int skip) {
    int budget = p.prefetch_stages;
    for (int uu = blockIdx.x; uu < T.n_units && budget > 0; uu += gridDim.x) {
        const UnitSpan ps = unit_span(T, uu);
        int pg, pmt;
        tile_coords(T, ps.tile, pg, pmt);
        const int halves = p.wide ? 2 : 1;
        const int k_len = ps.k_end - ps.k_begin;
        const int k_rot = kExt ? unit_k_rot(p, T, ps) : (p.k_rotate ? (ps.tile * 11) % k_len : 0);  // as the producer
        for (int i = (uu < (int)gridDim.x ? skip : 0); i < k_len && budget > 0; ++i, --budget) {
            const int kk = ps.k_begin + (i + k_rot) % k_len;
            for (int h = 0; h < halves; ++h)
                for (int j = 0; j < p.kps; ++j)
                    tma_prefetch_l2_2d(&T.tmW, (kk * p.kps + j) * kUmmaBK, (pg * halves + h) * kUmmaRows);
        }
    }
}

// kExt compiles in what only some chains and calls need: cluster reduction of split tiles (KParams::cluster),
// die-grouped claims (TaskDev::die_split) and the K rotation's weight-column mapping for M-tiled tasks.
// Everything else runs the instantiation without them: measured on B200, that code in the kernel (not
// executed), and the column mapping's divisions on the producer thread and in the L2 prefetch, made the
// dependent 36 x 4 layer chain 2.7 % (3.49 -> 3.40 ms) and the independent decode step 2-3 % slower.
// kChain likewise separates chain runs from single calls (back-to-back single launches on the tensor
// cores 3-6 % faster without the chains' dependency and readiness code, e.g. o at M = 16 15.2 -> 14.3 us).
template <bool kChain, bool kExt>
__global__ void __launch_bounds__(kThreads, 1) wsm_umma_kernel(const __grid_constant__ KParams p) {
    // kChain: a chain run (run counter, task dependencies, readiness counters), else a single call; each
    // instantiation carries only its own accounting
    unsigned int *const run_ctl = kChain ? p.run_ctl : nullptr;
    const bool indep = !kChain && p.independent;
    auto tdep = [](const TaskDev &X) { return kChain ? X.dep : -1; };
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[kAccBufs];
    __shared__ __align__(8) uint64_t acce_bar[kAccBufs];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ int stage_meta[kMaxStages][4];   // {task, unit, flags, MMA instruction descriptor}, by the producer
    __shared__ int acc_meta[kAccBufs][3];       // {task, unit, flags}, written by the MMA thread
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_flag;
    __shared__ int last_flag[kEpiSets];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = p.stages;
    // 1024-byte aligned ring (required by the 128-byte swizzle pattern)
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(&accf_bar[b], 2);                  // tcgen05.commit + the MMA thread's metadata arrive
            mbar_init(&acce_bar[b], kEpiThreads / 32);
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        if (indep) pdl_launch_dependents();  // other calls trigger once past their grid wait (epilogue)
    }
    const int halves = p.wide ? 2 : 1;          // 128-row W halves per tile
    const uint32_t acc_stride = (uint32_t)(halves * kUmmaMaxN);  // TMEM columns per accumulator buffer
    if (warp == 1) tmem_alloc(&tmem_base_sh, p.wide ? kTmemColsWide : kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if ((kExt && p.cluster)) {
        // exchange flags start at 0 (no task's index + 1) before any peer can write them
        float *xb = reinterpret_cast<float *>(ring + p.xbuf_off);
        for (int i = threadIdx.x; i < 3 * 32; i += blockDim.x) xb[(size_t)i * p.xrow + p.xrow - 4] = 0.f;
        cluster_sync_all();
    }
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
            bool slot_ok = false;           // the wait for ring slot s has already succeeded
            // mode 2 streams W before the previous kernel completes; an independent call never waits here
            bool grid_dep_ok = p.pdl != 2 || indep;
            if (p.pdl == 1 && !indep) pdl_wait();
            if (p.debug_stall_ns && blockIdx.x == 0) {
                // test hook: after the previous kernel (whose exit clears the launch error flag), wait on a
                // flag nothing sets until the limit passes, then abandon all of this CTA's work
                if (!grid_dep_ok || indep) {
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
                const bool col_dep = tdep(T) >= 0 && T.dep_col_cnt != nullptr;
                // nothing of X before the dependency is met (per column: the first chunks; after that the
                // chunk mask decides stage by stage)
                bool dep_ok = tdep(T) < 0 && grid_dep_ok;
                int pend_s[kMaxStages], pend_k[kMaxStages], pend_y[kMaxStages];
                int np = 0;
                // Per-column dependency: each stage's X waits only for the kColChunk-column chunks it
                // reads (seen-complete chunks are cached in chunk_mask).
                unsigned long long chunk_mask = 0;
                unsigned int run_no = 0;
                auto stage_chunks = [&](int k0, int &c0, int &c1) {
                    c0 = k0 / kColChunk;
                    c1 = (min(k0 + p.kps * kUmmaBK, T.K) - 1) / kColChunk;
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
                    // the first-round units' first stages sit in their claimers' rings: the whole ring
                    // ahead of the grid dependency, dep_ring_stages ahead of a task dependency
                    prefetch_w_l2<kExt>(p, T, (tdep(T) >= 0 && p.dep_ring_stages > 0) ? min(S, p.dep_ring_stages) : S);
                };
                auto flush = [&]() {
                    if (!grid_dep_ok) {
                        prefetch_l2();
                        pdl_wait();
                        grid_dep_ok = true;
                    }
                    if (tdep(T) >= 0 && !col_dep) {
                        if (!prefetched && !dependency_met(p, task_at(p, tdep(T)))) prefetch_l2();
                        wait_dependency(p, task_at(p, tdep(T)), t, p.status);
                    }
                    if (col_dep && run_no == 0) run_no = ld_acquire_gpu(&run_ctl[0]) + 1u;
                    if (!dep_ok) trace_stamp(p, t, 1, globaltimer());
                    for (int i = 0; i < np; ++i) {
                        if (col_dep) {
                            int c0, c1;
                            stage_chunks(pend_k[i], c0, c1);
                            wait_chunks(p, T, c0, c1, run_no, chunk_mask, t, p.status);
                        }
                        for (int j = 0; j < p.kps; ++j)
                            tma_load_2d(ring + (size_t)pend_s[i] * p.stage_bytes + p.x_off + j * p.x_stride, &T.tmX,
                                        &full_bar[pend_s[i]], pend_k[i] + j * kUmmaBK, pend_y[i], pol_x);
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
                    if (np > 0 && tdep(T) >= 0 && p.dep_ring_stages > 0 && np >= p.dep_ring_stages) flush();
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
                // (die-grouped claims: this CTA's die's range first, then the other die's)
                const bool by_die = kExt && T.die_split > 0;
                const int my_die = by_die ? cta_die(p) : 0;
                ClaimRange cr = by_die ? die_claim_range(T, my_die) : claim_range(T);
                // (cluster mode: every task's first round is static, so a split tile's units of that round
                // sit on the consecutive CTAs of one cluster)
                const bool static_first = (t == 0 || (kExt && p.cluster)) && T.n_groups <= 1 && !by_die;  // (independent: t == 0)
                const int n_static = static_first ? min((int)gridDim.x, T.n_units) : 0;
                int u;
                if (static_first) {
                    u = (int)blockIdx.x < T.n_units ? (int)blockIdx.x : T.n_units;
                } else {
                    if (!grid_dep_ok) {
                        pdl_wait();
                        grid_dep_ok = true;
                        dep_ok = tdep(T) < 0;
                    }
                    u = cr.lo + claim_unit(cr);
                }
                for (int pass = 0;; ++pass) {
                    while (u < cr.hi) {
                        if (first_unit) {
                            trace_stamp(p, t, 0, globaltimer());
                            trace_stamp(p, t, 3, smid());
                            first_unit = false;
                        }
                        const UnitSpan us = unit_span(T, u);
                        int g, mt;
                        tile_coords(T, us.tile, g, mt);
                        const int xy = mt * T.t_m;
                        int next_u = cr.hi - cr.lo - n_static;
                        bool claimed = false;
                        const int k_len = us.k_end - us.k_begin;
                        // (without M-tiles a unit's weight column is its tile: kExt covers the chains with them)
                        const int k_rot = kExt ? unit_k_rot(p, T, us)
                                               : (p.k_rotate ? (us.tile * 11) % (us.k_end - us.k_begin) : 0);
                        for (int kk = us.k_begin; kk < us.k_end; ++kk) {
                            if (!take_slot()) break;
                            slot_ok = false;
                            uint8_t *st = ring + (size_t)s * p.stage_bytes;
                            stage_meta[s][0] = t;
                            stage_meta[s][1] = u;
                            stage_meta[s][2] = (kk == us.k_begin ? kMetaFirst : 0) | (kk == us.k_end - 1 ? kMetaLast : 0);
                            stage_meta[s][3] = (int)T.idesc;  // the MMA thread reads no task table
                            mbar_arrive_expect_tx(&full_bar[s], T.tx_bytes);
                            // the stage this iteration loads (rotated within the unit when k_rotate)
                            const int kr = k_rot ? us.k_begin + (kk - us.k_begin + k_rot) % k_len : kk;
                            const int k0 = kr * p.kps * kUmmaBK;
                            for (int h = 0; h < halves; ++h)
                                for (int j = 0; j < p.kps; ++j)
                                    tma_load_2d(st + (h * p.kps + j) * (kUmmaRows * kUmmaBK * 2), &T.tmW, &full_bar[s],
                                                k0 + j * kUmmaBK, (g * halves + h) * kUmmaRows, pol_w);
                            if (x_now(k0)) {
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
                            // claim the next unit kClaimLead stages before this one ends: early enough to
                            // hide the claim's round trip, late enough not to hold work a faster CTA could
                            // take -- and never while this task's dependency is unmet, when every CTA would
                            // hold a second unit it cannot start (the claim counters belong to the previous
                            // kernel until the grid dependency is resolved)
                            if (!claimed && !indep && dep_ok && us.k_end - kk <= kClaimLead) {
                                next_u = claim_unit(cr);
                                claimed = true;
                            }
                        }
                        if (aborted) break;
                        if (!claimed && !indep) {
                            // the unit streamed completely before its dependencies were resolved
                            if (!dep_ok) flush();
                            next_u = claim_unit(cr);
                        }
                        // whatever comes next needs a free slot: wait for it before the claim's result is used,
                        // so the claim's round trip overlaps the wait
                        if (!take_slot()) break;
                        u = indep ? u + (int)gridDim.x : cr.lo + next_u + n_static;
                    }
                    if (aborted || !by_die || pass > 0) break;
                    // own die's range done: help with the other die's
                    cr = die_claim_range(T, my_die ^ 1);
                    u = cr.lo + claim_unit(cr);
                }
                if (np > 0) flush();
                if (aborted) break;
                if (tdep(T) < 0 && !first_unit) trace_stamp(p, t, 1, globaltimer());
            }
            if (!run_ctl && !indep) {
                // every CTA counts the end of its claims, aborted or not (after the grid dependency: until
                // then the claim counters belong to the previous kernel)
                if (!grid_dep_ok) {
                    pdl_wait();
                    grid_dep_ok = true;
                }
                claims_finished(p.single, gridDim.x);
            }
            if (!grid_dep_ok) pdl_wait();  // a CTA with no work still orders itself after the previous kernel
            // copies in flight must land before exit, abort or not (checked before the end marker below
            // advances one of these barriers again)
            drain_issued(full_bar, S, issued, wlim, p.status);
            // end-of-work marker for the MMA thread (a stage with no data)
            if (!aborted && (slot_ok || mbar_wait_bounded(&empty_bar[s], ph ^ 1, &abort_flag, wlim, p.status, -1,
                                                          kSiteEmpty))) {
                stage_meta[s][0] = 0;
                stage_meta[s][1] = 0;
                stage_meta[s][2] = kMetaDone;
                mbar_arrive(&full_bar[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t acc_i = 0;   // accumulators handed to the epilogue so far
            bool any_mma = false;
            int buf = 0;
            int traced_t = -1;
            for (;;) {
                if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag, wlim, p.status, -1, kSiteFull)) break;
                tc_fence_after();
                const int t = stage_meta[s][0];
                const int u = stage_meta[s][1];
                const int flags = stage_meta[s][2];
                if (flags & kMetaDone) {
                    // the end marker goes to the next accumulator of EACH epilogue set
                    for (uint32_t d = 0; d < (uint32_t)kEpiSets; ++d) {
                        const uint32_t i = acc_i + d;
                        const int b = (int)(i % kAccBufs);
                        if (!mbar_wait_bounded(&acce_bar[b], ((i / kAccBufs) & 1) ^ 1, &abort_flag, wlim, p.status,
                                               -1, kSiteAcc))
                            break;
                        acc_meta[b][0] = 0;
                        acc_meta[b][1] = 0;
                        acc_meta[b][2] = kMetaDone;
                        mbar_arrive(&accf_bar[b]);
                        mbar_arrive(&accf_bar[b]);
                    }
                    break;
                }
                if (flags & kMetaFirst) {
                    buf = (int)(acc_i % kAccBufs);
                    if (!mbar_wait_bounded(&acce_bar[buf], ((acc_i / kAccBufs) & 1) ^ 1, &abort_flag, wlim, p.status,
                                           t, kSiteAcc))
                        break;
                    tc_fence_after();
                    if (kChain && p.trace && t != traced_t) {
                        trace_stamp(p, t, 7, globaltimer());
                        traced_t = t;
                    }
                }
                const uint32_t idesc = (uint32_t)stage_meta[s][3];
                const uint32_t st0 = smem_u32(ring + (size_t)s * p.stage_bytes);
                for (int h = 0; h < halves; ++h) {
                    // half h of the tile's W rows accumulates into columns h * 64 .. of the buffer
                    const uint32_t d_tmem = tmem_base + (uint32_t)buf * acc_stride + (uint32_t)(h * kUmmaMaxN);
                    for (int j = 0; j < p.kps; ++j) {
                        const uint32_t a0 = st0 + (uint32_t)((h * p.kps + j) * kUmmaRows * kUmmaBK * 2);
                        const uint32_t b0 = st0 + (uint32_t)(p.x_off + j * p.x_stride);
#pragma unroll
                        for (int k = 0; k < kUmmaBK / 16; ++k) {
                            // advancing K by 16 bf16 = 32 bytes inside the swizzle atom
                            tc_mma(d_tmem, sw128_desc(a0 + 32u * k), sw128_desc(b0 + 32u * k), idesc,
                                   ((flags & kMetaFirst) && j == 0 && k == 0) ? 0u : 1u);
                        }
                    }
                }
                any_mma = true;
                tc_commit(&empty_bar[s]);  // frees the stage once these MMAs have read it
                if (flags & kMetaLast) {
                    acc_meta[buf][0] = t;
                    acc_meta[buf][1] = u;
                    acc_meta[buf][2] = 0;
                    mbar_arrive(&accf_bar[buf]);   // publishes acc_meta
                    tc_commit(&accf_bar[buf]);     // accumulator complete
                    ++acc_i;
                }
                if (++s == S) {
                    s = 0;
                    ph ^= 1;
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
        // Two sets of four warps; set e takes accumulators e, e + 2, e + 4, ...
        const int set = (warp - kEpiWarp0) / 4;
        const int q = warp & 3;                 // TMEM lane quadrant this warp may access
        const int row = q * 32 + lane;          // row of the 128-row tile = TMEM lane
        const int etid = threadIdx.x - (kEpiWarp0 + 4 * set) * 32;
        const bool leader = (etid == 0);
        if (p.pdl && !indep) {
            pdl_wait();  // Y and the scratch may still be in use by the previous kernel
            // the next kernel may launch once every CTA has seen this one's predecessor complete: so at most
            // this kernel and the independent calls queued after it can still run when one of those starts
            if (set == 0 && leader) pdl_launch_dependents();
        }
        if (!run_ctl && !indep && etid < 32) {
            // a single call: the tile counters a failed call before it left mid-count are repaired first
            if (blockIdx.x == 0 && set == 0) repair_after_failure(p, lane);
            else if (leader) wait_repaired(p);
        }
        const unsigned int run_no = run_ctl ? ld_acquire_gpu(&run_ctl[0]) + 1u : 0u;  // this chain run
        int warm_t = 0;                         // the task whose descriptor the set warms while it waits
        for (uint32_t k = 0;; ++k) {
            const uint32_t acc_i = kEpiSets * k + (uint32_t)set;
            const int buf = (int)(acc_i % kAccBufs);
            const uint32_t aph = (acc_i / kAccBufs) & 1;
            if (leader) prefetch_task_l1(p, warm_t);
            const bool ab = !mbar_wait_bounded(&accf_bar[buf], aph, &abort_flag, wlim, p.status, -1, kSiteAcc);
            // the four warps of the set stop together (an abort anywhere, or the end marker)
            const int flags = ab ? kMetaDone : acc_meta[buf][2];
            if (vote_or(ab || (flags & kMetaDone), 1 + set, kEpiThreads)) break;
            const int t = acc_meta[buf][0];
            const int u = acc_meta[buf][1];
            warm_t = t + 1;
            if (leader) trace_stamp(p, t, 4, globaltimer());
            const TaskDev &T = task_at(p, t);
            const UnitSpan us = unit_span(T, u);
            const int tile = us.tile;
            int g, mt;
            tile_coords(T, tile, g, mt);
            const int m0 = mt * T.t_m;
            const int mrows = min(T.t_m, T.M - m0);
            UnitOut uo = unit_out(T);  // no task-table reads after the first store below
            unit_out_group(uo, T, tile);
            if ((kExt && p.cluster) && us.nu > 1 && u < min((int)gridDim.x, T.u_head)) {
                // a split tile of a static first round: its units are on this cluster's CTAs
                xchg_epilogue(p, uo, us, t, u, tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)buf * acc_stride, q,
                              lane, g * kUmmaRows + row, m0, mrows, set, leader,
                              reinterpret_cast<float *>(ring + p.xbuf_off), &acce_bar[buf], &abort_flag);
                continue;
            }
            // The accumulator, 16 columns (X rows) at a time, per 128-row half of the tile: TMEM ->
            // registers -> outputs (whole tile) or this unit's partial rows [row][m] (split tile).  The
            // loops are not unrolled: one copy of the epilogue code per kind keeps the kernel small.
            tc_fence_after();
#pragma unroll 1
            for (int h = 0; h < halves; ++h) {
                const int n = (g * halves + h) * kUmmaRows + row;
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)buf * acc_stride + (uint32_t)(h * kUmmaMaxN);
                float4 *dst = reinterpret_cast<float4 *>(uo.part + (size_t)u * uo.slot_elems +
                                                         (size_t)(h * kUmmaRows + row) * uo.t_mpad);
#pragma unroll 1
                for (int c = 0; c < mrows; c += 16) {
                    uint32_t r[16];
                    tmem_ld16(taddr + (uint32_t)c, r);
                    tmem_ld_wait16(r);
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
                    if (us.nu == 1) {
                        emit_outputs<16>(uo.e, n, m0 + c, min(16, mrows - c), v);
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if (c + 4 * i < mrows)
                                dst[c / 4 + i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar[buf]);

            if (us.nu == 1) {
                if (uo.done || uo.col_cnt) {
                    epi_bar(set);
                    if (leader) tile_finished(uo, g, halves * kUmmaRows, run_no);  // release covers the set's stores
                }
            } else {
                // the last unit of the tile to arrive adds all the partials
                epi_bar(set);
                if (leader) {
                    // acq_rel: releases this set's partial (stored before the barrier) and acquires the
                    // others' for the last arriver
                    const unsigned int old = atom_add_acqrel_gpu(&uo.tile_cnt[tile], 1u);
                    last_flag[set] = (old == (unsigned int)(us.nu - 1)) ? 1 : 0;
                    trace_stamp(p, t, 5, globaltimer());
                }
                epi_bar(set);
                if (last_flag[set]) {
                    // the leader's acquire + the barrier order these loads after every partial
#pragma unroll 1
                    for (int h = 0; h < halves; ++h) {
                        const int n = (g * halves + h) * kUmmaRows + row;
                        if (mrows <= 4)
                            reduce_row_partials<4, 16>(uo, us, h * kUmmaRows + row, mrows, m0, n);
                        else
                            reduce_row_partials<16, 4>(uo, us, h * kUmmaRows + row, mrows, m0, n);
                    }
                    epi_bar(set);
                    if (leader) {
                        trace_stamp(p, t, 6, globaltimer());
                        uo.tile_cnt[tile] = 0u;  // ready for the next call
                        tile_finished(uo, g, halves * kUmmaRows, run_no);
                    }
                }
            }
            if (leader) trace_stamp(p, t, 2, globaltimer());
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if ((kExt && p.cluster)) cluster_sync_all();  // no CTA leaves while a peer may still write its exchange buffer
    if (warp == 1) tmem_dealloc(tmem_base, p.wide ? kTmemColsWide : kTmemCols);
    if (threadIdx.x == 0) {
        if (run_ctl) chain_run_done(p);
        // an independent call completes only after the kernel before it (later kernels rely on stream
        // order): one CTA waits for it, the others leave their SMs to the calls beside this one
        else if (indep && blockIdx.x == 0 && p.pdl) pdl_wait();
    }
}

template __global__ void wsm_umma_kernel<false, false>(const __grid_constant__ KParams p);
template __global__ void wsm_umma_kernel<false, true>(const __grid_constant__ KParams p);
template __global__ void wsm_umma_kernel<true, false>(const __grid_constant__ KParams p);
template __global__ void wsm_umma_kernel<true, true>(const __grid_constant__ KParams p);

const void *umma_kernel_ptr(bool chain, bool ext) {
    if (chain)
        return ext ? reinterpret_cast<const void *>(&wsm_umma_kernel<true, true>)
                   : reinterpret_cast<const void *>(&wsm_umma_kernel<true, false>);
    return ext ? reinterpret_cast<const void *>(&wsm_umma_kernel<false, true>)
               : reinterpret_cast<const void *>(&wsm_umma_kernel<false, false>);
}

}  // namespace wsm
