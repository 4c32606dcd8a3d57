// wsm_internal.cuh -- definitions shared by the weight-streaming kernels and
// the host runtime of libwsm (not part of the public C ABI).
//
// Work decomposition (both kernel paths):
//   A GEMM is cut into tiles: `tile_rows` rows of W (outputs along N) times one
//   M-tile of X.  A tile's K range is cut into `kb` pipeline stages, and the
//   stages into `nu` work units of `ku` consecutive stages (the last unit may
//   be shorter).  Units are numbered tile-major (u = tile * nu + j); CTA c
//   starts with unit c, and the rest are handed out IN ORDER from one atomic
//   counter per task: each persistent CTA's producer claims its next unit when
//   it starts the current one.  The SMs of
//   a B200 do not stream at the same rate (measured: a 2x spread between the
//   fastest and slowest SMs on the same access pattern), so claiming units
//   lets every SM work until the task is done instead of the task waiting for
//   the slowest SM's fixed share.
//
//   A tile split into nu > 1 units gets one fp32 partial per unit, stored in
//   the unit's own slot; the unit that arrives last on the tile's counter adds
//   the nu partials in unit order (= K order).  Where a unit ends is fixed by
//   the plan, not by which CTA ran it, so the result is the same for every run
//   and every grid size.  This is the inter-CTA split-K of the FlyDSL article
//   ("AMD: ROCm Low-Latency-GEMM-Kernel ... MI355X", technique 1), with the
//   split placed per unit.  Claiming in order also keeps the M-tiles of one
//   weight column (adjacent unit numbers) in flight together, the cooperative
//   M-major traversal of "Fleet ..." (reading notes, section 3f, Eq.(1)).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace wsm {

constexpr int kMaxStages = 16;
constexpr int kUmmaRows = 128;     // rows of W per UMMA tile (MMA M)
constexpr int kUmmaBK = 64;        // K elements per UMMA box (one 128-byte swizzle row)
constexpr int kUmmaMaxN = 64;      // largest MMA N (= X rows per tile)
constexpr int kStreamBoxK = 256;   // K elements per TMA box on the FMA path
// Status block (the first 256 bytes of a call's scratch or a chain's buffer):
//   [0] first error code, [1] its task, [2] its CTA, [3] its site -- sticky: kept over later calls until the
//       host reads and clears them (wsm_stream_status, wsm_workspace_status, wsm_chain_status,
//       gemm_chain_status);
//   [4] an error was recorded in the CURRENT launch: bounded waits give up early on it, and the launch's
//       last CTA repairs the counters the launch left mid-count and clears it at exit;
//   [5] never written by anyone: the flag the stall test hook waits on.
constexpr int kStatusWords = 4;    // words the host reads: [0] code, [1] task, [2] CTA, [3] site
constexpr int kStatusLaunchErr = 4;
constexpr int kStatusStallFlag = 5;
// Independent single calls (KParams::independent) record into a second status block in the same 256-byte
// status region: their launch error word must not make the calls running beside them give up, and no
// call clears it (none of their waits consult it).
constexpr int kIndStatusOff = 32;  // ints
static_assert(kIndStatusOff + kStatusStallFlag < 64, "the status region holds 64 ints");

constexpr int kSchedWords = 2;     // per task: [0] next unit to claim, [1] CTAs done claiming
constexpr int kClaimLead = 4;      // a CTA claims its next unit this many stages before its unit ends
constexpr int kColChunk = 256;     // output columns per readiness chunk (per-column data dependencies)
// A task's `done` counter counts quarter tiles (32-row quadrants of a 128-row tile's outputs; a wide tile's
// quarter is 64 rows): a finished tile adds 4, and in a cluster reduction each CTA adds the quadrants it
// reduced and stored.  (With two-level readiness `done` counts groups instead.)
constexpr int kDonePerTile = 4;
constexpr int kClusterCtas = 4;    // CTAs per thread-block cluster in cluster-reduction chains
constexpr int kMaxSmIds = 1024;    // entries of the SM-id -> die table of die-grouped chains
// Trace stamps per CTA and task (%globaltimer ns unless noted): [0] first stage issued, [1] dependency
// met, [2] last unit's outputs written, [3] SM id, [4] last unit's accumulator at the epilogue, [5] its
// split-K arrival counted, [6] its in-order reduction done (last arriver only), [7] first stage of the
// task complete at the MMA issuer.
constexpr int kTraceSlots = 8;

// Epilogues (== WSM_EPI_*).
enum : int { kEpiNone = 0, kEpiSiluMul = 1, kEpiResidual = 2 };

// Error sites recorded in status[3].
enum : int { kSiteNone = 0, kSiteDep = 1, kSiteFull = 2, kSiteEmpty = 3, kSiteAcc = 4, kSiteDrain = 5, kSiteStall = 6,
             kSiteXchg = 7, kSiteRepair = 8 };
constexpr int kCodeTimeout = 6;    // == WSM_ERR_TIMEOUT

// Stage / accumulator metadata flags (producer -> consumers).
constexpr int kMetaFirst = 1;      // first stage of its unit
constexpr int kMetaLast = 2;       // last stage of its unit
constexpr int kMetaDone = 4;       // no more work for this CTA: the role exits

// One GEMM as the kernels see it.  Lives in kernel parameter space (single
// GEMM) or in a device table (chain); 64-byte aligned for the tensor maps.
struct __align__(64) TaskDev {
    CUtensorMap tmW;            // W [N, K] bf16
    CUtensorMap tmX;            // X [M, K] bf16
    __nv_bfloat16 *Y;           // [M, N]
    float *Yf32;                // optional [M, N]
    float *part;                // n_units partial slots of slot_elems floats
    unsigned int *tile_cnt;     // [n_tiles] arrival counters, zero between calls
    unsigned int *sched;        // [kSchedWords] unit claim counters, zero between calls
    unsigned int *done;         // tiles finished (monotonic over runs), chain only
    int M, N, K;
    int dep;                    // -1 or index of an earlier task
    int n_g;                    // column tiles along N
    int n_mt;                   // M-tiles
    int t_m;                    // X rows per M-tile
    int t_mpad;                 // X rows loaded per M-tile (UMMA: multiple of 16)
    int kb;                     // stages per tile
    // Work units.  The first t_head tiles of the schedule are split into nu
    // units of ku stages (u_head = t_head * nu units), the remaining tiles
    // into nu_t units of ku_t stages: big units first, small ones last, so the
    // end of a task is spread evenly over the CTAs.
    int ku;                     // stages per head unit
    int nu;                     // units per head tile
    int t_head;                 // head tiles
    int u_head;                 // t_head * nu
    int ku_t;                   // stages per tail unit
    int nu_t;                   // units per tail tile
    int n_units;                // u_head + (n_g * n_mt - t_head) * nu_t
    int k_major;                // units ordered K-range first: unit u = K-range u / tiles of tile u % tiles
                                // (no tail split); partial slot u either way
    int order;                  // 0: M-tile inner (M-major), 1: M-tile outer
    int notify;                 // bump `done` after each finished tile
    int epi;                    // kEpi*
    int y_cols;                 // output columns: N, or N / 2 with SiLU*mul
    const __nv_bfloat16 *R;     // residual [M, N] (kEpiResidual)
    unsigned int *col_cnt;      // per kColChunk output columns: tiles finished (monotonic over runs), or nullptr
    const unsigned int *col_need;      // tiles that touch each chunk, per run
    const unsigned int *dep_col_cnt;   // per-column dependency: the dep task's col_cnt, else nullptr
    const unsigned int *dep_col_need;  // ... and its col_need
    // Two-level readiness (n_groups > 1): CTA c belongs to group c % n_groups, group g owns the
    // contiguous tiles [g T / G, (g+1) T / G) and claims their units from grp_sched[g]; a finished tile
    // bumps grp_done[g] and the group's last tile bumps `done` once: done counts groups, not tiles.
    int n_groups;
    unsigned int *grp_sched;    // [n_groups] claim counters, zero between runs
    unsigned int *grp_done;     // [n_groups] finished tiles per group (monotonic over runs)
    // Die-grouped claims (die_split > 0): tiles [0, die_split) belong to die 0, the rest to die 1; a CTA
    // claims its die's range from die_sched[die], then the other range.  No tail units.
    int die_split;
    unsigned int *die_sched;    // [2] claim counters, zero between runs
    int w_evict_first;          // L2 policy of the weight loads
    uint32_t idesc;             // UMMA instruction descriptor (MMA N = t_mpad)
    uint32_t tx_bytes;          // bytes landing in one stage
    int slot_elems;             // floats per partial slot
};

struct KParams {
    TaskDev single;                 // used when tasks == nullptr
    const TaskDev *tasks;           // chain table (device), or nullptr
    int n_tasks;
    int stages;                     // ring depth
    int stage_bytes;                // bytes per ring stage
    int x_off;                      // offset of the X part inside a stage
    uint32_t dep_target_extra;      // 0; a test hook makes every dependency unreachable with it
    int prefetch_stages;            // W stages a waiting CTA prefetches into L2 (0: none)
    unsigned int *run_ctl;          // chain: [0] runs completed, [1] CTAs done with this run; or nullptr
    int kps;                        // UMMA path: 64-wide K boxes per stage
    int x_stride;                   // UMMA path: bytes between the X boxes of a stage
    int pdl;                        // 0: plain launch; 1: wait for the previous kernel before any
                                    // global access; 2: stream W before that wait, X after it
    int k_rotate;                   // each unit walks its K stages starting at a tile-dependent offset
                                    // (wrapping), so CTAs do not all read the same weight columns at once
    int dep_ring_stages;            // W stages a CTA issues into its ring while its task's dependency is
                                    // unmet (0: the whole ring)
    int wide;                       // UMMA path: tiles of 2 x 128 W rows sharing each X stage (two MMAs into
                                    // two accumulators), so X is re-read half as often; 0: 128-row tiles
    int *status;                    // kStatusWords ints
    unsigned long long dep_timeout_ns;
    unsigned long long wait_timeout_ns;
    unsigned long long *trace;      // [grid][n_tasks][kTraceSlots] or nullptr
    unsigned long long debug_stall_ns;  // test hook, 0 in real use: CTA 0's producer waits this long on a flag
                                        // nothing sets, records a time-out and abandons its work
    int cluster;                    // 0, or kClusterCtas: launched as clusters; every task's first round of
                                    // units is static (unit c on CTA c) and a split tile of that round, whose
                                    // units sit on the CTAs of one cluster, is reduced through distributed
                                    // shared memory instead of global partials
    int xbuf_off;                   // cluster mode: byte offset of the exchange buffer from the ring's start
    int xrow;                       // cluster mode: floats per exchange-buffer row (widest X tile + 4, the
                                    // last 4 holding the row's flag)
    const signed char *sm_die;      // die-grouped claims: die of each SM id (kMaxSmIds entries), or nullptr
    int cnt_words;                  // single calls: words of the scratch's counter region from single.sched on
                                    // (zeroed by the next call after a failed one)
    int independent;                // single call that shares no data with the kernel before it and splits no
                                    // tile: CTA c runs units c, c + grid, ... (no claim counters, no scratch),
                                    // loads and stores without waiting for the previous kernel, and waits for it
                                    // only before exiting (so stream order stays transitive for later kernels)
};

#if defined(__CUDACC__)

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smid() {
    uint32_t v;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(v));
    return v;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// true when the phase with parity `parity` has completed
__device__ __forceinline__ bool mbar_try(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// L2 prefetch of one box of a tensor map: no shared memory, nothing to wait for.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_gpu_add(unsigned int *p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned int atom_add_acqrel_gpu(unsigned int *p, unsigned int v) {
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ unsigned int atom_add_relaxed_gpu(unsigned int *p, unsigned int v) {
    unsigned int old;
    asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void st_relaxed_gpu(unsigned int *p, unsigned int v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_release_gpu(unsigned int *p, unsigned int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ thread-block clusters

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster: all have arrived (and their earlier shared-memory writes,
// mbarrier initialisation included, are visible cluster-wide) before any continues.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared::cluster address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Arrive (count 1) on an mbarrier of another CTA of the cluster; release: this thread's earlier writes
// (its distributed shared memory stores included) are visible to the thread that sees the phase complete.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Arrive with `count` on a local mbarrier; returns the token of the phase arrived on.
__device__ __forceinline__ uint64_t mbar_arrive_count(uint64_t *bar, uint32_t count) {
    uint64_t state;
    asm volatile("mbarrier.arrive.shared::cta.b64 %0, [%1], %2;" : "=l"(state) : "r"(smem_u32(bar)), "r"(count)
                 : "memory");
    return state;
}

// true once the phase of `state` has completed; acquire at cluster scope (remote writers' stores visible)
__device__ __forceinline__ bool mbar_try_token_cluster(uint64_t *bar, uint64_t state) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "l"(state)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ float ld_cg_f32(const float *p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// Programmatic dependent launch: let the next kernel on the stream begin its
// prologue, and wait for the previous kernel's completion (and memory).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Record an error: the first one since the host last cleared the status (code, task, cta, site), and the
// current launch's error flag.
__device__ __forceinline__ void record_error(int *status, int code, int task, int site) {
    if (!status) return;
    if (atomicCAS(status, 0, code) == 0) {
        status[1] = task;
        status[2] = (int)blockIdx.x;
        status[3] = site;
    }
    *((volatile int *)&status[kStatusLaunchErr]) = 1;
    __threadfence();
}

// An error was recorded in the current launch (an earlier launch's sticky error does not count: the
// counters that launch left were repaired when it ended).
__device__ __forceinline__ bool launch_failed(const int *status) {
    return status && *((volatile const int *)&status[kStatusLaunchErr]) != 0;
}

// Bounded wait on an mbarrier phase.  Returns false (and records an error)
// when `limit_ns` of %globaltimer pass, or when `abort_flag` is raised.  The
// spin loop is a real call (not inlined at the many wait sites): the
// kernels' hot code stays small enough for the instruction caches.
static __device__ __noinline__ bool mbar_wait_spin(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                            unsigned long long limit_ns, int *status, int task, int site);
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                  unsigned long long limit_ns, int *status, int task, int site) {
    if (mbar_try(bar, parity)) return true;
    return mbar_wait_spin(bar, parity, abort_flag, limit_ns, status, task, site);
}
static __device__ __noinline__ bool mbar_wait_spin(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                            unsigned long long limit_ns, int *status, int task, int site) {
    unsigned long long t0 = globaltimer();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try(bar, parity)) return true;
        if ((spin & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) {
                record_error(status, kCodeTimeout, task, site);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Before a CTA exits, every TMA copy it issued must have landed: wait for the
// full barriers of the last min(S, issued) stages, under ONE overall
// deadline (a healthy run finds them all complete already).
__device__ __forceinline__ void drain_issued(uint64_t *full_bars, int S, long long issued,
                                             unsigned long long limit_ns, int *status) {
    const unsigned long long t0 = globaltimer();
    const long long first = issued > S ? issued - S : 0;
    for (long long i = first; i < issued; ++i) {
        uint64_t *b = &full_bars[i % S];
        const uint32_t ph = (uint32_t)((i / S) & 1);
        while (!mbar_try(b, ph)) {
            if (globaltimer() - t0 > limit_ns) {
                record_error(status, kCodeTimeout, -1, kSiteDrain);
                return;
            }
        }
    }
}

// ------------------------------------------------------------------ scheduling

__device__ __forceinline__ const TaskDev &task_at(const KParams &p, int t) {
    return p.tasks ? p.tasks[t] : p.single;
}

// Warm this SM's L1 with the part of task t's descriptor past its tensor maps
// (the fields the epilogue reads), so a CTA's first unit of a task does not
// wait on loaded L2 round trips for them.  Chains only: a single GEMM's
// descriptor is a kernel parameter.
__device__ __forceinline__ void prefetch_task_l1(const KParams &p, int t) {
    if (!p.tasks || t >= p.n_tasks) return;
    const char *b = reinterpret_cast<const char *>(p.tasks + t);
    for (size_t off = 2 * sizeof(CUtensorMap); off < sizeof(TaskDev); off += 128)
        asm volatile("prefetch.global.L1 [%0];" ::"l"(b + off));
}

// Tile index -> (column tile g, M-tile mt).
__device__ __forceinline__ void tile_coords(const TaskDev &T, int tile, int &g, int &mt) {
    if (T.order == 0) {
        g = tile / T.n_mt;
        mt = tile - g * T.n_mt;
    } else {
        mt = tile / T.n_g;
        g = tile - mt * T.n_g;
    }
}

// Work unit u of task T: its tile, the tile's first unit and unit count (its
// partial slots are u0 .. u0 + nu - 1, in K order) and its stage range.
struct UnitSpan {
    int tile, u0, nu, k_begin, k_end;
    int slot_stride;  // partial slot of the tile's unit j = u0 + j * slot_stride
};
__device__ __forceinline__ UnitSpan unit_span(const TaskDev &T, int u) {
    UnitSpan r;
    int j, ku;
    r.slot_stride = 1;
    if (T.k_major) {
        const int tiles = T.n_g * T.n_mt;
        j = u / tiles;
        r.tile = u - j * tiles;
        r.nu = T.nu;
        r.u0 = r.tile;
        r.slot_stride = tiles;
        r.k_begin = j * T.ku;
        r.k_end = min(r.k_begin + T.ku, T.kb);
        return r;
    }
    if (u < T.u_head) {
        r.tile = u / T.nu;
        j = u - r.tile * T.nu;
        r.nu = T.nu;
        ku = T.ku;
    } else {
        const int v = u - T.u_head;
        const int tt = v / T.nu_t;
        r.tile = T.t_head + tt;
        j = v - tt * T.nu_t;
        r.nu = T.nu_t;
        ku = T.ku_t;
    }
    r.u0 = u - j;
    r.k_begin = j * ku;
    r.k_end = min(r.k_begin + ku, T.kb);
    return r;
}

// First stage a unit streams, counted from its k_begin: with k_rotate, units
// start at an offset that depends on their weight column and wrap around, so
// CTAs that run in lockstep do not all read the same columns of their weight
// rows at once.
// The offset depends on the tile's weight column, not on the tile: the M-tiles that share a column (M-major
// order) then stream its stages in the same order, close together in time, so all but the first find them
// in L2 (Eq.(1) of the Fleet reading notes, section 3f).  Measured on B200 with a per-tile offset instead
// (L2-reuse chain, M = 32 / 64 in 16-row M-tiles): 853 MB read from DRAM for 607 MB of weights, L2 hit rate
// 52 %.
__device__ __forceinline__ int unit_k_rot(const KParams &p, const TaskDev &T, const UnitSpan &us) {
    if (!p.k_rotate) return 0;
    const int col = T.order == 0 ? us.tile / T.n_mt : us.tile % T.n_g;
    return (col * 11) % (us.k_end - us.k_begin);
}

// The units a CTA claims from: all of the task's, or with two-level readiness
// its group's tiles (tile-major units, so a contiguous range).
struct ClaimRange {
    unsigned int *ctr;
    int lo, hi;
};
__device__ __forceinline__ int group_tile_lo(const TaskDev &T, int g) {
    return (int)((long long)g * (T.n_g * T.n_mt) / T.n_groups);
}
__device__ __forceinline__ int group_of_tile(const TaskDev &T, int tile) {
    return (int)(((long long)(tile + 1) * T.n_groups - 1) / (T.n_g * T.n_mt));
}
__device__ __forceinline__ ClaimRange claim_range(const TaskDev &T) {
    ClaimRange r;
    if (T.n_groups <= 1) {
        r.ctr = &T.sched[0];
        r.lo = 0;
        r.hi = T.n_units;
    } else {
        const int g = (int)blockIdx.x % T.n_groups;
        r.ctr = &T.grp_sched[g];
        r.lo = group_tile_lo(T, g) * T.nu;
        r.hi = group_tile_lo(T, g + 1) * T.nu;
    }
    return r;
}

// Die-grouped claims: the range of die `d` (0 or 1) of task T.
__device__ __forceinline__ ClaimRange die_claim_range(const TaskDev &T, int d) {
    ClaimRange r;
    r.ctr = &T.die_sched[d];
    r.lo = d == 0 ? 0 : T.die_split * T.nu;
    r.hi = d == 0 ? T.die_split * T.nu : T.n_units;
    return r;
}
// ... and the die of the SM this CTA runs on (0 when the table has no entry for it).
__device__ __forceinline__ int cta_die(const KParams &p) {
    const uint32_t sm = smid();
    return (p.sm_die && sm < (uint32_t)kMaxSmIds && p.sm_die[sm] == 1) ? 1 : 0;
}

// Claim the next dynamic unit: the caller adds cr.lo and the number of units
// handed out statically (unit c to CTA c); a result >= cr.hi means none left.
__device__ __forceinline__ int claim_unit(const ClaimRange &cr) { return (int)atom_add_relaxed_gpu(cr.ctr, 1u); }

// Single GEMM accounting, kept off the end of the launch (an atomic there delayed every launch's completion
// by its round trip: measured on B200, M = 1 4096 x 4096 back to back 10.5 -> 10.8 us).
//
// claims_finished: called once per CTA by the producer thread after its last claim, aborted or not; the
// last CTA to finish claiming resets the claim counters for the next call.
//
// A launch that records an error (some CTA abandoned its work) may leave split-tile arrival counters
// mid-count, and its launch error flag set.  The next single call on the same scratch repairs them before
// any of its CTAs counts an arrival: the warp of CTA 0's first epilogue leader, once the previous kernel
// has completed, zeroes the tile counters (the whole counter region: the failed call's shape is not known)
// and clears the flag (repair_after_failure); every other epilogue leader waits, bounded, until the flag
// is clear (wait_repaired).  The claim counters need no repair (every CTA counts its claims' end).  The sticky error
// words stay for the host to read.  A chain resets its counters at the end of each run (chain_run_done).
__device__ __forceinline__ void claims_finished(const TaskDev &T, unsigned int grid) {
    const unsigned int old = atom_add_acqrel_gpu(&T.sched[1], 1u);
    if (old == grid - 1) {
        st_relaxed_gpu(&T.sched[0], 0u);
        st_relaxed_gpu(&T.sched[1], 0u);
    }
}

// CTA 0: the warp of its (first) epilogue leader, all 32 lanes, after the grid dependency.
__device__ __forceinline__ void repair_after_failure(const KParams &p, int lane) {
    unsigned int *flag = reinterpret_cast<unsigned int *>(&p.status[kStatusLaunchErr]);
    unsigned int v = lane == 0 ? ld_acquire_gpu(flag) : 0u;
    v = __shfl_sync(0xffffffffu, v, 0);
    if (v == 0u) return;
    unsigned int *cnt = p.single.sched + kSchedWords;
    for (int i = lane; i < p.cnt_words - kSchedWords; i += 32) st_relaxed_gpu(&cnt[i], 0u);
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_gpu(flag, 0u);
}

// Every other epilogue leader (the only thread that counts arrivals), after the grid dependency; false
// (with an error recorded) if the repair did not come within the limit.
static __device__ __noinline__ bool wait_repaired(const KParams &p) {
    const unsigned int *flag = reinterpret_cast<const unsigned int *>(&p.status[kStatusLaunchErr]);
    if (ld_acquire_gpu(flag) == 0u) return true;
    // the repair follows within microseconds (CTA 0 passed the same grid dependency); a flag that stays set
    // was set by this launch itself, whose own failure is on record already
    const unsigned long long limit = p.wait_timeout_ns < 100000000ull ? p.wait_timeout_ns : 100000000ull;
    const unsigned long long t0 = globaltimer();
    for (uint32_t spin = 1;; ++spin) {
        if (ld_acquire_gpu(flag) == 0u) return true;
        if ((spin & 31u) == 0) {
            if (globaltimer() - t0 > limit) {
                record_error(p.status, kCodeTimeout, -1, kSiteRepair);
                return false;
            }
            __nanosleep(256);
        }
    }
}

// Test hook (KParams::debug_stall_ns): a bounded wait on a status word that nothing ever sets.  When the
// limit passes it records a time-out and raises the CTA's abort flag; the caller then abandons its work.
static __device__ __noinline__ void debug_stall(const KParams &p, volatile int *abort_flag) {
    const unsigned int *flag = reinterpret_cast<const unsigned int *>(&p.status[kStatusStallFlag]);
    const unsigned long long t0 = globaltimer();
    for (uint32_t spin = 1;; ++spin) {
        if (ld_acquire_gpu(flag) != 0u) return;
        if ((spin & 31u) == 0 && globaltimer() - t0 > p.debug_stall_ns) break;
        __nanosleep(256);
    }
    record_error(p.status, kCodeTimeout, -1, kSiteStall);
    *abort_flag = 1;
}

// Sum, in unit order (= K order), of the partials of rows m0 .. m0+MB-1 (those
// below mrows) of the nu units of one tile, at element `off` of row 0 of each
// slot.  The loads of a block of CB units x MB rows are issued together, so
// the reduction costs a few L2 round trips rather than one per partial.
template <int MB, int CB>
__device__ __forceinline__ void ordered_unit_sums(const float *tile_slots, int slot_elems, int row_stride, int off,
                                                  int m0, int mrows, int nu, float (&sum)[MB]) {
    for (int jb = 0; jb < nu; jb += CB) {
        float v[CB][MB];
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            const float *q = tile_slots + (size_t)(jb + u) * slot_elems + off;
#pragma unroll
            for (int i = 0; i < MB; ++i)
                v[u][i] = (jb + u < nu && m0 + i < mrows) ? ld_cg_f32(q + (size_t)(m0 + i) * row_stride) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            if (jb + u < nu) {
#pragma unroll
                for (int i = 0; i < MB; ++i) sum[i] = (jb + u == 0) ? v[u][i] : sum[i] + v[u][i];
            }
        }
    }
}

// Bounded wait for task `dep` of a chain to have finished all its tiles in
// this run.  On time-out (or an error elsewhere) records it and returns; the
// caller then proceeds with whatever X holds, so the kernel always ends.
// The run number is read from device memory (not a launch parameter) so a
// chain captured once in a CUDA graph stays correct over any number of
// replays; the last CTA to finish a run advances it (chain_run_done).
// What an epilogue writes, copied out of the task table into registers once
// per unit: loads through the table reference cannot be hoisted over the
// output stores (they might alias), and each reload is an L2 round trip.
struct EpiOut {
    __nv_bfloat16 *Y;
    float *Yf32;
    const __nv_bfloat16 *R;
    int N, y_cols, epi;
};
__device__ __forceinline__ EpiOut epi_out(const TaskDev &T) {
    EpiOut e;
    e.Y = T.Y;
    e.Yf32 = T.Yf32;
    e.R = T.R;
    e.N = T.N;
    e.y_cols = T.y_cols;
    e.epi = T.epi;
    return e;
}

// Everything a unit's epilogue touches after its first store, in registers
// (see EpiOut).
struct UnitOut {
    EpiOut e;
    float *part;
    unsigned int *tile_cnt;
    unsigned int *done;     // nullptr unless some task waits for this whole task
    unsigned int *col_cnt;  // nullptr unless some task waits for its columns
    unsigned int *grp_done; // two-level readiness, else nullptr
    int slot_elems, t_mpad;
    int grp_tiles;          // two-level: tiles of the unit's group
    int grp;                // ... and the group
};
__device__ __forceinline__ UnitOut unit_out(const TaskDev &T) {
    UnitOut o;
    o.e = epi_out(T);
    o.part = T.part;
    o.tile_cnt = T.tile_cnt;
    o.done = T.notify ? T.done : nullptr;
    o.col_cnt = T.col_cnt;
    o.slot_elems = T.slot_elems;
    o.t_mpad = T.t_mpad;
    o.grp_done = (T.notify && T.n_groups > 1) ? T.grp_done : nullptr;
    o.grp = 0;
    o.grp_tiles = 0;
    return o;
}
// Two-level readiness: the group of the unit's tile (call before the first store).
__device__ __forceinline__ void unit_out_group(UnitOut &o, const TaskDev &T, int tile) {
    if (!o.grp_done) return;
    o.grp = group_of_tile(T, tile);
    o.grp_tiles = group_tile_lo(T, o.grp + 1) - group_tile_lo(T, o.grp);
}

// A finished tile (column tile g, rows_per_tile rows of W) counts toward every
// kColChunk-column chunk of the output it wrote.  Called by one thread after a
// barrier that follows all the tile's stores (release).
__device__ __forceinline__ void notify_columns(const UnitOut &o, int g, int rows_per_tile) {
    int c_lo = g * rows_per_tile;
    int c_hi = min(o.e.N, c_lo + rows_per_tile);
    if (o.e.epi == kEpiSiluMul) {  // N and the tile heights are multiples of 16
        c_lo >>= 1;
        c_hi >>= 1;
    }
    for (int c = c_lo / kColChunk; c <= (c_hi - 1) / kColChunk; ++c) red_release_gpu_add(&o.col_cnt[c], 1u);
}

// The tile is complete: whole-task and per-column readiness (leader thread,
// after the barrier that follows the tile's last stores).
__device__ __forceinline__ void tile_finished(const UnitOut &o, int g, int rows_per_tile, unsigned int run) {
    if (o.grp_done) {
        // first level: the group's count of finished tiles (acq_rel: the group's last tile sees every
        // earlier tile's stores and its release to `done` covers them); second level: once per group
        const unsigned int old = atom_add_acqrel_gpu(&o.grp_done[o.grp], 1u);
        if (old + 1u == run * (unsigned int)o.grp_tiles) red_release_gpu_add(o.done, 1u);
    } else if (o.done) {
        red_release_gpu_add(o.done, (unsigned int)kDonePerTile);
    }
    if (o.col_cnt) notify_columns(o, g, rows_per_tile);
}

// Per-column dependency: wait (bounded) until the chunks c0 .. c1 of the dep
// task's output are complete in run `run`; `mask` caches chunks < 64 already
// seen complete (they stay complete for the rest of the run).
static __device__ __noinline__ void wait_chunks(const KParams &p, const TaskDev &T, int c0, int c1, unsigned int run,
                                                unsigned long long &mask, int task, int *status) {
    for (int c = c0; c <= c1; ++c) {
        if (c < 64 && ((mask >> c) & 1ull)) continue;
        const unsigned int target = run * T.dep_col_need[c] + p.dep_target_extra;
        if (ld_acquire_gpu(&T.dep_col_cnt[c]) - target >= 0x80000000u) {  // counter < target (wrap-safe)
            const unsigned long long t0 = globaltimer();
            for (uint32_t spin = 1;; ++spin) {
                if (ld_acquire_gpu(&T.dep_col_cnt[c]) - target < 0x80000000u) break;
                if ((spin & 31u) == 0) {
                    if (launch_failed(status)) return;
                    if (globaltimer() - t0 > p.dep_timeout_ns) {
                        record_error(status, kCodeTimeout, task, kSiteDep);
                        return;
                    }
                    __nanosleep(64);
                }
            }
        }
        if (c < 64) mask |= 1ull << c;
    }
    fence_proxy_async_global();
}

// What a task's `done` counter reaches in each run: groups with two-level readiness, else quarter tiles.
__device__ __forceinline__ unsigned int done_per_run(const TaskDev &D) {
    return (unsigned int)(D.n_groups > 1 ? D.n_groups : D.n_g * D.n_mt * kDonePerTile);
}

__device__ __forceinline__ bool dependency_met(const KParams &p, const TaskDev &D) {
    const unsigned int run = ld_acquire_gpu(&p.run_ctl[0]) + 1u;
    const unsigned int target = run * done_per_run(D) + p.dep_target_extra;
    return ld_acquire_gpu(D.done) - target < 0x80000000u;  // done >= target (wrap-safe)
}

static __device__ __noinline__ void wait_dependency(const KParams &p, const TaskDev &D, int task, int *status) {
    const unsigned int run = ld_acquire_gpu(&p.run_ctl[0]) + 1u;
    const unsigned int target = run * done_per_run(D) + p.dep_target_extra;
    if (ld_acquire_gpu(D.done) - target < 0x80000000u) {  // done >= target (wrap-safe)
        fence_proxy_async_global();
        return;
    }
    unsigned long long t0 = globaltimer();
    for (uint32_t spin = 1;; ++spin) {
        if (ld_acquire_gpu(D.done) - target < 0x80000000u) break;
        if ((spin & 31u) == 0) {
            if (launch_failed(status)) break;
            if (globaltimer() - t0 > p.dep_timeout_ns) {
                record_error(status, kCodeTimeout, task, kSiteDep);
                break;
            }
            __nanosleep(64);
        }
    }
    fence_proxy_async_global();
}

// Called by one thread per CTA after the CTA has finished all its work of a
// chain run: the last CTA (every other CTA has stopped claiming) resets the
// tasks' claim counters and advances the run counter for the next run.  If
// the run recorded an error, some CTA abandoned its work and the counters of
// this run may be left mid-count: the last CTA first sets every readiness
// counter to the value a completed run leaves (run x tiles, per group, per
// column chunk) and clears the tile arrival counters, so the next run waits
// for exactly its own work again; the sticky error words stay for the host.
__device__ __forceinline__ void chain_run_done(const KParams &p) {
    if (!p.run_ctl) return;
    const unsigned int old = atom_add_acqrel_gpu(&p.run_ctl[1], 1u);
    if (old == gridDim.x - 1) {
        const bool heal = launch_failed(p.status);
        const unsigned int run = ld_acquire_gpu(&p.run_ctl[0]) + 1u;
        for (int t = 0; t < p.n_tasks; ++t) {
            const TaskDev &T = task_at(p, t);
            st_relaxed_gpu(&T.sched[0], 0u);
            if (T.n_groups > 1)
                for (int g = 0; g < T.n_groups; ++g) st_relaxed_gpu(&T.grp_sched[g], 0u);
            if (T.die_split > 0) {
                st_relaxed_gpu(&T.die_sched[0], 0u);
                st_relaxed_gpu(&T.die_sched[1], 0u);
            }
            if (!heal) continue;
            const int tiles = T.n_g * T.n_mt;
            for (int i = 0; i < tiles; ++i) st_relaxed_gpu(&T.tile_cnt[i], 0u);
            if (T.notify) {
                if (T.n_groups > 1) {
                    for (int g = 0; g < T.n_groups; ++g)
                        st_relaxed_gpu(&T.grp_done[g], run * (unsigned int)(group_tile_lo(T, g + 1) - group_tile_lo(T, g)));
                    st_relaxed_gpu(T.done, run * (unsigned int)T.n_groups);
                } else {
                    st_relaxed_gpu(T.done, run * (unsigned int)(tiles * kDonePerTile));
                }
            }
            if (T.col_cnt) {
                const int chunks = (T.y_cols + kColChunk - 1) / kColChunk;
                for (int c = 0; c < chunks; ++c) st_relaxed_gpu(&T.col_cnt[c], run * T.col_need[c]);
            }
        }
        if (heal) st_relaxed_gpu(reinterpret_cast<unsigned int *>(&p.status[kStatusLaunchErr]), 0u);
        st_relaxed_gpu(&p.run_ctl[1], 0u);
        red_release_gpu_add(&p.run_ctl[0], 1u);
    }
}

// Trace stamps: [cta][task][kTraceSlots], the slots listed at kTraceSlots.
__device__ __forceinline__ void trace_stamp(const KParams &p, int task, int slot, unsigned long long v) {
    if (p.trace) p.trace[((size_t)blockIdx.x * p.n_tasks + task) * kTraceSlots + slot] = v;
}

#endif  // __CUDACC__

}  // namespace wsm
