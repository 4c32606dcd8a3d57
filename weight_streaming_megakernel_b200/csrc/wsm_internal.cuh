// wsm_internal.cuh -- definitions shared by the weight-streaming kernels and
// the host runtime of libwsm (not part of the public C ABI).
//
// Work decomposition (both kernel paths):
//   A GEMM is cut into tiles: `tile_rows` rows of W (outputs along N) times one
//   M-tile of X.  A tile's K range is cut into `kb` pipeline stages.  The
//   flattened list of (tile, stage) iterations, tile-major, is divided into
//   `grid` contiguous ranges of equal length, one per persistent CTA (a
//   stream-K split: every CTA streams the same number of weight bytes, so the
//   split is balanced to one stage whatever N and K are).  A tile whose stages
//   fall into several CTAs' ranges gets one fp32 partial per CTA; the CTA that
//   arrives last on the tile's counter adds the partials in CTA order (= K
//   order), so the result does not depend on arrival order.  This is the
//   inter-CTA split-K of the FlyDSL article ("AMD: ROCm Low-Latency-GEMM-Kernel
//   ... MI355X", technique 1), balanced per stage instead of per fixed factor.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace wsm {

constexpr int kMaxStages = 16;
constexpr int kUmmaRows = 128;     // rows of W per UMMA tile (MMA M)
constexpr int kUmmaBK = 64;        // K elements per UMMA stage (one 128-byte swizzle row)
constexpr int kUmmaMaxN = 64;      // largest MMA N (= X rows per tile)
constexpr int kStreamBoxK = 256;   // K elements per TMA box on the FMA path
constexpr int kStatusWords = 4;    // [0] error code, [1] failing task, [2] failing CTA, [3] site

// Error sites recorded in status[3].
enum : int { kSiteNone = 0, kSiteDep = 1, kSiteFull = 2, kSiteEmpty = 3, kSiteAcc = 4, kSiteDrain = 5 };
constexpr int kCodeTimeout = 6;    // == WSM_ERR_TIMEOUT

// One GEMM as the kernels see it.  Lives in kernel parameter space (single
// GEMM) or in a device table (chain); 64-byte aligned for the tensor maps.
struct __align__(64) TaskDev {
    CUtensorMap tmW;            // W [N, K] bf16
    CUtensorMap tmX;            // X [M, K] bf16
    __nv_bfloat16 *Y;           // [M, N]
    float *Yf32;                // optional [M, N]
    float *part;                // 2 * grid partial slots of slot_elems floats
    unsigned int *tile_cnt;     // [n_tiles] arrival counters, zero between calls
    unsigned int *done;         // tiles finished (monotonic over runs), chain only
    int M, N, K;
    int dep;                    // -1 or index of an earlier task
    int n_g;                    // column tiles along N
    int n_mt;                   // M-tiles
    int t_m;                    // X rows per M-tile
    int t_mpad;                 // X rows loaded per M-tile (UMMA: multiple of 16)
    int kb;                     // stages per tile
    int order;                  // 0: M-tile inner (M-major), 1: M-tile outer
    int notify;                 // bump `done` after each finished tile
    int w_evict_first;          // L2 policy of the weight loads
    uint32_t idesc;             // UMMA instruction descriptor (MMA N = t_mpad)
    uint32_t tx_bytes;          // bytes landing in one stage
    int slot_elems;             // floats per partial slot
    int pad_[2];
};

struct KParams {
    TaskDev single;                 // used when tasks == nullptr
    const TaskDev *tasks;           // chain table (device), or nullptr
    int n_tasks;
    int stages;                     // ring depth
    int stage_bytes;                // bytes per ring stage
    int x_off;                      // offset of the X part inside a stage
    uint32_t epoch;                 // chain run number (>= 1)
    uint32_t dep_target_extra;      // 0; a test hook makes every dependency unreachable with it
    int kps;                        // UMMA path: 64-wide K boxes per stage
    int x_stride;                   // UMMA path: bytes between the X boxes of a stage
    int pdl;                        // 0: plain launch; 1: wait for the previous kernel before any
                                    // global access; 2: stream W before that wait, X after it
    int pad2_;
    int *status;                    // kStatusWords ints
    unsigned long long dep_timeout_ns;
    unsigned long long wait_timeout_ns;
    unsigned long long *trace;      // [grid][n_tasks][3] or nullptr
};

// ------------------------------------------------------------------ schedule

// First iteration of CTA c when T iterations are split over G CTAs.
__host__ __device__ __forceinline__ long long range_lo(long long T, int c, int G) {
    return (T * (long long)c) / G;
}
// The CTA whose range holds iteration i (the largest c with range_lo(c) <= i).
__host__ __device__ __forceinline__ int cta_of(long long i, long long T, int G) {
    return (int)(((i + 1) * (long long)G - 1) / T);
}
// True when CTA c has at least one iteration (false only when T < G).
__host__ __device__ __forceinline__ bool cta_has_work(long long T, int c, int G) {
    return range_lo(T, c, G) < range_lo(T, c + 1, G);
}
// CTAs [c_first, c_last] hold the stages [tlo, thi) of one tile; returns how
// many of them have any work (all of them unless T < G).
__host__ __device__ __forceinline__ int tile_contributors(long long tlo, long long thi, long long T, int G,
                                                          int &c_first, int &c_last) {
    c_first = cta_of(tlo, T, G);
    c_last = cta_of(thi - 1, T, G);
    if (T >= G) return c_last - c_first + 1;
    int n = 0;
    for (int c = c_first; c <= c_last; ++c) n += cta_has_work(T, c, G) ? 1 : 0;
    return n;
}
// Slot of CTA c's partial for the segment starting at `seg_start`: its first
// segment uses slot 2c, its last (if different) slot 2c+1.
__host__ __device__ __forceinline__ int partial_slot(int c, long long seg_start, long long lo) {
    return 2 * c + (seg_start == lo ? 0 : 1);
}

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

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float ld_cg_f32(const float *p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// Record the first error of a launch (code, task, cta, site).
__device__ __forceinline__ void record_error(int *status, int code, int task, int site) {
    if (status && atomicCAS(status, 0, code) == 0) {
        status[1] = task;
        status[2] = (int)blockIdx.x;
        status[3] = site;
        __threadfence();
    }
}

__device__ __forceinline__ bool status_set(const int *status) {
    return status && *((volatile const int *)status) != 0;
}

// Bounded wait on an mbarrier phase.  Returns false (and records an error)
// when `limit_ns` of %globaltimer pass, or when `abort_flag` is raised.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                  unsigned long long limit_ns, int *status, int task, int site) {
    if (mbar_try(bar, parity)) return true;
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

// The slot holding contributor cj's partial of the tile whose stages start at
// tile_lo (c_first's slot is 2c+1 when the tile is its LAST segment).
__device__ __forceinline__ int contributor_slot(int cj, int c_first, int first_slot) {
    return cj == c_first ? first_slot : 2 * cj;
}

// Sum, in CTA order (= K order), of the partials of rows m0 .. m0+MB-1 (those
// below mrows) of one tile row `off` from every contributor; the loads of a
// block of CB contributors x MB rows are issued together so the reduction
// costs a few L2 round trips, not one per partial.  `sum` is written for the
// rows below mrows.
template <int MB, int CB>
__device__ __forceinline__ void ordered_partial_sums(const float *part, int slot_elems, int row_stride, int off,
                                                     int m0, int mrows, int c_first, int c_last, int first_slot,
                                                     long long T, int G, float (&sum)[MB]) {
    bool first = true;
    for (int cb = c_first; cb <= c_last; cb += CB) {
        float v[CB][MB];
        bool ok[CB];
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            const int cj = cb + u;
            ok[u] = cj <= c_last && (T >= G || cta_has_work(T, cj, G));
            const float *q = part + (size_t)contributor_slot(cj, c_first, first_slot) * slot_elems + off;
#pragma unroll
            for (int i = 0; i < MB; ++i)
                v[u][i] = (ok[u] && m0 + i < mrows) ? ld_cg_f32(q + (size_t)(m0 + i) * row_stride) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            if (ok[u]) {
#pragma unroll
                for (int i = 0; i < MB; ++i) sum[i] = first ? v[u][i] : sum[i] + v[u][i];
                first = false;
            }
        }
    }
}

// Programmatic dependent launch: let the next kernel on the stream begin its
// prologue, and wait for the previous kernel's completion (and memory).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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

// Incremental walk over a CTA's iterations [lo, hi) in tile-major order:
// (tile, k-stage kk, column tile g, M-tile mt) with no division per step.
struct IterWalk {
    int tile, kk, g, mt;
    __device__ __forceinline__ void start(const TaskDev &T, long long lo) {
        tile = (int)(lo / T.kb);
        kk = (int)(lo - (long long)tile * T.kb);
        tile_coords(T, tile, g, mt);
    }
    __device__ __forceinline__ void next(const TaskDev &T) {
        if (++kk == T.kb) {
            kk = 0;
            ++tile;
            if (T.order == 0) {
                if (++mt == T.n_mt) { mt = 0; ++g; }
            } else {
                if (++g == T.n_g) { g = 0; ++mt; }
            }
        }
    }
};

// Bounded wait for task `dep` of a chain to have finished all its tiles in
// this run.  On time-out (or an error elsewhere) records it and returns; the
// caller then proceeds with whatever X holds, so the kernel always ends.
__device__ __forceinline__ void wait_dependency(const KParams &p, const TaskDev &D, int task, int *status) {
    const unsigned int target = p.epoch * (unsigned int)(D.n_g * D.n_mt) + p.dep_target_extra;
    if (ld_acquire_gpu(D.done) - target < 0x80000000u) {  // done >= target (wrap-safe)
        fence_proxy_async_global();
        return;
    }
    unsigned long long t0 = globaltimer();
    for (uint32_t spin = 1;; ++spin) {
        if (ld_acquire_gpu(D.done) - target < 0x80000000u) break;
        if ((spin & 31u) == 0) {
            if (status_set(status)) break;
            if (globaltimer() - t0 > p.dep_timeout_ns) {
                record_error(status, kCodeTimeout, task, kSiteDep);
                break;
            }
            __nanosleep(64);
        }
    }
    fence_proxy_async_global();
}

#endif  // __CUDACC__

}  // namespace wsm
