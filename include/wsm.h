/*
 * wsm.h -- C ABI of libwsm, the weight-streaming decode GEMM library for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (every entry point below computes it):
 *
 *     Y[m, n] = sum_k X[m, k] * W[n, k]       Y = X . W^T
 *
 * with X [M, K], W [N, K] and Y [M, N] bf16, row-major and contiguous (K is
 * the contiguous dimension of X and W, N that of Y), fp32 accumulation and one
 * round-to-nearest-even of the fp32 result to bf16.  M is the decode batch
 * (1..64); K and N are in the thousands.  This is the decode-phase GEMM of
 * "AMD: ROCm Low-Latency-GEMM-Kernel beschleunigen LLM-Inferenz bis zu 1,79x
 * auf Instinct MI355X" (section "Was ist GEMM und die Decode-Phase eines
 * LLMs?"), whose cost is streaming W from HBM once per call.  The chain entry
 * runs a list of such GEMMs inside one resident kernel, the persistent
 * megakernel of "Fleet: Hierarchical Task-based Abstraction for Megakernels
 * on Multi-Die GPUs" (reading notes, sections 2a and 3d), with readiness
 * counters in place of kernel launches.
 *
 * Conventions for every entry point:
 *  - Pointers named X, W, Y, Yf32, workspace are DEVICE pointers on the
 *    current CUDA device, owned by the caller, and must stay valid until the
 *    work queued on `stream` has finished.  X, W, Y must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  All work
 *    is queued asynchronously on it; no entry point synchronises unless its
 *    comment says so.
 *  - Arguments are checked before anything is queued; a bad argument returns
 *    an error code and queues nothing.  wsm_last_error() then holds a message
 *    (per host thread).
 *  - Shapes: 1 <= M <= 64, N >= 1, K >= 8 and K % 8 == 0 (rows must be
 *    16-byte multiples for the tensor-memory-access engine).  Anything else
 *    returns WSM_ERR_UNSUPPORTED; there is no slow fallback.
 *  - Calls queued on one stream are serialised by the stream.  Calls on
 *    different streams may run concurrently: the library keeps one scratch
 *    workspace per (device, stream).  A call captured into a CUDA graph keeps
 *    the capture stream's workspace of that moment (the library never frees
 *    a workspace it has outgrown, so the graph stays valid); replay such a
 *    graph on that stream, or at least never concurrently with other calls
 *    on it.
 *  - The library never reads the values of Y before writing it.
 */
#ifndef WSM_H
#define WSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *wsm_stream_t;

typedef enum {
    WSM_OK = 0,
    WSM_ERR_INVALID = 1,     /* null pointer, negative size, bad option value */
    WSM_ERR_UNSUPPORTED = 2, /* shape outside the supported range */
    WSM_ERR_ALIGN = 3,       /* pointer not 16-byte aligned */
    WSM_ERR_NOMEM = 4,       /* device allocation failed, or caller workspace too small */
    WSM_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed (message has details) */
    WSM_ERR_TIMEOUT = 6      /* a bounded device-side wait ran out (chain dependency or pipeline) */
} wsm_status;

/* Kernel path.  AUTO takes the FMA path for M <= 2 at any size and for
 * M <= 4 up to 64 MiB of weights (measured crossovers on B200), the
 * tensor-core path otherwise; for calls with WSM_FLAG_INDEPENDENT the
 * tensor-core path from M = 3. */
enum {
    WSM_PATH_AUTO = 0,
    WSM_PATH_STREAM = 1, /* fp32 FMA dot products + warp-shuffle reduction, M <= 8 */
    WSM_PATH_UMMA = 2    /* tcgen05 MMA into tensor memory, any M (1..64) */
};

/* Order of (N-column tile, M-tile) pairs when M is split into several
 * M-tiles (UMMA path with m_tile < M).  M-major keeps the M-tiles of one
 * weight column adjacent in time so the column is fetched from HBM once and
 * re-read from L2 ("Fleet ..." reading notes, section 3f, Eq.(1)). */
enum {
    WSM_ORDER_AUTO = 0,    /* = M-major */
    WSM_ORDER_M_MAJOR = 1, /* column outer, M-tile inner */
    WSM_ORDER_NAIVE = 2    /* M-tile outer, column inner (ablation) */
};

/* L2 policy of the weight stream.  Evict-first is only right when each weight
 * byte has one reader; with several M-tiles sharing a column it would evict
 * the column before its last reader ("Fleet ..." reading notes, section 3f,
 * the bs = 64 shortfall of Eq.(1)). */
enum {
    WSM_L2_AUTO = 0,        /* evict-first when one M-tile, normal otherwise */
    WSM_L2_EVICT_FIRST = 1,
    WSM_L2_NORMAL = 2
};

/* Flags of wsm_opts / wsm_chain_opts.
 *
 * Every launch uses programmatic dependent launch: the kernel may start while
 * the kernel queued before it on the stream is finishing, and waits for it
 * (griddepcontrol.wait) before touching global memory, so stream order is
 * kept; it lets the kernel after it launch only once each of its CTAs has
 * seen that wait through.  WSM_FLAG_W_READONLY relaxes the wait for W only:
 * the caller promises that no call that may still run when this one starts
 * writes W -- the call just before it, and when that is an independent call
 * (below), every call back to and including the last one without
 * WSM_FLAG_INDEPENDENT -- and the weight stream (which is the whole cost of a
 * decode GEMM) then starts before those have finished; X, Y and the scratch
 * still wait.  WSM_FLAG_NO_PDL launches without programmatic dependent
 * launch.
 *
 * WSM_FLAG_INDEPENDENT (single calls only) goes further.  Such a call may run
 * at the same time as every call queued since the last library call without
 * the flag, that call included; the caller promises that none of those writes
 * this call's X, W or R, or reads or writes its Y or Yf32 (e.g. a q
 * projection without the flag, then k and v with it, all reading one X; or
 * back-to-back GEMMs on unrelated buffers).  The plan then takes whole tiles
 * (unless unit_stages or tail_tiles ask for split ones), CTA c runs units c,
 * c + grid, ... without claim counters or partial slots, loads and stores
 * without waiting, lets the next kernel launch at once, and waits for the
 * kernel before it only on exit (in one CTA; the others free their SMs at
 * once): every call still completes after all work queued before it, so
 * later work on the stream sees theirs.  Consecutive independent calls share
 * the GPU: with wsm_opts.grid = 0 each takes at most a quarter of the SMs,
 * in even rounds of its units (measured best on B200 for back-to-back decode
 * GEMMs of 30-200 MB); a grid given explicitly is taken as it is.  A plan
 * that splits tiles (asked for explicitly) ignores the flag.  A device-side time-out inside an independent call is kept apart
 * from the calls beside it and reported by the same status query as any
 * other call on that stream or workspace. */
enum {
    WSM_FLAG_W_READONLY = 1,
    WSM_FLAG_NO_PDL = 2,
    WSM_FLAG_INDEPENDENT = 4
};

/* Epilogue applied to the fp32 result, before its one rounding to bf16.
 * SILU_MUL is the gate+up projection of a gated MLP with the activation fused
 * ("Fleet ..." reading notes, sections 3f and 7b: gate and up concatenated into
 * one GEMM sharing one activation, SiLU fused).  W is the fused weight [N, K],
 * N = 2I a multiple of 16, holding gate and up rows interleaved in blocks of 8:
 * rows 16b .. 16b+7 are gate rows 8b .. 8b+7 and rows 16b+8 .. 16b+15 the
 * matching up rows.  The output is H [M, I]:
 *     H[m, 8b + i] = silu(G) * U,  G = (X W^T)[m, 16b + i],
 *                                  U = (X W^T)[m, 16b + 8 + i],
 * silu(z) = z / (1 + e^-z) in fp32.  RESIDUAL adds a bf16 [M, N] input R:
 * Y = X W^T + R (R may be Y itself: each element is read before it is
 * written, by the same thread). */
enum {
    WSM_EPI_NONE = 0,
    WSM_EPI_SILU_MUL = 1,
    WSM_EPI_RESIDUAL = 2
};

/* Options of skinny_gemm_ex; zero-initialised = all automatic. */
typedef struct {
    int path;        /* WSM_PATH_* */
    int m_tile;      /* UMMA path: rows of X per tile, 0 = all of M in one tile;
                        otherwise a multiple of 16 in [16, 64] */
    int order;       /* WSM_ORDER_* */
    int l2_policy;   /* WSM_L2_* */
    int grid;        /* persistent CTAs, 0 = one per SM; values above the
                        number of SMs are clamped */
    int stage_k;     /* UMMA path: K elements per pipeline stage, 0 = auto,
                        else 64, 128, 192 or 256 */
    int flags;       /* WSM_FLAG_* */
    int unit_stages; /* pipeline stages per work unit, 0 = auto (see wsm_plan_info) */
    int tail_tiles;  /* the last tail_tiles tiles of the schedule are split into
                        smaller units of tail_unit_stages stages, so the end of
                        the GEMM spreads evenly over the CTAs: 0 = auto, -1 = none */
    int tail_unit_stages; /* pipeline stages per tail unit, 0 = auto */
    int l2_prefetch_stages; /* W pipeline stages per CTA prefetched into L2 while the
                               CTA waits for the previous kernel (WSM_FLAG_W_READONLY):
                               0 = auto (4 on the tensor-core path, none on the FMA
                               path), -1 = none */
    int tile_rows;   /* W rows per tile, 0 = auto.  Tensor-core path: 128, or 256 (two
                        128-row halves share each X stage and accumulate into two
                        TMEM accumulators, so X is re-read half as often).  FMA
                        path: 16 or 32 (32: larger TMA boxes, a faster stream per
                        SM; auto takes 32 unless it leaves fewer tiles than CTAs) */
    int k_order;     /* order of a work unit's K stages: 0 = auto (increasing for a
                        single GEMM), 1 = increasing, 2 = rotated by a tile-dependent
                        offset (so CTAs that start together do not all read the same
                        columns of their weight rows at once) */
    int epilogue;    /* WSM_EPI_*; with SILU_MUL, Y (and Yf32) are [M, N/2] */
    const void *R;   /* WSM_EPI_RESIDUAL: bf16 [M, N], device */
    float *Yf32;     /* optional device [M, N] fp32: the result before rounding */
    void *workspace; /* optional caller scratch (device, >= wsm_workspace_bytes,
                        16-byte aligned, zero-filled before its first use; the
                        library leaves it in a reusable state after each call).
                        NULL = library-owned per-stream scratch. */
    size_t workspace_bytes;
} wsm_opts;

/* What the planner chose for a shape (wsm_plan). */
typedef struct {
    int path;          /* WSM_PATH_STREAM or WSM_PATH_UMMA */
    int grid;          /* persistent CTAs */
    int tile_rows;     /* rows of W (outputs along N) per tile */
    int tile_k;        /* K elements per pipeline stage */
    int m_tile;        /* X rows per tile (padded to the MMA width on UMMA) */
    int m_tiles;       /* number of M-tiles */
    int n_tiles;       /* number of N-column tiles */
    int unit_stages;   /* pipeline stages per work unit (head tiles) */
    int tail_tiles;    /* tiles split into tail units (the last ones of the schedule) */
    int tail_unit_stages; /* pipeline stages per tail unit */
    long long units;   /* work units: (n_tiles * m_tiles - tail_tiles) * ceil(k_iters / unit_stages)
                          + tail_tiles * ceil(k_iters / tail_unit_stages) */
    int k_iters;       /* pipeline stages per tile */
    int stages;        /* shared-memory ring depth */
    int order;         /* WSM_ORDER_M_MAJOR or WSM_ORDER_NAIVE */
    int l2_policy;     /* WSM_L2_EVICT_FIRST or WSM_L2_NORMAL */
    int smem_bytes;    /* dynamic shared memory per CTA */
    long long iters;   /* total stages = n_tiles * m_tiles * k_iters */
    size_t workspace_bytes;
} wsm_plan_info;

/* Y = X . W^T, automatic plan.  Device pointers; asynchronous on `stream`.
 * The decode GEMM of the FlyDSL article (section "Was ist GEMM und die
 * Decode-Phase eines LLMs?"), computed as inter-CTA split-K over work units
 * with an in-order reduction, intra-CTA K-slicing and a multi-stage shared-
 * memory pipeline (its section "Drei Techniken von FlyDSL im AITER-Framework").
 * Errors: WSM_ERR_INVALID / _UNSUPPORTED / _ALIGN for bad arguments (nothing
 * queued), WSM_ERR_NOMEM if the stream's scratch must grow and cannot (or must
 * grow during graph capture), WSM_ERR_CUDA for a failed launch.  A device-side
 * time-out is reported later by wsm_stream_status. */
wsm_status skinny_gemm(const void *X, const void *W, void *Y, int M, int N, int K,
                       wsm_stream_t stream);

/* Same with options (opts may be NULL); passages as skinny_gemm, plus the
 * Fleet reading notes' section 3f for the M-tile order and L2 policy options
 * and section 3f / 7b for the fused SiLU*mul epilogue.  With opts->workspace
 * the caller's buffer is used and nothing is allocated; a device-side time-out
 * of such a call is reported by wsm_workspace_status. */
wsm_status skinny_gemm_ex(const void *X, const void *W, void *Y, int M, int N, int K,
                          const wsm_opts *opts, wsm_stream_t stream);

/* Pure host function (no CUDA calls): the plan for a shape on a GPU with
 * `num_sms` SMs -- path, tile geometry, split of each tile's K range into work
 * units (the per-shape split factor of the FlyDSL article's split-K), ring
 * depth, L2 policy.  Used by the tests and by wsm_workspace_bytes.  Errors as
 * skinny_gemm's argument errors; `out` untouched on error. */
wsm_status wsm_plan(int M, int N, int K, int num_sms, const wsm_opts *opts,
                    wsm_plan_info *out);

/* Scratch a call with this shape needs on the current device (0 on error,
 * with wsm_last_error() set).  `opts` may be NULL: the same plan as
 * skinny_gemm. */
size_t wsm_workspace_bytes(int M, int N, int K, const wsm_opts *opts);

/* Device-side time-outs.  Every wait inside the kernels is bounded.  A wait
 * that runs out (never in a healthy run) records a sticky error in the status
 * words of the call's scratch, and the CTA that hit it abandons its work, so
 * that call's outputs are incomplete.  The counters it left mid-count are
 * repaired on the device -- a chain's by the end of the failed run, a single
 * call's by the next single call on the same scratch before it uses them --
 * so the next call on the same scratch computes correct results.  The error stays recorded until one of the status
 * queries below reads and clears it: each synchronises the stream, returns
 * WSM_ERR_TIMEOUT once per recorded time-out (*code = WSM_ERR_TIMEOUT, message
 * in wsm_last_error()) and WSM_OK (*code = 0) otherwise.  This follows the
 * Fleet reading notes' section 2 on the runtime: the megakernel fails the call
 * and leaves the retry to the framework. */

/* skinny_gemm / skinny_gemm_ex calls with the library-owned workspace queued
 * on `stream`, and skinny_gemm_noalloc calls on the current device (their
 * array is shared by all streams). */
wsm_status wsm_stream_status(wsm_stream_t stream, int *code);

/* skinny_gemm_ex calls given this caller workspace (the pointer and size
 * passed in wsm_opts).  WSM_ERR_INVALID / WSM_ERR_ALIGN for a null, misaligned
 * or too small buffer. */
wsm_status wsm_workspace_status(const void *workspace, size_t workspace_bytes, wsm_stream_t stream,
                                int *code);

/* Test hook, not for real use: each of the next `calls` launches of any entry
 * point (a hybrid chain launches one kernel per part) makes its CTA 0 wait on
 * a flag that nothing ever sets for `limit_ns` (at most 10 s), then record
 * WSM_ERR_TIMEOUT and abandon its work -- a device-side time-out on demand,
 * with no fault: every other wait stays bounded and the kernel ends.  calls =
 * 0 cancels.  WSM_ERR_INVALID for calls < 0 or a limit outside (0, 10 s]. */
wsm_status wsm_debug_stall(int calls, unsigned long long limit_ns);

/* Bytes of the fixed scratch array skinny_gemm_noalloc uses on each device. */
#define WSM_NOALLOC_SCRATCH_BYTES (16 << 20)

/* skinny_gemm for callers that cannot allocate device memory after start-up:
 * an inference loop that reserved its whole memory budget up front, a host
 * framework whose own allocator must own every device allocation, or a
 * latency-critical caller that cannot afford cudaMalloc's implicit
 * synchronisation.  (No counterpart on the pages: it is an interface choice of
 * this library, not part of the method.)  Same arguments, plan and results as
 * skinny_gemm; it never calls cudaMalloc or cudaFree.  Its scratch is one
 * array of WSM_NOALLOC_SCRATCH_BYTES in the library's device image, present
 * on every GPU that loads the library until the process exits.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Shapes whose plan needs more scratch than the array holds return
 *    WSM_ERR_UNSUPPORTED with a message naming both sizes (split-K
 *    tensor-core plans with M > 16 on the widest N, e.g. 24..64 x 57344 x
 *    8192, are the ones that do not fit).
 *  - Every call shares the array.  Each call clears the part that must start
 *    at zero (queued on `stream`), but calls that overlap on the GPU -- on
 *    different streams, or on different host threads -- race on it; queue
 *    them on one stream.
 *  - A device-side time-out is recorded in the array's status words and kept
 *    across later calls until wsm_stream_status (with this device current)
 *    reads it.
 *  - After a device reset the next call looks the array's address up again. */
wsm_status skinny_gemm_noalloc(const void *X, const void *W, void *Y, int M, int N, int K,
                               wsm_stream_t stream);

/* What the die probe found (wsm_sm_die_map). */
typedef struct {
    int num_sms;        /* SMs probed (all of the device's) */
    int dies;           /* 2 when the SMs split into two groups with distinct near lines, else 1 */
    int sms_die0;       /* SMs on die 0 (the die of the lowest SM id), */
    int sms_die1;       /* and on die 1 */
    float agreement;    /* mean fraction of probed lines on which an SM's near/far pattern agrees
                           with its die's (1 = clean split, 0.5 = no structure) */
    float near_cycles;  /* mean L2-hit latency (SM clock cycles) to lines homed on the SM's die, */
    float far_cycles;   /* and to lines homed on the other die */
} wsm_die_info;

/* Which die of the current device each SM sits on: die_of_sm[smid] = 0 or 1
 * (-1 past the last SM id), for smid < capacity; `info` may be NULL.  CUDA
 * does not expose this, so it is measured: one CTA per SM times L2 hits to a
 * set of lines; each line is nearer to the SMs of its home die, so the SMs of
 * one die agree on which lines are near (the die of SM id 0's reference
 * group is die 0).  Runs once per device (synchronous, a few ms, allocates
 * ~9 MB of device memory while it runs) and is cached.  If the SMs do not
 * split cleanly, info->dies = 1 and every SM is reported on die 0.  No
 * counterpart API on the pages; it serves the chiplet-aware grouping of the
 * Fleet reading notes (sections 3b and 3f). */
wsm_status wsm_sm_die_map(int *die_of_sm, int capacity, wsm_die_info *info);

/* ---------------------------------------------------------------- chains */

/* One GEMM of a chain.  dep = -1, or the index of an EARLIER task whose Y
 * must be complete before this task reads its X (dep < own index, so a chain
 * can never deadlock: tiles are claimed in task order).  The wait covers X
 * only: W is streamed before the dependency is met.
 *
 * dep_cols != 0 makes the dependency a data dependency per column: X must be
 * the dep task's output (same pointer, K = its output columns, same M), and
 * each pipeline stage waits only until the 256-column chunks of X it reads
 * are complete, instead of the whole dep task.  Such a task's work units are
 * ordered K-range first (the first K-range of every tile, then the second,
 * ...), so early units need only the columns the dep task finishes first. */
typedef struct {
    const void *X;
    const void *W;
    void *Y;
    int M, N, K;
    int dep;
    float *Yf32;   /* optional fp32 result, may be NULL */
    int epilogue;  /* WSM_EPI_* (as in wsm_opts) */
    const void *R; /* WSM_EPI_RESIDUAL: bf16 [M, N] */
    int dep_cols;  /* nonzero: per-column data dependency on task dep (see above) */
    int m_tile;    /* tensor-core path: X rows per tile as in wsm_opts.m_tile (0 = all of M;
                      else a multiple of 16 in [16, 64]); the FMA path takes 0 only */
} wsm_task;

typedef struct {
    int path;                  /* WSM_PATH_* for every task (AUTO: the FMA path only if AUTO
                                  picks it for every task at the chain's largest M) */
    int grid;                  /* 0 = one CTA per SM */
    unsigned long long timeout_ns; /* bound on each dependency wait, 0 = 2 s */
    int trace;                 /* nonzero: record per-CTA, per-task %globaltimer stamps
                                  (wsm_chain_trace); 1: cleared before every run (a memset queued
                                  on the stream, between this run and the previous kernel), 2:
                                  never cleared after creation, so back-to-back runs keep their
                                  programmatic overlap (a CTA that records nothing in a run keeps
                                  its earlier stamps) */
    int debug_unmet_dependency; /* test hook, 0 in real use: nonzero makes every dependency
                                   target unreachable, so each dependency wait runs out after
                                   timeout_ns and the run reports WSM_ERR_TIMEOUT */
    int flags;                 /* WSM_FLAG_* (for the whole chain) */
    int stage_k;               /* as in wsm_opts (UMMA path), 0 = auto */
    int unit_stages;           /* as in wsm_opts, for every task */
    int tail_tiles;            /* as in wsm_opts, for every task */
    int tail_unit_stages;      /* as in wsm_opts, for every task */
    int l2_prefetch_stages;    /* W stages per CTA prefetched into L2 while the CTA waits for
                                  a dependency or the previous kernel: 0 = auto (tensor-core
                                  path: 12 for a chain without dependencies whose X tiles are
                                  16 rows, 4 otherwise; FMA path: none), -1 = none */
    int counter_groups;        /* 0 or 1: one readiness counter per task, bumped by every
                                  finished tile.  G >= 2: two-level readiness ("Fleet ..."
                                  reading notes, section 3d and the two-level event
                                  synchronisation flowchart): CTA c belongs to group c % G,
                                  each task's tiles are split into G contiguous ranges, one
                                  per group, a group claims only its own range, a finished
                                  tile bumps its group's counter and the group's last tile
                                  bumps the task's counter once.  An ablation: the pages use
                                  it to save cross-die fences, which B200's coherent L2 does
                                  not need.  Not with dep_cols tasks (WSM_ERR_UNSUPPORTED). */
    int tile_rows;             /* as in wsm_opts, one value for every task; auto: tensor-core
                                  path 256 only if auto picks it for every task, FMA path the
                                  height with the lower modelled time over the tasks */
    int k_order;               /* as in wsm_opts; auto: rotated on the tensor-core path unless a
                                  task waits per column (dep_cols), increasing otherwise (on the
                                  FMA path rotation measured 4-10 % slower) */
    int dep_ring_stages;       /* W stages a CTA streams into its ring ahead of an unmet
                                  dependency: 0 = auto (1 on the tensor-core path, the whole
                                  ring on the FMA path), -1 = the whole ring */
    int kernels;               /* WSM_CHAIN_KERNELS_*: hybrid dispatch.  One kernel sizes its
                                  pipeline stages for the chain's widest X tile, which costs
                                  tasks of M <= 32 about 5 % when M > 32 tasks share the chain;
                                  SPLIT runs such a tensor-core chain as one kernel per run of
                                  consecutive tasks of one kind, back to back on the stream (a
                                  dependency on an earlier kernel is met by stream order;
                                  wsm_chain_trace is then not available), at about 20 us per
                                  extra kernel boundary.  AUTO splits when the narrow tasks'
                                  weights exceed 1.5 GB per extra boundary. */
    int cluster;               /* WSM_CHAIN_CLUSTER_*: cluster reduction.  The kernel runs as
                                  thread-block clusters of 4 CTAs; each task's first round of
                                  work units is handed out statically (unit c to CTA c) with 1, 2
                                  or 4 units per tile, so a split tile's partial sums meet inside
                                  one cluster and are added through distributed shared memory
                                  (in unit order: the same bits as the global-memory reduction of
                                  the same split) instead of round trips through L2 -- the part of
                                  a dependency boundary that dominates dependent chains.  Only
                                  clusters that the GPU keeps resident run (on B200 33 of them:
                                  132 CTAs).  It applies to tensor-core chains in which every
                                  task waits for the whole task before it.  Measured on B200 it
                                  does not pay (a 36 x 4 dependent chain at M = 16: 3.41-3.51 ms
                                  against 3.46 ms): at a dependency boundary every memory
                                  operation waits behind the memory system's load, the exchange
                                  included, and the 16 SMs left out cost as much as it saves.
                                  AUTO and OFF: never; ON: always (WSM_ERR_UNSUPPORTED where it
                                  does not apply). */
    int die_groups;            /* WSM_DIE_GROUPS_*: group the CTAs by the die their SM sits on
                                  (wsm_sm_die_map) -- the chiplet-aware scheduling of the Fleet
                                  reading notes, sections 3b and 3f.  Each task's tiles are cut
                                  into one contiguous range per die (in proportion to the die's
                                  SMs); a CTA claims the units of its own die's range first (in
                                  M-major order, so the M-tiles of a weight column are read by
                                  SMs of one die) and then helps with the other range, so no
                                  range waits for a die without CTAs.  Tensor-core path only; not
                                  with counter_groups, cluster reduction or dep_cols.  Measured on
                                  B200 (M = 32 / 64 in 16-row M-tiles): 2.2 % faster, DRAM bytes
                                  unchanged (every column is read from HBM once either way).
                                  AUTO: on for a chain with an M-tiled task (m_tile < M) when the
                                  probe finds two dies; ON: always (WSM_ERR_UNSUPPORTED where it
                                  does not apply); OFF: never.  Creating the first chain that uses
                                  it on a device runs the die probe (synchronous, a few ms). */
} wsm_chain_opts;

enum {
    WSM_DIE_GROUPS_AUTO = 0,
    WSM_DIE_GROUPS_ON = 1,
    WSM_DIE_GROUPS_OFF = 2
};

enum {
    WSM_CHAIN_CLUSTER_AUTO = 0,
    WSM_CHAIN_CLUSTER_OFF = 1,
    WSM_CHAIN_CLUSTER_ON = 2
};

enum {
    WSM_CHAIN_KERNELS_AUTO = 0,
    WSM_CHAIN_KERNELS_ONE = 1,
    WSM_CHAIN_KERNELS_SPLIT = 2
};

/* Values of wsm_opts.k_order / wsm_chain_opts.k_order. */
enum {
    WSM_K_ORDER_AUTO = 0,
    WSM_K_ORDER_INCREASING = 1,
    WSM_K_ORDER_ROTATED = 2
};

/* One task's part of a chain plan (wsm_chain_plan). */
typedef struct {
    wsm_plan_info plan;     /* the task's plan: the chain's grid and ring, its own tiles and work
                               units (workspace_bytes 0: a chain owns its scratch) */
    int kernel;             /* which of the chain's kernels runs the task, from 0 (hybrid
                               dispatch runs one kernel per run of tasks of one X width) */
    int l2_prefetch_stages; /* that kernel's settings, resolved: W stages prefetched into L2
                               while waiting (0 = none), */
    int k_order;            /* WSM_K_ORDER_INCREASING or WSM_K_ORDER_ROTATED, */
    int dep_ring_stages;    /* W stages streamed ahead of an unmet dependency (0 = the whole ring) */
    int cluster;            /* CTAs per thread-block cluster with cluster reduction, 0 without */
    int die_split;          /* die-grouped claims: first tile of the second die's range (host-only
                               planning assumes two dies of equal SM counts); 0 without */
} wsm_chain_task_info;

/* Pure host function (no CUDA calls, no memory touched): the plan
 * wsm_chain_create would make for this task list and these options on a GPU
 * with `num_sms` SMs.  The task pointers are validated (non-null, aligned,
 * dep_cols wiring) but never dereferenced, so placeholders will do.  Fills
 * out[0 .. n_tasks - 1] and *n_kernels (may be NULL).  Errors as
 * wsm_chain_create's. */
wsm_status wsm_chain_plan(const wsm_task *tasks, int n_tasks, const wsm_chain_opts *opts, int num_sms,
                          wsm_chain_task_info *out, int *n_kernels);

typedef struct wsm_chain wsm_chain;  /* opaque prepared chain */

/* Validate a task list and prepare it on the current device: device task
 * table, tensor maps, per-task scratch and readiness counters.  Validation
 * runs before any allocation and rejects null pointers (WSM_ERR_INVALID),
 * shapes outside the supported range (WSM_ERR_UNSUPPORTED), misaligned
 * pointers (WSM_ERR_ALIGN) and a dependency index outside [-1, own index)
 * (WSM_ERR_INVALID: forward and self dependencies could deadlock).  A
 * dependency does not have to be a data dependency; it may order tasks only.
 * The task array is copied; the caller may free it on return. */
wsm_status wsm_chain_create(const wsm_task *tasks, int n_tasks, const wsm_chain_opts *opts,
                            wsm_chain **out);

/* Run a prepared chain as ONE persistent kernel on `stream`. */
wsm_status wsm_chain_run(wsm_chain *chain, wsm_stream_t stream);

/* Synchronise `stream`, then report the device-side status of the chain's
 * runs since the last check: WSM_OK, or WSM_ERR_TIMEOUT with *failed_task =
 * the task whose wait ran out first (-1 when the wait was not a task's; may be
 * NULL), clearing the record (see "Device-side time-outs" above). */
wsm_status wsm_chain_status(wsm_chain *chain, wsm_stream_t stream, int *failed_task);

/* The plan of task `task` of a prepared chain (the chain's grid, ring and
 * work units; workspace_bytes is 0: the chain owns its scratch).  A chain
 * sizes each task's automatic work units for the work that can overlap them:
 * tasks followed, before the next dependency wait, by much more work get
 * longer units (whole tiles when there is enough), the rest the single-call
 * choice.  WSM_ERR_INVALID for a null chain or a task out of range. */
wsm_status wsm_chain_task_plan(wsm_chain *chain, int task, wsm_plan_info *out);

/* Copy the trace of the last run (trace != 0 at create) into host `out`:
 * stamps[cta][task][8] = {first stage issued, dependency met, last unit's
 * outputs written, SM the CTA ran on, last unit's accumulator handed to the
 * epilogue, its split-K arrival counted, its in-order reduction done (the
 * tile's last arriver only), first stage of the task complete at the MMA
 * issuer} -- %globaltimer nanoseconds except the SM id, 0 where the CTA had
 * no such event for the task; the tensor-core path records all eight, the
 * FMA path the first four.  `capacity` is the number of uint64 slots in
 * `out`; returns the number needed (grid * n_tasks * 8), or 0 when tracing
 * was not enabled.  Synchronises `stream`. */
size_t wsm_chain_trace(wsm_chain *chain, wsm_stream_t stream, unsigned long long *out,
                       size_t capacity);

/* Free a prepared chain (synchronises the device). */
void wsm_chain_destroy(wsm_chain *chain);

/* One-shot: validate, prepare (cached by the task list's contents, per
 * device) and run the chain on `stream`.  Equivalent to create + run.
 *  - Every call with the same list runs the same prepared chain, whose
 *    readiness counters and scratch are its own: queue such calls on one
 *    stream (runs that overlap on the GPU race on the counters).
 *  - A list is prepared on its first call, which must not be made during
 *    stream capture (WSM_ERR_INVALID; run it once before capturing).  A chain
 *    that ran during a capture stays prepared for the life of the process,
 *    so the graph stays valid; up to 16 others are kept, then dropped
 *    together (dropping synchronises the device). */
wsm_status gemm_chain(const wsm_task *tasks, int n_tasks, wsm_stream_t stream);

/* Synchronise `stream`, then report whether a gemm_chain run on the current
 * device recorded a device-side time-out since the last check: WSM_OK, or
 * WSM_ERR_TIMEOUT with *failed_task = the waiting task's index in its list
 * (-1 when not a task's wait; may be NULL), clearing the record.  Runs still
 * queued on other streams are not waited for. */
wsm_status gemm_chain_status(wsm_stream_t stream, int *failed_task);

/* Validation only (pure host function, no CUDA calls). */
wsm_status wsm_chain_validate(const wsm_task *tasks, int n_tasks);

/* ---------------------------------------------------------------- misc */

/* Message of the last error on this host thread ("" when none). */
const char *wsm_last_error(void);

/* ABI version of this header (bumped on any incompatible change). */
int wsm_abi_version(void);

#define WSM_ABI_VERSION 2

#ifdef __cplusplus
}
#endif

#endif /* WSM_H */
