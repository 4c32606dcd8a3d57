// wsm_api.cu -- host runtime and C ABI of libwsm (declared in include/wsm.h).
//
// Responsibilities: argument checks (before anything is queued), the plan
// (kernel path, tile geometry, ring depth, L2 policy), TMA tensor maps, the
// per-(device, stream) scratch workspace, chain preparation (device task
// table, per-task partial slots and readiness counters) and kernel launches.
#include "wsm_internal.cuh"
#include "../../include/wsm.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

namespace wsm {

const void *umma_kernel_ptr(bool chain, bool ext);       // wsm_umma.cu
const void *stream_kernel_ptr(int mmax, int tile_rows);  // wsm_stream.cu
void *noalloc_scratch_ptr(int dev);                      // wsm_noalloc.cu: nullptr until set up on `dev`
wsm_status die_map_of_device(int dev, const std::vector<int> **die, wsm_die_info *info);  // wsm_die.cu

namespace {

thread_local std::string g_err;

wsm_status fail(wsm_status code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

wsm_status cuda_fail(cudaError_t e, const char *what) {
    return fail(WSM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define WSM_CUDA(call)                                      \
    do {                                                    \
        cudaError_t e_ = (call);                            \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
    } while (0)

std::mutex g_mu;

// sm_100 opt-in limit of dynamic + static shared memory per block.
constexpr int kSmemOptin = 232448;
constexpr int kRingBudget = kSmemOptin - 8192;  // static shared memory + 1 KB alignment slack
constexpr int kStaticSmemMax = 2048;            // bound on the kernels' static shared memory (ptxas: 1 KB)
// Clusters of kClusterCtas CTAs resident at once, per 148 SMs, at one CTA per SM: measured on B200
// (cudaOccupancyMaxActiveClusters: 33, i.e. 132 CTAs; clusters never straddle a GPC, so some SMs stay
// out).  Used only to model the grid of a cluster chain in host-only planning (wsm_chain_plan); chain
// creation asks the device.
constexpr int kClustersPer148Sms = 33;

// Exchange buffer of a cluster-reduction chain: the quadrant rows of up to three senders, each lane's row
// the widest X tile's values plus 4 floats (the row's flag and padding; see the kernel).
int xbuf_bytes_of(int t_mpad) { return 3 * 32 * (t_mpad + 4) * 4; }

// W stages per waiting CTA prefetched into L2 (auto).  Measured on B200: 4
// stages gain ~4 % on a dependent layer chain and 1-4 % on back-to-back
// tensor-core launches (8-16 lose up to 10 % there); on the FMA path the
// prefetch costs 1-8 %, so none.  A chain without dependencies waits only at
// its start, for the previous kernel: with X tiles of 16 rows 12 stages beat
// 4 by ~1 % (the decode step of 20 GEMMs 304.3 -> 301.3 us, the K = 7168 /
// 8192 set 635 -> 629 us), with wider X tiles 4 stay best (the M = 32 / 64
// set 127 us against 129-132 us with 8-16).
constexpr int kDefaultPrefetchStagesUmma = 4;
constexpr int kDefaultPrefetchStagesIndependentChain = 12;
constexpr unsigned long long kDefaultDepTimeoutNs = 2000000000ull;
constexpr unsigned long long kPipeTimeoutNs = 4000000000ull;

// ------------------------------------------------------------------ geometry

struct Geo {
    int path = 0;
    int mmax = 0;              // stream path register width (1, 2, 4, 8)
    int rw = 0, rg = 0, kw = 0;
    int tile_rows = 0;         // rows of W per tile
    int tile_k = 0;            // K per stage
    int t_m = 0, t_mpad = 0, n_mt = 1;
    int n_g = 0, kb = 0;
    int stage_bytes = 0, x_off = 0, stages = 0;
    int slot_elems = 0;
    int ku = 1, nu = 1;        // head tiles: stages per work unit, units per tile
    int ku_t = 1, nu_t = 1;    // tail tiles: the same
    int tail = 0;              // tail tiles (the last ones of the schedule)
    bool ext = false;          // tensor-core kernel with cluster reduction and die-grouped claims compiled in
    bool chain = false;        // tensor-core kernel instantiated for chain runs
    int order = WSM_ORDER_M_MAJOR;
    int l2 = WSM_L2_EVICT_FIRST;
    int grid = 0;
    int threads = 0;
    int kps = 1;               // UMMA: 64-wide K boxes per stage
    int x_stride = 0;          // UMMA: bytes between X boxes inside a stage
    int wide = 0;              // UMMA: tiles of 2 x 128 W rows sharing each X stage
    long long iters() const { return (long long)n_g * n_mt * kb; }
    long long tiles() const { return (long long)n_g * n_mt; }
    long long units() const { return (tiles() - tail) * nu + (long long)tail * nu_t; }
    bool split() const { return nu > 1 || (tail > 0 && nu_t > 1); }
};

// l2_prefetch_stages option -> stages (0 = auto, -1 = none); -2 = invalid
int prefetch_stages_of(int v, int path) {
    if (v < -1) return -2;
    if (v == 0) return path == WSM_PATH_UMMA ? kDefaultPrefetchStagesUmma : 0;
    return v < 0 ? 0 : v;
}

int pow2ceil(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

bool shape_ok(int M, int N, int K) { return M >= 1 && M <= 64 && N >= 1 && K >= 8 && (K % 8) == 0; }

// Stream (FMA) geometry per register width and tile height (16 or 32 rows:
// 8 rows per warp, 8 consumer warps as 2 x 4 or 4 x 2); see wsm_stream.cu.
void stream_geo(int mmax, Geo &g, int tile_rows) {
    g.mmax = mmax;
    g.rw = 8; g.rg = tile_rows / 8; g.kw = 8 / g.rg;
    g.tile_rows = g.rg * g.rw;                 // 16 or 32
    g.tile_k = g.kw * kStreamBoxK;             // 1024 or 512
    g.x_off = g.kw * g.tile_rows * 512;        // W part of a stage
    g.stage_bytes = g.x_off + g.kw * mmax * 512;
    g.slot_elems = g.tile_rows * mmax;
    g.threads = 32 * (1 + g.rg * g.kw);
}

// Work units: ku consecutive stages of one tile, nu units per tile.  Every
// unit costs a claim and, when its tile is split, a partial store, a tile
// counter round trip and a share of the in-order reduction; and the last
// units of a GEMM decide when it ends, with SMs that stream up to ~2x slower
// than others.  Tensor-core path: nu in 1..4 minimising a cost in stages,
// fitted to measured B200 times of the decode shapes (9 shapes at M = 8, 16,
// 32, 64; back-to-back launches; mean 1.5 % above the best split, 2.0 % with
// a threshold of 2 x CTAs, which cost gate_up 5-9 % at M = 8..32):
//   units <= 3 x CTAs:  ceil(units / CTAs) x (ku + c)           (whole rounds)
//   otherwise:          units / CTAs x (ku + c) + 2 x ku        (dynamic claims
//                                                   smooth the rounds; a tail of
//                                                   about two units remains)
// with c = 1 stage of per-unit overhead at X tiles <= 32 rows, 4 above
// (larger partials).  FMA path (consumer warps run the epilogue themselves):
// whole tiles unless there are fewer than half as many tiles as CTAs, then 2
// units per tile (measured on B200: with 32-row tiles, o at M = 1 10.2 us
// whole against 12.8 us split over 2 units -- the split's reduction costs
// more than the idle SMs; the split pays only with very few tiles).
// Tail: the last tiles of the schedule may be split into smaller units, so
// the end of a GEMM (which in a chain every dependent task waits for) is
// spread evenly over CTAs that stream at different speeds.
int auto_units_per_tile(const Geo &g, int ctas) {
    if (g.path != WSM_PATH_UMMA) return std::max(1, std::min(g.tiles() * 2 >= ctas ? 1 : 2, g.kb));
    const double G = std::max(1, ctas);
    const double c = (g.t_mpad <= 32) ? 1.0 : 4.0;
    int best = 1;
    double best_cost = 1e300;
    for (int nu = 1; nu <= std::min(4, g.kb); ++nu) {
        const int ku = (g.kb + nu - 1) / nu;
        const double units = (double)g.tiles() * ((g.kb + ku - 1) / ku);
        const double cost = units <= 3 * G ? std::ceil(units / G) * (ku + c) : units / G * (ku + c) + 2.0 * ku;
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = nu;
        }
    }
    return best;
}

// Units of a chain task whose end nothing waits for soon.  The CTAs run a
// chain's tasks back to back -- a CTA that finds no unit left in a task claims
// from the next one -- so a task's units delay the kernel only where no later
// work can fill in: at the next task that waits on a dependency, or at the end
// of the kernel.  With `later` stages of work before that point, units of up
// to later / G stages (X tiles <= 32 rows) or 2 later / G (larger X tiles,
// whose partials cost 4x more per unit) keep the kernel's end short while
// cutting split-K partials and reductions.  Measured on B200 (24 independent
// tasks of one shape, whole tiles against the single-launch choice): gate_up
// at M = 16 30.8 us per task against 33.5, qkv 8.8 against 9.1, o 6.5 against
// 7.0; at M = 64 qkv 10.0 against 12.3, o 7.5 against 9.8.  The limit, swept
// on the default decode step and the L2-reuse set (later / (d G) for d = 1..4
// and m later / G for m = 1, 2, 4): later / G is best on the first (6.33 TB/s
// against 6.23-6.28 for the others), 2 later / G on the second (5.54-5.65
// against 5.31-5.37 at later / G).  Never fewer stages per unit than the
// single-launch choice; K split evenly between a tile's units.
int chain_unit_stages(const Geo &g, int ctas, long long later) {
    const int nu0 = auto_units_per_tile(g, ctas);
    const int ku0 = (g.kb + nu0 - 1) / nu0;
    const long long cap = later * (g.t_mpad <= 32 ? 1 : 2) / std::max(1, ctas);
    if (cap <= ku0) return ku0;
    const int nu = (int)std::max<long long>(1, (g.kb + cap - 1) / cap);
    return std::max(ku0, (g.kb + nu - 1) / nu);
}

wsm_status plan_units(Geo &g, int ctas, int unit_stages, int tail_tiles, int tail_unit_stages) {
    if (unit_stages < 0) return fail(WSM_ERR_INVALID, "bad unit_stages %d", unit_stages);
    if (tail_tiles < -1) return fail(WSM_ERR_INVALID, "bad tail_tiles %d", tail_tiles);
    if (tail_unit_stages < 0) return fail(WSM_ERR_INVALID, "bad tail_unit_stages %d", tail_unit_stages);
    if (unit_stages > 0) {
        g.ku = std::min(unit_stages, g.kb);
    } else {
        const int nu = auto_units_per_tile(g, ctas);
        g.ku = (g.kb + nu - 1) / nu;
    }
    g.nu = (g.kb + g.ku - 1) / g.ku;
    long long tt = tail_tiles > 0 ? tail_tiles : 0;  // auto: no tail
    tt = std::min(tt, g.tiles());
    g.tail = (int)tt;
    g.ku_t = tail_unit_stages > 0 ? std::min(tail_unit_stages, g.kb) : std::max(1, g.ku / 4);
    if (g.tail == 0) g.ku_t = g.ku;
    g.nu_t = (g.kb + g.ku_t - 1) / g.ku_t;
    return WSM_OK;
}

// Automatic path choice.  Measured on B200 (back-to-back launches of the nine
// decode shapes, 29-896 MiB of weights, at M = 1, 2, 4): at M <= 2 the FMA
// path with the better of its two tile heights is fastest at every size (e.g.
// 896 MiB at M = 1: 138 us against 144 us on the tensor cores; 192 MiB:
// 35.8 against 39.5 us); at M = 3, 4 it wins up to about 64 MiB of weights
// (it is ALU-bound from there: 8 FMA per weight element at M = 8); the
// tensor-core path wins everywhere else.
// Independent calls (WSM_FLAG_INDEPENDENT, several running side by side on a
// quarter of the SMs each) take the tensor cores from M = 3: measured with 32
// back-to-back launches per decode shape, at M = 3-4 qkv 84-86 % of the copy
// peak against 72-75 % on the FMA path, o 78 against 69-70, gate_up 100
// against 87-88, down 96 against 90; at M <= 2 the FMA path stays ahead on
// o, qkv and down (80-99 % against 76-97).
int auto_path(int M, long long w_bytes, bool independent = false) {
    const long long MiB = 1ll << 20;
    if (M <= 2) return WSM_PATH_STREAM;
    if (independent) return WSM_PATH_UMMA;
    if (M <= 4 && w_bytes <= 64 * MiB) return WSM_PATH_STREAM;
    return WSM_PATH_UMMA;
}

// Tile height on the FMA path.  An SM streams at most ~33 GB/s with the
// 16-row tiles' 8 KB boxes and ~45 GB/s with the 32-row tiles' 16 KB boxes
// (under load; the rates fitted to the measured times), so 32 rows win unless
// they leave too few tiles: fewer than half as many as CTAs split K in two
// (~4 us for the partial sums and their reduction), and fewer tiles than CTAs
// mean more bytes per busy SM.  Cost per tile height: the longer of the HBM
// time and the busiest CTA's stream (rounds of units x unit bytes / SM rate),
// plus the split.  On the 15 measured (shape, M) cases at M = 1, 2, 4 whose
// choice it decides (o, qkv, down, 7168 x 2112 and x 4096), it lands within
// 1 % of the faster height; above them both heights have whole tiles and
// 32 rows win on the stream rate.  A chain on this path takes the height
// with the lower total over its tasks.
double fma_cost_us(int rows, int N, int K, int ctas) {
    const double sm_gbs = rows == 32 ? 45.0 : 33.0;
    const double G = std::max(1, ctas);
    const int tile_k = (8 / (rows / 8)) * kStreamBoxK;
    const long long kb = (K + tile_k - 1) / tile_k;
    const long long tiles = (N + rows - 1) / rows;
    const long long nu = tiles * 2 >= ctas ? 1 : std::min<long long>(2, kb);  // as auto_units_per_tile
    const long long ku = (kb + nu - 1) / nu;
    const double unit_bytes = (double)rows * ku * tile_k * 2;
    const double rounds = std::ceil((double)(tiles * nu) / G);
    const double us = std::max(2.0 * N * K / 6.5e6, rounds * unit_bytes / (sm_gbs * 1e3));
    return us + (nu > 1 ? 4.0 : 0.0);
}
int auto_fma_rows(int N, int K, int ctas) { return fma_cost_us(32, N, K, ctas) < fma_cost_us(16, N, K, ctas) ? 32 : 16; }

// K per pipeline stage on the tensor-core path, measured on B200 (the decode
// shapes, M = 1..64): 256 (4 boxes) everywhere except X tiles of 32 rows,
// where 256 leaves 2 stages of 80 KB in the ring and 192 (3 boxes) 3 stages of
// 60 KB, 1-4 % faster; wide tiles carry twice the W per stage, so 128.
int auto_stage_k(int t_mpad, bool wide) {
    if (wide) return 128;
    return t_mpad == 32 ? 192 : 256;
}

// Wide tiles (tensor-core path): two 128-row halves of W share each X stage,
// so X is re-read by half as many tiles.  Measured on B200 (the decode shapes
// at M = 16..64) they are slower at every shape (e.g. gate_up at M = 64:
// 54.3 us against 52.0 us; down: 52.6 against 34.8 us): twice the W per
// stage needs 128-wide stages, and the ring then holds fewer bytes in flight.
// An option (tile_rows = 256), never the automatic choice.
bool auto_wide(int t_mpad) {
    (void)t_mpad;
    return false;
}

// force_mmax: a chain's FMA kernel has one register width for all tasks.
wsm_status make_geo(int M, int N, int K, int num_sms, const wsm_opts *o, Geo &g, int force_mmax = 0) {
    if (!shape_ok(M, N, K))
        return fail(WSM_ERR_UNSUPPORTED, "unsupported shape M=%d N=%d K=%d (need 1<=M<=64, N>=1, K>=8, K%%8==0)", M,
                    N, K);
    if (num_sms < 1) return fail(WSM_ERR_INVALID, "num_sms must be positive");
    wsm_opts z{};
    if (!o) o = &z;
    int path = o->path;
    if (path < 0 || path > WSM_PATH_UMMA) return fail(WSM_ERR_INVALID, "bad path %d", path);
    if (o->order < 0 || o->order > WSM_ORDER_NAIVE) return fail(WSM_ERR_INVALID, "bad order %d", o->order);
    if (o->l2_policy < 0 || o->l2_policy > WSM_L2_NORMAL) return fail(WSM_ERR_INVALID, "bad l2_policy %d", o->l2_policy);
    if (o->grid < 0) return fail(WSM_ERR_INVALID, "bad grid %d", o->grid);
    if (o->flags & ~(WSM_FLAG_W_READONLY | WSM_FLAG_NO_PDL | WSM_FLAG_INDEPENDENT))
        return fail(WSM_ERR_INVALID, "bad flags %#x", o->flags);
    if (o->l2_prefetch_stages < -1)
        return fail(WSM_ERR_INVALID, "bad l2_prefetch_stages %d", o->l2_prefetch_stages);
    if (o->k_order < 0 || o->k_order > 2) return fail(WSM_ERR_INVALID, "bad k_order %d", o->k_order);
    if (path == WSM_PATH_AUTO) path = auto_path(M, 2ll * N * K, (o->flags & WSM_FLAG_INDEPENDENT) != 0);
    g = Geo{};
    g.path = path;
    g.grid = (o->grid > 0) ? std::min(o->grid, num_sms) : num_sms;
    g.order = (o->order == WSM_ORDER_NAIVE) ? WSM_ORDER_NAIVE : WSM_ORDER_M_MAJOR;
    if (path == WSM_PATH_STREAM) {
        if (M > 8) return fail(WSM_ERR_UNSUPPORTED, "the FMA path takes M <= 8 (M=%d)", M);
        if (o->stage_k != 0) return fail(WSM_ERR_UNSUPPORTED, "stage_k applies to the UMMA path only");
        if (o->m_tile != 0 && o->m_tile != M) return fail(WSM_ERR_UNSUPPORTED, "the FMA path has no M-tiling");
        if (o->tile_rows != 0 && o->tile_rows != 16 && o->tile_rows != 32)
            return fail(WSM_ERR_UNSUPPORTED, "tile_rows must be 0, 16 or 32 on the FMA path (got %d)", o->tile_rows);
        stream_geo(force_mmax ? force_mmax : pow2ceil(M), g,
                   o->tile_rows ? o->tile_rows : auto_fma_rows(N, K, g.grid));
        g.t_m = M;
        g.t_mpad = M;
        g.n_mt = 1;
        g.n_g = (N + g.tile_rows - 1) / g.tile_rows;
        g.kb = (K + g.tile_k - 1) / g.tile_k;
    } else {
        int tm = o->m_tile;
        if (tm == 0) {
            g.t_m = M;
            g.t_mpad = (M + 15) / 16 * 16;
        } else {
            if (tm % 16 != 0 || tm < 16 || tm > kUmmaMaxN)
                return fail(WSM_ERR_UNSUPPORTED, "m_tile must be a multiple of 16 in [16, 64] (got %d)", tm);
            g.t_m = std::min(tm, M);
            g.t_mpad = (g.t_m + 15) / 16 * 16;
        }
        g.n_mt = (M + g.t_m - 1) / g.t_m;
        if (o->tile_rows != 0 && o->tile_rows != kUmmaRows && o->tile_rows != 2 * kUmmaRows)
            return fail(WSM_ERR_UNSUPPORTED, "tile_rows must be 0, 128 or 256 on the UMMA path (got %d)", o->tile_rows);
        g.wide = (o->tile_rows == 0) ? auto_wide(g.t_mpad) : (o->tile_rows == 2 * kUmmaRows);
        int sk = o->stage_k;
        if (sk == 0) sk = auto_stage_k(g.t_mpad, g.wide);
        if (sk != 64 && sk != 128 && sk != 192 && sk != 256)
            return fail(WSM_ERR_UNSUPPORTED, "stage_k must be 64, 128, 192 or 256 on the UMMA path (got %d)", sk);
        const int halves = g.wide ? 2 : 1;
        g.kps = sk / kUmmaBK;
        g.tile_rows = halves * kUmmaRows;
        g.tile_k = sk;
        g.n_g = (N + g.tile_rows - 1) / g.tile_rows;
        g.kb = (K + g.tile_k - 1) / g.tile_k;
        g.x_stride = g.t_mpad * kUmmaBK * 2;                        // X rows x 128 B (multiple of 1024)
        g.x_off = halves * g.kps * kUmmaRows * kUmmaBK * 2;         // W boxes, 16 KB each
        g.stage_bytes = g.x_off + g.kps * g.x_stride;
        g.slot_elems = g.tile_rows * g.t_mpad;
        if (g.stage_bytes > kRingBudget)
            return fail(WSM_ERR_UNSUPPORTED, "a pipeline stage of %d bytes does not fit in shared memory (use a "
                                             "smaller stage_k with wide tiles)", g.stage_bytes);
        g.threads = 64 + 2 * 128;   // producer, MMA, two epilogue warp sets
    }
    g.stages = std::min(kMaxStages, kRingBudget / g.stage_bytes);
    // an independent call takes whole tiles unless told otherwise: no partial slots, no claims, no waits
    const int unit_stages = ((o->flags & WSM_FLAG_INDEPENDENT) && o->unit_stages == 0 && o->tail_tiles <= 0)
                                ? g.kb : o->unit_stages;
    wsm_status st = plan_units(g, g.grid, unit_stages, o->tail_tiles, o->tail_unit_stages);
    if (st != WSM_OK) return st;
    if ((o->flags & WSM_FLAG_INDEPENDENT) && o->grid == 0 && !g.split()) {
        // independent calls run side by side: at most a quarter of the SMs each, in even rounds of units
        const long long u = g.units();
        const long long q = std::max(1, num_sms / 4);
        const long long rounds = (u + q - 1) / q;
        g.grid = (int)((u + rounds - 1) / rounds);
    }
    // no more CTAs than work units
    if ((long long)g.grid > g.units()) g.grid = (int)g.units();
    if (g.l2 = o->l2_policy, g.l2 == WSM_L2_AUTO) g.l2 = (g.n_mt > 1) ? WSM_L2_NORMAL : WSM_L2_EVICT_FIRST;
    return WSM_OK;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Scratch of one GEMM: [status 256 B][tile counters][partial slots].  Where
// the counters end depends ONLY on the buffer's size (1/16 of it), never on
// the shape: a buffer reused for calls of different shapes then never finds
// one call's partial sums where another call expects zeroed counters.  Every
// completed call leaves the counters it used at zero.
struct WsLayout {
    size_t status_off = 0, cnt_off = 0, part_off = 0, total = 0;
};
WsLayout ws_layout_of(size_t bytes) {
    WsLayout L;
    L.status_off = 0;
    L.cnt_off = 256;
    const size_t rest = bytes > 256 ? bytes - 256 : 0;
    L.part_off = 256 + (rest / 16) / 256 * 256;
    L.total = bytes;
    return L;
}
// counters: [kSchedWords claim counters][one arrival counter per tile]
size_t ws_counter_bytes(const Geo &g) { return ((size_t)kSchedWords + (size_t)g.tiles()) * 4; }
size_t ws_partial_bytes(const Geo &g) { return g.split() ? (size_t)g.units() * g.slot_elems * 4 : 0; }
bool ws_fits(const Geo &g, size_t bytes) {
    if (bytes < 512) return false;
    const WsLayout L = ws_layout_of(bytes);
    return L.cnt_off + ws_counter_bytes(g) <= L.part_off && L.part_off + ws_partial_bytes(g) <= bytes;
}
size_t ws_required(const Geo &g) {
    const size_t cnt = ws_counter_bytes(g);
    const size_t parts = ws_partial_bytes(g);
    // smallest multiple of 256 that fits, from a close lower bound upwards
    size_t z = round_up(256 + std::max(16 * (cnt + 256), parts + parts / 15 + 16 * 256), 256);
    while (!ws_fits(g, z)) z += 256;
    while (z > 512 && ws_fits(g, z - 256)) z -= 256;
    return z;
}

void fill_plan_info(const Geo &g, wsm_plan_info *out) {
    out->path = g.path;
    out->grid = g.grid;
    out->tile_rows = g.tile_rows;
    out->tile_k = g.tile_k;
    out->m_tile = g.t_mpad;
    out->m_tiles = g.n_mt;
    out->n_tiles = g.n_g;
    out->unit_stages = g.ku;
    out->tail_tiles = g.tail;
    out->tail_unit_stages = g.ku_t;
    out->units = g.units();
    out->k_iters = g.kb;
    out->stages = g.stages;
    out->order = g.order;
    out->l2_policy = g.l2;
    out->smem_bytes = g.stages * g.stage_bytes + 1024;
    out->iters = g.iters();
    out->workspace_bytes = ws_required(g);
}

// ------------------------------------------------------------------ device state

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn g_encode = nullptr;

wsm_status get_encode(EncodeTiledFn *fn) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(WSM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
        g_encode = reinterpret_cast<EncodeTiledFn>(p);
    }
    *fn = g_encode;
    return WSM_OK;
}

struct DevInfo {
    int sms = 0;
    int smem_optin = 0;
    bool attr_set[16] = {};
    int cluster_ctas = -1;  // CTAs of the tensor-core kernel resident as clusters of kClusterCtas (-1: not asked)
};
std::map<int, DevInfo> g_dev;

wsm_status dev_info(int dev, DevInfo **out) {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_dev.find(dev);
    if (it == g_dev.end()) {
        DevInfo d;
        WSM_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        WSM_CUDA(cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
        int major = 0, minor = 0;
        WSM_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
        WSM_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
        if (major != 10 || minor != 0)
            return fail(WSM_ERR_UNSUPPORTED, "libwsm is built for sm_100a (B200); device %d is sm_%d%d", dev, major,
                        minor);
        it = g_dev.emplace(dev, d).first;
    }
    *out = &it->second;
    return WSM_OK;
}

// Kernel for a geometry, and its slot in DevInfo::attr_set.
const void *kernel_for(const Geo &g, int *slot) {
    if (g.path == WSM_PATH_UMMA) {
        *slot = g.chain ? (g.ext ? 12 : 11) : (g.ext ? 10 : 0);
        return umma_kernel_ptr(g.chain, g.ext);
    }
    *slot = (g.mmax == 1 ? 1 : g.mmax == 2 ? 2 : g.mmax == 4 ? 3 : 4) + (g.tile_rows == 32 ? 4 : 0);
    return stream_kernel_ptr(g.mmax, g.tile_rows);
}

wsm_status prepare_kernel(DevInfo *d, const Geo &g, const void **fn) {
    int slot = 0;
    *fn = kernel_for(g, &slot);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d->attr_set[slot]) {
        // all the shared memory a block may have, less the kernel's static part (the ring, its alignment
        // slack and, in cluster chains, the exchange buffer are dynamic)
        cudaFuncAttributes fa;
        WSM_CUDA(cudaFuncGetAttributes(&fa, *fn));
        WSM_CUDA(cudaFuncSetAttribute(*fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kSmemOptin - (int)fa.sharedSizeBytes));
        d->attr_set[slot] = true;
    }
    return WSM_OK;
}

// CTAs of the tensor-core kernel that can be resident at once as clusters of kClusterCtas (0 if none).
wsm_status cluster_ctas_of(DevInfo *d, int *out) {
    Geo g;
    g.path = WSM_PATH_UMMA;
    g.ext = true;
    g.chain = true;
    const void *fn;
    wsm_status st = prepare_kernel(d, g, &fn);
    if (st != WSM_OK) return st;
    std::lock_guard<std::mutex> lk(g_mu);
    if (d->cluster_ctas < 0) {
        cudaFuncAttributes fa;
        WSM_CUDA(cudaFuncGetAttributes(&fa, fn));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(d->sms / kClusterCtas * kClusterCtas));
        cfg.blockDim = dim3(64 + 2 * 128);
        cfg.dynamicSmemBytes = (size_t)(kSmemOptin - (int)fa.sharedSizeBytes);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kClusterCtas;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        WSM_CUDA(cudaOccupancyMaxActiveClusters(&n, fn, &cfg));
        d->cluster_ctas = n * kClusterCtas;
    }
    *out = d->cluster_ctas;
    return WSM_OK;
}

wsm_status encode_2d(CUtensorMap *map, const void *base, int rows, int cols, int box_cols, int box_rows,
                     CUtensorMapSwizzle swz) {
    EncodeTiledFn enc;
    wsm_status st = get_encode(&enc);
    if (st != WSM_OK) return st;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(WSM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for [%d x %d] box [%d x %d]", (int)r, rows, cols,
                    box_rows, box_cols);
    return WSM_OK;
}

uint32_t umma_idesc(int n) {
    uint32_t d = 0;
    d |= 1u << 4;                          // D format: f32
    d |= 1u << 7;                          // A format: bf16
    d |= 1u << 10;                         // B format: bf16
    // bits 15/16 = 0: A and B K-major
    d |= (uint32_t)(n >> 3) << 17;         // N / 8
    d |= (uint32_t)(kUmmaRows >> 4) << 24; // M / 16
    return d;
}

// Fill a TaskDev for (X, W, Y) under geometry g.
wsm_status fill_task(TaskDev &T, const Geo &g, const void *X, const void *W, void *Y, float *Yf32, int M, int N,
                     int K, int epi, const void *R) {
    memset(&T, 0, sizeof T);
    wsm_status st;
    if (g.path == WSM_PATH_UMMA) {
        if ((st = encode_2d(&T.tmW, W, N, K, kUmmaBK, kUmmaRows, CU_TENSOR_MAP_SWIZZLE_128B)) != WSM_OK) return st;
        if ((st = encode_2d(&T.tmX, X, M, K, kUmmaBK, g.t_mpad, CU_TENSOR_MAP_SWIZZLE_128B)) != WSM_OK) return st;
        T.tx_bytes = (uint32_t)(g.kps * ((g.wide ? 2 : 1) * kUmmaRows * kUmmaBK * 2 + g.t_mpad * kUmmaBK * 2));
        T.idesc = umma_idesc(g.t_mpad);
    } else {
        if ((st = encode_2d(&T.tmW, W, N, K, kStreamBoxK, g.tile_rows, CU_TENSOR_MAP_SWIZZLE_NONE)) != WSM_OK)
            return st;
        if ((st = encode_2d(&T.tmX, X, M, K, kStreamBoxK, M, CU_TENSOR_MAP_SWIZZLE_NONE)) != WSM_OK) return st;
        T.tx_bytes = (uint32_t)(g.kw * (g.tile_rows * 512 + M * 512));
    }
    T.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
    T.Yf32 = Yf32;
    T.epi = epi;
    T.y_cols = (epi == WSM_EPI_SILU_MUL) ? N / 2 : N;
    T.R = reinterpret_cast<const __nv_bfloat16 *>(R);
    T.M = M;
    T.N = N;
    T.K = K;
    T.dep = -1;
    T.n_g = g.n_g;
    T.n_mt = g.n_mt;
    T.t_m = g.t_m;
    T.t_mpad = g.t_mpad;
    T.kb = g.kb;
    T.order = (g.order == WSM_ORDER_NAIVE) ? 1 : 0;
    T.notify = 0;
    T.w_evict_first = (g.l2 == WSM_L2_EVICT_FIRST) ? 1 : 0;
    T.slot_elems = g.slot_elems;
    T.ku = g.ku;
    T.nu = g.nu;
    T.t_head = (int)(g.tiles() - g.tail);
    T.u_head = T.t_head * g.nu;
    T.ku_t = g.ku_t;
    T.nu_t = g.nu_t;
    T.n_units = (int)g.units();
    return WSM_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

wsm_status check_epilogue(int epi, const void *R, int N) {
    if (epi < WSM_EPI_NONE || epi > WSM_EPI_RESIDUAL) return fail(WSM_ERR_INVALID, "bad epilogue %d", epi);
    if (epi == WSM_EPI_SILU_MUL && N % 16 != 0)
        return fail(WSM_ERR_UNSUPPORTED, "the SiLU*mul epilogue needs N (gate + up rows) a multiple of 16, got %d", N);
    if (epi == WSM_EPI_RESIDUAL && (!R || (reinterpret_cast<uintptr_t>(R) & 1u)))
        return fail(WSM_ERR_INVALID, "the residual epilogue needs a non-null, 2-byte aligned R");
    return WSM_OK;
}

wsm_status check_ptrs(const void *X, const void *W, const void *Y, const float *Yf32) {
    if (!X || !W || !Y) return fail(WSM_ERR_INVALID, "X, W and Y must be non-null device pointers");
    if (!aligned16(X) || !aligned16(W) || !aligned16(Y))
        return fail(WSM_ERR_ALIGN, "X, W and Y must be 16-byte aligned");
    if (Yf32 && (reinterpret_cast<uintptr_t>(Yf32) & 3u)) return fail(WSM_ERR_ALIGN, "Yf32 must be 4-byte aligned");
    return WSM_OK;
}

// ------------------------------------------------------------------ per-stream workspace

struct Workspace {
    void *ptr = nullptr;
    size_t bytes = 0;
    // Buffers this workspace has outgrown.  They stay allocated until the
    // process exits: a CUDA graph captured while one of them was current still
    // points at it, and replaying that graph must not touch freed memory.  The
    // workspace at least doubles on each growth, so they hold less than the
    // current one.  Their status words are still read by wsm_stream_status:
    // calls queued before a growth record their time-outs there.
    std::vector<void *> retired;
};
std::map<std::pair<int, uintptr_t>, Workspace> g_ws;

wsm_status stream_workspace(int dev, cudaStream_t stream, const Geo &g, void **out, size_t *out_bytes) {
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace &w = g_ws[{dev, reinterpret_cast<uintptr_t>(stream)}];
    if (w.ptr && ws_fits(g, w.bytes)) {
        *out = w.ptr;
        *out_bytes = w.bytes;
        return WSM_OK;
    }
    const size_t need = std::max(ws_required(g), 2 * w.bytes);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    WSM_CUDA(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone)
        return fail(WSM_ERR_NOMEM,
                    "the stream's scratch workspace must grow to %zu bytes, which cannot happen during graph capture: "
                    "run the same call once outside capture first",
                    need);
    size_t bytes = round_up(std::max(need, (size_t)1 << 20), 256);
    void *p = nullptr;
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) return fail(WSM_ERR_NOMEM, "cudaMalloc(%zu) for the workspace failed: %s", bytes, cudaGetErrorString(e));
    if ((e = cudaMemsetAsync(p, 0, bytes, stream)) != cudaSuccess) {
        cudaFree(p);
        return cuda_fail(e, "cudaMemsetAsync(workspace)");
    }
    if (w.ptr) w.retired.push_back(w.ptr);
    w.ptr = p;
    w.bytes = bytes;
    *out = p;
    *out_bytes = bytes;
    return WSM_OK;
}

// The stall test hook (wsm_debug_stall): launches left to stall, and the stall's limit.
std::atomic<int> g_stall_calls{0};
std::atomic<unsigned long long> g_stall_ns{0};

// Called right before a launch: the stall limit for it (0 = none), consuming one stalled launch.
unsigned long long take_stall() {
    int c = g_stall_calls.load(std::memory_order_relaxed);
    while (c > 0) {
        if (g_stall_calls.compare_exchange_weak(c, c - 1)) return g_stall_ns.load();
    }
    return 0;
}

// Read the sticky error words of a status block after `stream` has drained, and clear them.  Returns the
// error code (0 = none); h receives the four words.
wsm_status read_clear_status(const void *status, cudaStream_t stream, int (&h)[kStatusWords]) {
    WSM_CUDA(cudaStreamSynchronize(stream));
    WSM_CUDA(cudaMemcpy(h, status, sizeof h, cudaMemcpyDeviceToHost));
    if (h[0] != 0) WSM_CUDA(cudaMemset(const_cast<void *>(status), 0, sizeof h));
    return WSM_OK;
}

int pdl_mode(int flags) {
    if (flags & WSM_FLAG_NO_PDL) return 0;
    return (flags & WSM_FLAG_W_READONLY) ? 2 : 1;
}

wsm_status launch(const void *fn, const Geo &g, const KParams &kp, cudaStream_t stream, bool cooperative,
                  size_t extra_smem = 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g.grid);
    cfg.blockDim = dim3((unsigned)g.threads);
    cfg.dynamicSmemBytes = (size_t)kp.stages * kp.stage_bytes + 1024 + extra_smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[3];
    int na = 0;
    if (kp.cluster) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)kp.cluster;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (cooperative) {
        attr[na].id = cudaLaunchAttributeCooperative;
        attr[na].val.cooperative = 1;
        ++na;
    }
    if (kp.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    void *args[1] = {const_cast<KParams *>(&kp)};
    WSM_CUDA(cudaLaunchKernelExC(&cfg, fn, args));
    return WSM_OK;
}

}  // namespace

// ------------------------------------------------------------------ chains

}  // namespace wsm

struct wsm_chain {
    int device = 0;
    int n = 0;
    std::vector<wsm_chain *> parts;    // hybrid dispatch: one chain per run of tasks of one kind
    std::vector<int> part_first;       // ... and the index of its first task
    wsm::Geo geo;                      // ring geometry shared by all tasks
    std::vector<wsm_task> tasks;
    std::vector<wsm::TaskDev> host_table;
    wsm::TaskDev *d_table = nullptr;
    void *d_buf = nullptr;             // status + counters + partials
    size_t buf_bytes = 0;
    int *d_status = nullptr;
    unsigned int *d_counters = nullptr;
    size_t counter_bytes = 0;
    unsigned long long *d_trace = nullptr;
    size_t trace_elems = 0;
    unsigned int *d_run_ctl = nullptr;   // [runs completed, CTAs done with the current run]
    bool needs_reset = false;
    bool any_dep = false;
    unsigned long long dep_timeout_ns = 0;
    uint32_t dep_target_extra = 0;
    int pdl = 1;
    int prefetch_stages = 0;
    int k_rotate = 0;
    int dep_ring_stages = 0;
    int cluster = 0;                   // CTAs per cluster (cluster reduction), or 0
    int xbuf_bytes = 0;                // cluster reduction: exchange buffer behind the ring
    signed char *d_sm_die = nullptr;   // die-grouped claims: SM id -> die table (inside d_buf), or nullptr
    int trace_mode = 0;                // wsm_chain_opts.trace
    std::vector<wsm::Geo> task_geo;    // each task's plan (wsm_chain_task_plan)
    const void *fn = nullptr;
};

namespace wsm {
namespace {

// gemm_chain's prepared chains, by device and task list.  A chain that ran
// while its stream was being captured is pinned: a CUDA graph points at its
// table and scratch, so it is never freed.  The others are dropped together
// when 16 of them have accumulated.
struct CachedChain {
    wsm_chain *ch = nullptr;
    bool pinned = false;
};
std::map<std::pair<int, std::string>, CachedChain> g_chain_cache;
constexpr size_t kChainCacheUnpinned = 16;

wsm_status validate_tasks(const wsm_task *tasks, int n) {
    if (!tasks || n < 1) return fail(WSM_ERR_INVALID, "task list must be non-null with n_tasks >= 1");
    for (int i = 0; i < n; ++i) {
        const wsm_task &t = tasks[i];
        if (!shape_ok(t.M, t.N, t.K))
            return fail(WSM_ERR_UNSUPPORTED, "task %d: unsupported shape M=%d N=%d K=%d", i, t.M, t.N, t.K);
        wsm_status st = check_ptrs(t.X, t.W, t.Y, t.Yf32);
        if (st != WSM_OK) return fail(st, "task %d: %s", i, g_err.c_str());
        if (t.dep < -1 || t.dep >= i)
            return fail(WSM_ERR_INVALID, "task %d: dependency %d must be -1 or an earlier task", i, t.dep);
        if ((st = check_epilogue(t.epilogue, t.R, t.N)) != WSM_OK) return fail(st, "task %d: %s", i, g_err.c_str());
        if (t.dep_cols) {
            if (t.dep < 0) return fail(WSM_ERR_INVALID, "task %d: dep_cols needs a dependency", i);
            const wsm_task &d = tasks[t.dep];
            const int d_cols = (d.epilogue == WSM_EPI_SILU_MUL) ? d.N / 2 : d.N;
            if (t.X != d.Y || t.K != d_cols || t.M != d.M)
                return fail(WSM_ERR_INVALID,
                            "task %d: dep_cols needs X = task %d's Y, K = its output columns (%d) and the same M", i,
                            t.dep, d_cols);
        }
    }
    return WSM_OK;
}

// A chain's plan, computed on the host alone (no CUDA call): kernel path,
// hybrid split, each task's geometry and work units, the shared ring and the
// chain-wide settings.  wsm_chain_create builds the device state from it;
// wsm_chain_plan reports it.
struct ChainPlan {
    int path = 0;
    std::vector<std::pair<int, int>> parts;  // hybrid dispatch: [first, end) of each kernel's tasks; empty: one kernel
    std::vector<Geo> geos;                   // one kernel: each task's plan
    Geo ring;                                // one kernel: the stage geometry all tasks share
    int grid = 0;
    int groups = 1;
    int prefetch_stages = 0, k_rotate = 0, dep_ring_stages = 0;
    int cluster = 0;     // CTAs per cluster with cluster reduction, else 0
    int xbuf_bytes = 0;  // its exchange buffer
    bool die_groups = false;  // claims grouped by die
};

// Die-grouped claims: the first tile of die 1's range, in proportion to the dies' SMs (0: not split).
int die_split_of(long long tiles, int sms_die0, int sms_die1) {
    if (tiles < 2 || sms_die0 + sms_die1 <= 0) return 0;
    const long long s = (tiles * sms_die0 + (sms_die0 + sms_die1) / 2) / (sms_die0 + sms_die1);
    return (int)std::min(tiles - 1, std::max(1ll, s));
}

// Units per tile of a task in a cluster-reduction chain: 1, 2 or 4, so the units of a tile of the static
// first round fall on the CTAs of one cluster; the same cost in pipeline stages as auto_units_per_tile
// (whole rounds of units plus a per-unit overhead), over the splits that are allowed.
int cluster_unit_stages(const Geo &g, int ctas) {
    const double G = std::max(1, ctas);
    const double c = (g.t_mpad <= 32) ? 1.0 : 4.0;
    int best_ku = g.kb;
    double best_cost = 1e300;
    for (int nu : {1, 2, 4}) {
        const int ku = (g.kb + nu - 1) / nu;
        const int nu_real = (g.kb + ku - 1) / ku;
        if (nu_real != nu) continue;
        const double units = (double)g.tiles() * nu;
        const double cost = units <= 3 * G ? std::ceil(units / G) * (ku + c) : units / G * (ku + c) + 2.0 * ku;
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best_ku = ku;
        }
    }
    return best_ku;
}

// Tasks [a, b) of a chain as a chain of their own: a dependency inside the
// range is renumbered; one on an earlier task is met by stream order (the
// earlier kernel has completed) and dropped.
std::vector<wsm_task> sub_chain(const wsm_task *tasks, int a, int b) {
    std::vector<wsm_task> sub(tasks + a, tasks + b);
    for (wsm_task &t : sub) {
        if (t.dep >= a) {
            t.dep -= a;
        } else {
            t.dep = -1;
            t.dep_cols = 0;
        }
    }
    return sub;
}

// Options of one kernel of a hybrid-dispatch chain.
wsm_chain_opts part_opts(const wsm_chain_opts &o) {
    wsm_chain_opts so = o;
    so.path = WSM_PATH_UMMA;
    so.kernels = WSM_CHAIN_KERNELS_ONE;
    return so;
}

// cluster_ctas: CTAs resident as clusters of kClusterCtas (from the device, or modelled), 0 if none.
wsm_status plan_chain(const wsm_task *tasks, int n, const wsm_chain_opts *opts, int sms, ChainPlan &cp,
                      int cluster_ctas) {
    cp = ChainPlan{};
    wsm_status st;
    if (opts->cluster < WSM_CHAIN_CLUSTER_AUTO || opts->cluster > WSM_CHAIN_CLUSTER_ON)
        return fail(WSM_ERR_INVALID, "bad cluster option %d", opts->cluster);
    if (opts->die_groups < WSM_DIE_GROUPS_AUTO || opts->die_groups > WSM_DIE_GROUPS_OFF)
        return fail(WSM_ERR_INVALID, "bad die_groups %d", opts->die_groups);
    if (opts->path < 0 || opts->path > WSM_PATH_UMMA) return fail(WSM_ERR_INVALID, "bad chain path %d", opts->path);
    if (opts->kernels < WSM_CHAIN_KERNELS_AUTO || opts->kernels > WSM_CHAIN_KERNELS_SPLIT)
        return fail(WSM_ERR_INVALID, "bad kernels option %d", opts->kernels);
    if (opts->flags & ~(WSM_FLAG_W_READONLY | WSM_FLAG_NO_PDL))
        return fail(WSM_ERR_INVALID, "bad chain flags %#x", opts->flags);
    if (opts->l2_prefetch_stages < -1)
        return fail(WSM_ERR_INVALID, "bad l2_prefetch_stages %d", opts->l2_prefetch_stages);
    if (opts->counter_groups < 0) return fail(WSM_ERR_INVALID, "bad counter_groups %d", opts->counter_groups);
    if (opts->k_order < 0 || opts->k_order > 2) return fail(WSM_ERR_INVALID, "bad k_order %d", opts->k_order);
    if (opts->dep_ring_stages < -1) return fail(WSM_ERR_INVALID, "bad dep_ring_stages %d", opts->dep_ring_stages);
    int maxM = 0, max_tile_m = 0;  // largest M, and largest X tile height (M, or the task's m_tile)
    auto tile_m = [&](int i) {
        const int tm = tasks[i].m_tile > 0 ? std::min(tasks[i].m_tile, tasks[i].M) : tasks[i].M;
        return (tm + 15) / 16 * 16;
    };
    for (int i = 0; i < n; ++i) {
        maxM = std::max(maxM, tasks[i].M);
        max_tile_m = std::max(max_tile_m, tile_m(i));
    }
    // AUTO: the FMA path only if it is the automatic choice for every task at the chain's largest M
    int path = opts->path;
    if (path == WSM_PATH_AUTO) {
        path = WSM_PATH_STREAM;
        for (int i = 0; i < n; ++i)
            if (auto_path(maxM, 2ll * tasks[i].N * tasks[i].K) != WSM_PATH_STREAM) path = WSM_PATH_UMMA;
    }
    if (path == WSM_PATH_STREAM && maxM > 8) return fail(WSM_ERR_UNSUPPORTED, "the FMA path takes M <= 8 (max M=%d)", maxM);
    cp.path = path;

    // Hybrid dispatch.  One kernel sizes its ring stages for the widest X tile: with M > 32 tasks in
    // the chain, tasks of M <= 32 get 2 stages of 96 KB instead of 3 of 72 KB, about 5 % slower
    // (measured on B200).  Split into one kernel per run of consecutive tasks of one kind, they keep
    // their own ring; each extra kernel boundary costs up to about 20 us (the next task no longer
    // overlaps the previous one's tail).  AUTO splits when the narrow tasks carry more than 1.5 GB of
    // weights per extra kernel (measured: a 1.9 GB narrow run next to one M = 64 task gains 5 % from
    // the split; 12 alternating runs of 0.3-0.4 GB lose 27 %).  A dependency that crosses kernels
    // is met by stream order.
    if (path == WSM_PATH_UMMA && opts->kernels != WSM_CHAIN_KERNELS_ONE) {
        auto wide = [&](int i) { return tile_m(i) > 32; };
        int kinds = 0, segments = 1;
        double narrow_bytes = 0;
        for (int i = 0; i < n; ++i) {
            kinds |= wide(i) ? 2 : 1;
            if (i > 0 && wide(i) != wide(i - 1)) ++segments;
            if (!wide(i)) narrow_bytes += 2.0 * tasks[i].N * (double)tasks[i].K;
        }
        const bool split = kinds == 3 && (opts->kernels == WSM_CHAIN_KERNELS_SPLIT ||
                                          narrow_bytes > 1.5e9 * (segments - 1));
        if (split) {
            for (int a = 0, b; a < n; a = b) {
                for (b = a + 1; b < n && wide(b) == wide(a); ++b) {}
                cp.parts.push_back({a, b});
            }
            return WSM_OK;
        }
    }

    const int groups = opts->counter_groups > 1 ? opts->counter_groups : 1;
    if (groups > 1)
        for (int i = 0; i < n; ++i)
            if (tasks[i].dep_cols)
                return fail(WSM_ERR_UNSUPPORTED, "task %d: two-level readiness does not combine with dep_cols", i);
    // per-task geometry; the ring is sized for the widest task
    std::vector<Geo> geos(n);
    wsm_opts to{};
    to.path = path;
    to.grid = opts->grid;
    // one stage geometry for the whole chain (the ring and the kernel's boxes per stage are shared):
    // wide tiles only if every task would take them
    bool chain_wide = false;
    if (path == WSM_PATH_UMMA) {
        if (opts->tile_rows != 0 && opts->tile_rows != kUmmaRows && opts->tile_rows != 2 * kUmmaRows)
            return fail(WSM_ERR_UNSUPPORTED, "tile_rows must be 0, 128 or 256 (got %d)", opts->tile_rows);
        chain_wide = opts->tile_rows == 2 * kUmmaRows;
        if (opts->tile_rows == 0) {
            chain_wide = true;
            for (int i = 0; i < n; ++i) chain_wide = chain_wide && auto_wide(tile_m(i));
        }
        to.tile_rows = chain_wide ? 2 * kUmmaRows : kUmmaRows;
    } else {
        // FMA path: one tile height for the chain's ring, the one with the lower modelled total over the
        // tasks (see auto_fma_rows)
        if (opts->tile_rows != 0 && opts->tile_rows != 16 && opts->tile_rows != 32)
            return fail(WSM_ERR_UNSUPPORTED, "tile_rows must be 0, 16 or 32 on the FMA path (got %d)", opts->tile_rows);
        to.tile_rows = opts->tile_rows;
        if (to.tile_rows == 0) {
            const int ctas = (opts->grid > 0) ? std::min(opts->grid, sms) : sms;
            double c16 = 0, c32 = 0;
            for (int i = 0; i < n; ++i) {
                c16 += fma_cost_us(16, tasks[i].N, tasks[i].K, ctas);
                c32 += fma_cost_us(32, tasks[i].N, tasks[i].K, ctas);
            }
            to.tile_rows = c32 < c16 ? 32 : 16;
        }
    }
    to.stage_k = (path == WSM_PATH_UMMA) ? (opts->stage_k ? opts->stage_k : auto_stage_k(max_tile_m, chain_wide))
                                          : 0;
    const int chain_mmax = (path == WSM_PATH_STREAM) ? pow2ceil(maxM) : 0;
    for (int i = 0; i < n; ++i) {
        wsm_opts ti = to;
        ti.m_tile = tasks[i].m_tile;
        if ((st = make_geo(tasks[i].M, tasks[i].N, tasks[i].K, sms, &ti, geos[i], chain_mmax)) != WSM_OK)
            return fail(st, "task %d: %s", i, g_err.c_str());
    }
    // one grid for the whole chain (make_geo clamps it per task to the task's stages)
    int chain_grid = (opts->grid > 0) ? std::min(opts->grid, sms) : sms;
    Geo ring = geos[0];
    if (path == WSM_PATH_STREAM) {
        stream_geo(pow2ceil(maxM), ring, to.tile_rows);
    } else {
        int tmp = 16;
        for (auto &g : geos) tmp = std::max(tmp, g.t_mpad);
        ring.x_stride = tmp * kUmmaBK * 2;
        ring.x_off = (ring.wide ? 2 : 1) * ring.kps * kUmmaRows * kUmmaBK * 2;
        ring.stage_bytes = ring.x_off + ring.kps * ring.x_stride;
        if (ring.stage_bytes > kRingBudget)
            return fail(WSM_ERR_UNSUPPORTED, "the chain's pipeline stage of %d bytes does not fit in shared memory",
                        ring.stage_bytes);
    }
    ring.stages = std::min(kMaxStages, kRingBudget / ring.stage_bytes);
    for (int i = 0; i < n; ++i)
        if (geos[i].kps != ring.kps || geos[i].tile_k != ring.tile_k || geos[i].wide != ring.wide)
            return fail(WSM_ERR_INVALID, "task %d: stage geometry differs from the chain's", i);  // cannot happen

    // Cluster reduction (KParams::cluster), on request: for a linear dependent chain on the tensor-core path
    // -- every task waits for the one before it, so the CTAs of a cluster meet each task's first round
    // together and a CTA's exchanges never overlap.  The split tiles of each task's static first round are
    // reduced through distributed shared memory instead of partials in L2.  Measured on B200 (36 x 4 chain
    // at M = 16, traced): the exchange itself is not what bounds a dependency boundary -- at the boundary
    // every memory operation waits behind the memory system's load (the exchange ~2 us after the last
    // accumulator instead of ~0.2 us idle, the outputs' stores ~2-3 us), so it saves ~1 us per boundary,
    // while clusters of 4 leave 16 SMs out (132 CTAs) and push qkv to a 2-way split on 96 of them: 3.41-3.51
    // ms against 3.46 ms without.  Not the default.
    {
        bool linear = n >= 2;
        for (int i = 1; i < n; ++i) linear = linear && tasks[i].dep == i - 1 && !tasks[i].dep_cols;
        const int xb = path == WSM_PATH_UMMA ? xbuf_bytes_of((ring.x_stride / (kUmmaBK * 2))) : 0;
        const bool fits =
            path == WSM_PATH_UMMA && ring.stages * ring.stage_bytes + 1024 + xb + kStaticSmemMax <= kSmemOptin;
        const int cl_grid = (opts->grid > 0 ? std::min(opts->grid, cluster_ctas) : cluster_ctas) / kClusterCtas *
                            kClusterCtas;
        // an explicit split must give every tile 1, 2 or 4 units, and there are no tail units
        bool splits_ok = opts->tail_tiles <= 0;
        for (int i = 0; i < n && splits_ok && opts->unit_stages > 0; ++i) {
            const int ku = std::min(opts->unit_stages, geos[i].kb);
            splits_ok = kClusterCtas % ((geos[i].kb + ku - 1) / ku) == 0;
        }
        const bool ok = path == WSM_PATH_UMMA && linear && groups <= 1 && !ring.wide && fits &&
                        cl_grid >= kClusterCtas && splits_ok;
        if (opts->cluster == WSM_CHAIN_CLUSTER_ON && !ok)
            return fail(WSM_ERR_UNSUPPORTED,
                        "cluster reduction needs a tensor-core chain in which every task waits for the one before "
                        "it (whole-task waits, one counter level, 128-row tiles, 1, 2 or 4 units per tile, no tail "
                        "units), an exchange buffer that fits, and room for clusters of %d CTAs",
                        kClusterCtas);
        if (ok && opts->cluster == WSM_CHAIN_CLUSTER_ON) {
            cp.cluster = kClusterCtas;
            cp.xbuf_bytes = xb;
            chain_grid = cl_grid;
        }
    }
    for (auto &g : geos) g.grid = chain_grid;
    ring.grid = chain_grid;
    // Die-grouped claims.  AUTO: for chains with an M-tiled task, where M-tiles share weight columns (the
    // case grouping is about; measured on B200 2.2 % faster at 16-row M-tiles, 0.8 % at 32), if the device
    // has two dies (cp.die_groups is cleared at chain creation when the probe finds one).
    if (opts->die_groups != WSM_DIE_GROUPS_OFF) {
        bool any_dep_cols = false, any_m_tiled = false;
        for (int i = 0; i < n; ++i) {
            any_dep_cols = any_dep_cols || tasks[i].dep_cols;
            any_m_tiled = any_m_tiled || geos[i].n_mt > 1;
        }
        const bool ok = path == WSM_PATH_UMMA && groups <= 1 && !cp.cluster && !any_dep_cols;
        if (opts->die_groups == WSM_DIE_GROUPS_ON && !ok)
            return fail(WSM_ERR_UNSUPPORTED, "die-grouped claims need the tensor-core path, one counter level, no "
                                             "cluster reduction and no dep_cols tasks");
        cp.die_groups = ok && (opts->die_groups == WSM_DIE_GROUPS_ON || any_m_tiled);
    }
    cp.prefetch_stages = prefetch_stages_of(opts->l2_prefetch_stages, path);
    if (opts->l2_prefetch_stages == 0 && path == WSM_PATH_UMMA) {
        bool deps = false;
        for (int i = 0; i < n; ++i) deps = deps || tasks[i].dep >= 0;
        if (!deps && ring.x_stride <= 16 * kUmmaBK * 2) cp.prefetch_stages = kDefaultPrefetchStagesIndependentChain;
    }
    // auto: rotated on the tensor-core path.  A chain's units are long (whole tiles where later work can
    // overlap them) and start together, and in increasing order every CTA would read the same columns
    // of its weight rows at the same time.  Measured on B200: the decode step of 20 GEMMs 308.4 ->
    // 300.3 us, the M = 32 / 64 set 133.0 -> 128.0 us, the 36 x 4 layer chain 3335 -> 3296 us, the
    // fused data chain 3474 -> 3448 us, the K = 7168 / 8192 set within 0.4 %.  Single launches keep
    // the increasing order (rotated: 0.5-2.5 % slower on 8 of 10 decode shapes).  Per-column waits
    // read their dependency's chunks in increasing order, so those chains keep it too.
    bool any_dep_cols = false;
    for (int i = 0; i < n; ++i) any_dep_cols = any_dep_cols || tasks[i].dep_cols;
    cp.k_rotate = (opts->k_order == 2 || (opts->k_order == 0 && path == WSM_PATH_UMMA && !any_dep_cols)) ? 1 : 0;
    // measured on B200 (36 x 4 dependent chain at M = 16, 4 prefetch stages): 1 stage ahead of the
    // dependency is 2 % faster than 2 and 4 % faster than the whole ring (3), and none at all is 2 %
    // slower than 1.  The FMA path keeps its whole ring (unmeasured).
    cp.dep_ring_stages = opts->dep_ring_stages > 0 ? opts->dep_ring_stages
                          : (opts->dep_ring_stages == 0 && path == WSM_PATH_UMMA) ? 1 : 0;

    // work units per task, planned for the chain's grid (K-range-first units, no tail, for a task that
    // waits per column); automatic units grow with the later work a task's units can overlap: the
    // stages of the tasks after it, up to the next one that waits on a dependency
    std::vector<long long> later(n, 0);
    for (int i = n - 2; i >= 0; --i)
        later[i] = tasks[i + 1].dep >= 0 ? 0 : later[i + 1] + geos[i + 1].tiles() * (long long)geos[i + 1].kb;
    for (int i = 0; i < n; ++i) {
        if (cp.cluster) {
            // 1, 2 or 4 units per tile, no tail units
            const int unit_stages = opts->unit_stages ? opts->unit_stages : cluster_unit_stages(geos[i], chain_grid);
            if ((st = plan_units(geos[i], chain_grid, unit_stages, -1, 0)) != WSM_OK)
                return fail(st, "task %d: %s", i, g_err.c_str());
            if (kClusterCtas % geos[i].nu != 0)
                return fail(WSM_ERR_UNSUPPORTED, "task %d: cluster reduction needs 1, 2 or 4 units per tile (%d)", i,
                            geos[i].nu);
            continue;
        }
        const bool grow = opts->unit_stages == 0 && !tasks[i].dep_cols && groups <= 1;
        const int unit_stages = grow ? chain_unit_stages(geos[i], chain_grid, later[i]) : opts->unit_stages;
        if ((st = plan_units(geos[i], chain_grid, unit_stages,
                             (tasks[i].dep_cols || groups > 1 || cp.die_groups) ? -1 : opts->tail_tiles,
                             opts->tail_unit_stages)) !=
            WSM_OK)
            return fail(st, "task %d: %s", i, g_err.c_str());
    }
    cp.geos = geos;
    cp.ring = ring;
    cp.grid = chain_grid;
    cp.groups = groups;
    return WSM_OK;
}

}  // namespace
}  // namespace wsm

namespace wsm {
// Sets the message wsm_last_error() returns on this host thread.
void set_last_error_message(const char *msg) { g_err = msg ? msg : ""; }
}  // namespace wsm

using namespace wsm;

extern "C" {

const char *wsm_last_error(void) { return g_err.c_str(); }

int wsm_abi_version(void) { return WSM_ABI_VERSION; }

wsm_status wsm_plan(int M, int N, int K, int num_sms, const wsm_opts *opts, wsm_plan_info *out) {
    if (!out) return fail(WSM_ERR_INVALID, "out must be non-null");
    Geo g;
    wsm_status st = make_geo(M, N, K, num_sms, opts, g);
    if (st != WSM_OK) return st;
    fill_plan_info(g, out);
    g_err.clear();
    return WSM_OK;
}

size_t wsm_workspace_bytes(int M, int N, int K, const wsm_opts *opts) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        fail(WSM_ERR_CUDA, "no CUDA device");
        return 0;
    }
    DevInfo *d;
    if (dev_info(dev, &d) != WSM_OK) return 0;
    Geo g;
    if (make_geo(M, N, K, d->sms, opts, g) != WSM_OK) return 0;
    return ws_required(g);
}

wsm_status skinny_gemm_ex(const void *X, const void *W, void *Y, int M, int N, int K, const wsm_opts *opts,
                          wsm_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    wsm_opts z{};
    if (!opts) opts = &z;
    wsm_status st = check_ptrs(X, W, Y, opts->Yf32);
    if (st != WSM_OK) return st;
    if ((st = check_epilogue(opts->epilogue, opts->R, N)) != WSM_OK) return st;
    if (!shape_ok(M, N, K))
        return fail(WSM_ERR_UNSUPPORTED, "unsupported shape M=%d N=%d K=%d (need 1<=M<=64, N>=1, K>=8, K%%8==0)", M,
                    N, K);
    int dev = 0;
    WSM_CUDA(cudaGetDevice(&dev));
    DevInfo *d;
    if ((st = dev_info(dev, &d)) != WSM_OK) return st;
    Geo g;
    if ((st = make_geo(M, N, K, d->sms, opts, g)) != WSM_OK) return st;
    void *ws = nullptr;
    size_t ws_bytes = 0;
    if (opts->workspace) {
        if (!ws_fits(g, opts->workspace_bytes))
            return fail(WSM_ERR_NOMEM, "caller workspace of %zu bytes is smaller than the %zu needed",
                        opts->workspace_bytes, ws_required(g));
        if (!aligned16(opts->workspace)) return fail(WSM_ERR_ALIGN, "workspace must be 16-byte aligned");
        ws = opts->workspace;
        ws_bytes = opts->workspace_bytes;
    } else if ((st = stream_workspace(dev, stream, g, &ws, &ws_bytes)) != WSM_OK) {
        return st;
    }
    const WsLayout L = ws_layout_of(ws_bytes);
    KParams kp;
    memset(&kp, 0, sizeof kp);
    if ((st = fill_task(kp.single, g, X, W, Y, opts->Yf32, M, N, K, opts->epilogue, opts->R)) != WSM_OK) return st;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    kp.single.sched = reinterpret_cast<unsigned int *>(wsb + L.cnt_off);
    kp.single.tile_cnt = kp.single.sched + kSchedWords;
    kp.single.part = reinterpret_cast<float *>(wsb + L.part_off);
    kp.cnt_words = (int)((L.part_off - L.cnt_off) / 4);
    kp.tasks = nullptr;
    kp.n_tasks = 1;
    kp.stages = g.stages;
    kp.stage_bytes = g.stage_bytes;
    kp.x_off = g.x_off;
    kp.kps = g.kps;
    kp.x_stride = g.x_stride;
    kp.wide = g.wide;
    kp.k_rotate = (opts->k_order == 2) ? 1 : 0;
    kp.pdl = pdl_mode(opts->flags);
    kp.prefetch_stages = prefetch_stages_of(opts->l2_prefetch_stages, g.path);
    // an independent call whose tiles are not split needs no scratch and no claims; split plans wait as usual
    kp.independent = (opts->flags & WSM_FLAG_INDEPENDENT) && !g.split() ? 1 : 0;
    kp.run_ctl = nullptr;
    kp.status = reinterpret_cast<int *>(wsb + L.status_off) + (kp.independent ? kIndStatusOff : 0);
    kp.dep_timeout_ns = kDefaultDepTimeoutNs;
    kp.wait_timeout_ns = kPipeTimeoutNs;
    kp.trace = nullptr;
    const void *fn;
    g.ext = g.n_mt > 1;  // M-tiled: the tensor-core kernel with the K rotation's weight-column mapping
    if ((st = prepare_kernel(d, g, &fn)) != WSM_OK) return st;
    kp.debug_stall_ns = take_stall();
    if ((st = launch(fn, g, kp, stream, false)) != WSM_OK) return st;
    return WSM_OK;
}

wsm_status skinny_gemm(const void *X, const void *W, void *Y, int M, int N, int K, wsm_stream_t stream) {
    return skinny_gemm_ex(X, W, Y, M, N, K, nullptr, stream);
}

wsm_status wsm_stream_status(wsm_stream_t stream_, int *code) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (code) *code = 0;
    int dev = 0;
    WSM_CUDA(cudaGetDevice(&dev));
    // the stream's workspace, the buffers it has outgrown (calls queued before a growth), then the no-alloc
    // array of this device
    std::vector<void *> ptrs;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_ws.find({dev, reinterpret_cast<uintptr_t>(stream)});
        if (it != g_ws.end()) {
            std::vector<void *> bufs;
            if (it->second.ptr) bufs.push_back(it->second.ptr);
            bufs.insert(bufs.end(), it->second.retired.rbegin(), it->second.retired.rend());
            for (void *b : bufs) {
                ptrs.push_back(b);
                ptrs.push_back(static_cast<int *>(b) + kIndStatusOff);  // independent calls' block
            }
        }
    }
    const size_t n_stream = ptrs.size();
    if (void *na = wsm::noalloc_scratch_ptr(dev)) ptrs.push_back(na);
    WSM_CUDA(cudaStreamSynchronize(stream));
    int first[kStatusWords] = {};
    const char *where = nullptr;
    for (size_t i = 0; i < ptrs.size(); ++i) {
        int h[kStatusWords] = {};
        wsm_status st = read_clear_status(ptrs[i], stream, h);
        if (st != WSM_OK) return st;
        if (h[0] != 0 && first[0] == 0) {
            memcpy(first, h, sizeof h);
            where = i < n_stream ? "skinny_gemm on this stream" : "skinny_gemm_noalloc on this device";
        }
    }
    if (first[0] == 0) return WSM_OK;
    if (code) *code = first[0];
    return fail(WSM_ERR_TIMEOUT, "device-side wait ran out in %s (cta %d, site %d)", where, first[2], first[3]);
}

wsm_status wsm_workspace_status(const void *workspace, size_t workspace_bytes, wsm_stream_t stream_, int *code) {
    if (code) *code = 0;
    if (!workspace) return fail(WSM_ERR_INVALID, "workspace must be non-null");
    if (!aligned16(workspace)) return fail(WSM_ERR_ALIGN, "workspace must be 16-byte aligned");
    if (workspace_bytes < 512) return fail(WSM_ERR_INVALID, "workspace of %zu bytes is too small to be one", workspace_bytes);
    int h[kStatusWords] = {};
    int hi[kStatusWords] = {};  // independent calls' block
    wsm_status st = read_clear_status(workspace, reinterpret_cast<cudaStream_t>(stream_), h);
    if (st != WSM_OK) return st;
    if ((st = read_clear_status(static_cast<const int *>(workspace) + kIndStatusOff,
                                reinterpret_cast<cudaStream_t>(stream_), hi)) != WSM_OK)
        return st;
    if (h[0] == 0) memcpy(h, hi, sizeof h);
    if (h[0] == 0) return WSM_OK;
    if (code) *code = h[0];
    return fail(WSM_ERR_TIMEOUT, "device-side wait ran out in a call on this workspace (cta %d, site %d)", h[2], h[3]);
}

wsm_status wsm_debug_stall(int calls, unsigned long long limit_ns) {
    if (calls < 0) return fail(WSM_ERR_INVALID, "calls must be >= 0 (got %d)", calls);
    if (calls > 0 && (limit_ns == 0 || limit_ns > 10000000000ull))
        return fail(WSM_ERR_INVALID, "the stall limit must be in (0, 10 s] (got %llu ns)", limit_ns);
    g_stall_ns.store(limit_ns);
    g_stall_calls.store(calls);
    g_err.clear();
    return WSM_OK;
}

wsm_status wsm_chain_validate(const wsm_task *tasks, int n_tasks) {
    wsm_status st = validate_tasks(tasks, n_tasks);
    if (st == WSM_OK) g_err.clear();
    return st;
}

wsm_status wsm_chain_plan(const wsm_task *tasks, int n, const wsm_chain_opts *opts, int num_sms,
                          wsm_chain_task_info *out, int *n_kernels) {
    if (!out) return fail(WSM_ERR_INVALID, "out must be non-null");
    wsm_status st = validate_tasks(tasks, n);
    if (st != WSM_OK) return st;
    if (num_sms < 1) return fail(WSM_ERR_INVALID, "num_sms must be positive");
    wsm_chain_opts zo{};
    if (!opts) opts = &zo;
    ChainPlan cp;
    const int model_cluster_ctas = num_sms * kClustersPer148Sms / 148 * kClusterCtas;
    if ((st = plan_chain(tasks, n, opts, num_sms, cp, model_cluster_ctas)) != WSM_OK) return st;
    auto report = [&](const ChainPlan &kp, int first, int k) {
        for (size_t i = 0; i < kp.geos.size(); ++i) {
            Geo g = kp.geos[i];
            g.stages = kp.ring.stages;
            g.stage_bytes = kp.ring.stage_bytes;
            wsm_chain_task_info &o = out[first + (int)i];
            memset(&o, 0, sizeof o);
            fill_plan_info(g, &o.plan);
            o.plan.workspace_bytes = 0;  // a chain owns its scratch
            o.kernel = k;
            o.l2_prefetch_stages = kp.prefetch_stages;
            o.k_order = kp.k_rotate ? WSM_K_ORDER_ROTATED : WSM_K_ORDER_INCREASING;
            o.dep_ring_stages = kp.dep_ring_stages;
            o.cluster = kp.cluster;
            o.die_split = kp.die_groups ? die_split_of(g.tiles(), 1, 1) : 0;
        }
    };
    if (cp.parts.empty()) {
        report(cp, 0, 0);
    } else {
        for (size_t k = 0; k < cp.parts.size(); ++k) {
            const int a = cp.parts[k].first, b = cp.parts[k].second;
            std::vector<wsm_task> sub = sub_chain(tasks, a, b);
            const wsm_chain_opts so = part_opts(*opts);
            ChainPlan sp;
            if ((st = plan_chain(sub.data(), b - a, &so, num_sms, sp, model_cluster_ctas)) != WSM_OK)
                return fail(st, "tasks %d..%d: %s", a, b - 1, g_err.c_str());
            report(sp, a, (int)k);
        }
    }
    if (n_kernels) *n_kernels = cp.parts.empty() ? 1 : (int)cp.parts.size();
    g_err.clear();
    return WSM_OK;
}

wsm_status wsm_chain_create(const wsm_task *tasks, int n, const wsm_chain_opts *opts, wsm_chain **out) {
    if (!out) return fail(WSM_ERR_INVALID, "out must be non-null");
    *out = nullptr;
    wsm_status st = validate_tasks(tasks, n);
    if (st != WSM_OK) return st;
    wsm_chain_opts zo{};
    if (!opts) opts = &zo;
    int dev = 0;
    WSM_CUDA(cudaGetDevice(&dev));
    DevInfo *d;
    if ((st = dev_info(dev, &d)) != WSM_OK) return st;
    int cluster_ctas = 0;
    if ((st = cluster_ctas_of(d, &cluster_ctas)) != WSM_OK) return st;
    ChainPlan cp;
    if ((st = plan_chain(tasks, n, opts, d->sms, cp, cluster_ctas)) != WSM_OK) return st;

    if (!cp.parts.empty()) {
        // hybrid dispatch: one chain per run of tasks of one X width, run back to back
        std::unique_ptr<wsm_chain> parent(new wsm_chain());
        parent->device = dev;
        parent->n = n;
        parent->tasks.assign(tasks, tasks + n);
        auto cleanup = [&]() {
            for (wsm_chain *c : parent->parts) wsm_chain_destroy(c);
            parent->parts.clear();
        };
        for (const auto &ab : cp.parts) {
            const int a = ab.first, b = ab.second;
            std::vector<wsm_task> sub = sub_chain(tasks, a, b);
            wsm_chain_opts so = part_opts(*opts);
            so.trace = 0;
            wsm_chain *part = nullptr;
            if ((st = wsm_chain_create(sub.data(), b - a, &so, &part)) != WSM_OK) {
                cleanup();
                return fail(st, "tasks %d..%d: %s", a, b - 1, g_err.c_str());
            }
            parent->parts.push_back(part);
            parent->part_first.push_back(a);
        }
        *out = parent.release();
        g_err.clear();
        return WSM_OK;
    }

    std::unique_ptr<wsm_chain> ch(new wsm_chain());
    ch->device = dev;
    ch->n = n;
    ch->tasks.assign(tasks, tasks + n);
    ch->dep_timeout_ns = opts->timeout_ns ? opts->timeout_ns : kDefaultDepTimeoutNs;
    ch->dep_target_extra = opts->debug_unmet_dependency ? 0x40000000u : 0u;
    ch->pdl = pdl_mode(opts->flags);
    const int groups = cp.groups;
    const int chain_grid = cp.grid;
    std::vector<Geo> &geos = cp.geos;
    const Geo &ring = cp.ring;
    ch->geo = ring;
    ch->prefetch_stages = cp.prefetch_stages;
    ch->k_rotate = cp.k_rotate;
    ch->dep_ring_stages = cp.dep_ring_stages;
    ch->cluster = cp.cluster;
    ch->xbuf_bytes = cp.xbuf_bytes;
    ch->task_geo = geos;
    for (Geo &g : ch->task_geo) {
        g.stages = ring.stages;
        g.stage_bytes = ring.stage_bytes;
    }
    // per-column readiness: a task some other task reads per column publishes one counter per
    // kColChunk output columns; col_need[c] = tiles (all M-tiles) whose outputs touch chunk c
    std::vector<char> col_producer(n, 0);
    for (int i = 0; i < n; ++i)
        if (tasks[i].dep_cols) col_producer[tasks[i].dep] = 1;
    std::vector<size_t> n_chunks(n, 0);
    std::vector<std::vector<unsigned int>> col_need(n);
    for (int i = 0; i < n; ++i) {
        if (!col_producer[i]) continue;
        const Geo &gp = geos[i];
        const bool silu = tasks[i].epilogue == WSM_EPI_SILU_MUL;
        const int y_cols = silu ? tasks[i].N / 2 : tasks[i].N;
        n_chunks[i] = (size_t)(y_cols + kColChunk - 1) / kColChunk;
        col_need[i].assign(n_chunks[i], 0u);
        for (int g = 0; g < gp.n_g; ++g) {
            int lo = g * gp.tile_rows, hi = std::min(tasks[i].N, lo + gp.tile_rows);
            if (silu) lo /= 2, hi /= 2;
            for (int c = lo / kColChunk; c <= (hi - 1) / kColChunk; ++c) col_need[i][c] += (unsigned int)gp.n_mt;
        }
    }
    // scratch: status | counters (per task: claim counters + tile counters; then done counters; then
    // column counters) | partials | column needs (constant)
    std::vector<size_t> cnt_off(n), part_off(n), col_off(n), need_off(n);
    std::vector<int> n_groups(n, 1);
    // die-grouped claims: the measured SM -> die map, and each task's split of its tiles
    const std::vector<int> *die_map = nullptr;
    std::vector<int> die_split(n, 0);
    if (cp.die_groups) {
        wsm_die_info di;
        if ((st = die_map_of_device(dev, &die_map, &di)) != WSM_OK) return st;
        if (di.dies < 2 && opts->die_groups != WSM_DIE_GROUPS_ON) cp.die_groups = false;  // nothing to group
        for (int i = 0; i < n && cp.die_groups; ++i)
            die_split[i] = die_split_of(geos[i].tiles(), di.sms_die0, di.sms_die1);
    }
    size_t ncnt = 0;
    for (int i = 0; i < n; ++i) {
        // every group needs at least one tile and one CTA
        n_groups[i] = (int)std::min<long long>(groups, std::min<long long>(geos[i].tiles(), chain_grid));
        cnt_off[i] = ncnt;
        ncnt += kSchedWords + (size_t)geos[i].tiles() + (n_groups[i] > 1 ? 2 * (size_t)n_groups[i] : 0) +
                (die_split[i] > 0 ? 2 : 0);
    }
    const size_t done_off = ncnt;
    ncnt += n;
    for (int i = 0; i < n; ++i) {
        col_off[i] = ncnt;
        ncnt += n_chunks[i];
    }
    const size_t counters_at = 256;
    ch->counter_bytes = round_up(ncnt * 4, 256);
    size_t part_at = counters_at + ch->counter_bytes;
    for (int i = 0; i < n; ++i) {
        part_off[i] = part_at;
        part_at += round_up(ws_partial_bytes(geos[i]), 256);
    }
    for (int i = 0; i < n; ++i) {
        need_off[i] = part_at;
        part_at += round_up(n_chunks[i] * 4, 256);
    }
    const size_t die_off = part_at;
    if (cp.die_groups) part_at += kMaxSmIds;
    ch->buf_bytes = part_at;
    cudaError_t e = cudaMalloc(&ch->d_buf, ch->buf_bytes);
    if (e != cudaSuccess) return fail(WSM_ERR_NOMEM, "cudaMalloc(%zu) for chain scratch failed", ch->buf_bytes);
    e = cudaMalloc(reinterpret_cast<void **>(&ch->d_table), sizeof(TaskDev) * n);
    if (e != cudaSuccess) {
        cudaFree(ch->d_buf);
        return fail(WSM_ERR_NOMEM, "cudaMalloc for the task table failed");
    }
    auto cleanup = [&]() {
        cudaFree(ch->d_buf);
        cudaFree(ch->d_table);
        if (ch->d_trace) cudaFree(ch->d_trace);
    };
    uint8_t *base = static_cast<uint8_t *>(ch->d_buf);
    ch->d_status = reinterpret_cast<int *>(base);
    ch->d_run_ctl = reinterpret_cast<unsigned int *>(base + 64);  // inside the 256-byte status block
    ch->d_counters = reinterpret_cast<unsigned int *>(base + counters_at);
    e = cudaMemset(ch->d_buf, 0, ch->buf_bytes);
    if (e != cudaSuccess) {
        cleanup();
        return cuda_fail(e, "cudaMemset(chain scratch)");
    }
    if (cp.die_groups) {
        std::vector<signed char> table(kMaxSmIds, 0);
        for (int i = 0; i < kMaxSmIds && i < (int)die_map->size(); ++i) table[i] = (*die_map)[i] == 1 ? 1 : 0;
        ch->d_sm_die = reinterpret_cast<signed char *>(base + die_off);
        e = cudaMemcpy(ch->d_sm_die, table.data(), kMaxSmIds, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            cleanup();
            return cuda_fail(e, "cudaMemcpy(SM die table)");
        }
    }
    std::vector<char> depended(n, 0);
    for (int i = 0; i < n; ++i) {
        if (tasks[i].dep >= 0) ch->any_dep = true;
        if (tasks[i].dep >= 0 && !tasks[i].dep_cols) depended[tasks[i].dep] = 1;
    }
    for (int i = 0; i < n; ++i) {
        if (!n_chunks[i]) continue;
        e = cudaMemcpy(base + need_off[i], col_need[i].data(), n_chunks[i] * 4, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            cleanup();
            return cuda_fail(e, "cudaMemcpy(column needs)");
        }
    }
    ch->host_table.resize(n);
    for (int i = 0; i < n; ++i) {
        TaskDev &T = ch->host_table[i];
        Geo gi = geos[i];
        if ((st = fill_task(T, gi, tasks[i].X, tasks[i].W, tasks[i].Y, tasks[i].Yf32, tasks[i].M, tasks[i].N,
                            tasks[i].K, tasks[i].epilogue, tasks[i].R)) != WSM_OK) {
            cleanup();
            return fail(st, "task %d: %s", i, g_err.c_str());
        }
        T.dep = tasks[i].dep;
        T.sched = ch->d_counters + cnt_off[i];
        T.tile_cnt = T.sched + kSchedWords;
        T.n_groups = n_groups[i];
        if (n_groups[i] > 1) {
            T.grp_sched = T.tile_cnt + gi.tiles();
            T.grp_done = T.grp_sched + n_groups[i];
        }
        if (die_split[i] > 0) {
            T.die_split = die_split[i];
            T.die_sched = T.tile_cnt + gi.tiles() + (n_groups[i] > 1 ? 2 * n_groups[i] : 0);
        }
        T.done = ch->d_counters + done_off + i;
        T.notify = depended[i];
        T.part = reinterpret_cast<float *>(base + part_off[i]);
        if (n_chunks[i]) {
            T.col_cnt = ch->d_counters + col_off[i];
            T.col_need = reinterpret_cast<const unsigned int *>(base + need_off[i]);
        }
    }
    for (int i = 0; i < n; ++i) {
        if (!tasks[i].dep_cols) continue;
        TaskDev &T = ch->host_table[i];
        T.k_major = 1;
        T.dep_col_cnt = ch->host_table[tasks[i].dep].col_cnt;
        T.dep_col_need = ch->host_table[tasks[i].dep].col_need;
    }
    e = cudaMemcpy(ch->d_table, ch->host_table.data(), sizeof(TaskDev) * n, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cleanup();
        return cuda_fail(e, "cudaMemcpy(task table)");
    }
    ch->trace_mode = opts->trace;
    if (opts->trace) {
        ch->trace_elems = (size_t)ring.grid * n * kTraceSlots;
        e = cudaMalloc(reinterpret_cast<void **>(&ch->d_trace), ch->trace_elems * 8);
        if (e != cudaSuccess) {
            cleanup();
            return fail(WSM_ERR_NOMEM, "cudaMalloc for the trace failed");
        }
        cudaMemset(ch->d_trace, 0, ch->trace_elems * 8);
    }
    // cluster reduction, die-grouped claims and M-tiled tasks run in the kernel instantiation that has them
    // compiled in
    bool any_m_tiled = false;
    for (int i = 0; i < n; ++i) any_m_tiled = any_m_tiled || geos[i].n_mt > 1;
    ch->geo.ext = cp.cluster != 0 || cp.die_groups || any_m_tiled;
    ch->geo.chain = true;
    if ((st = prepare_kernel(d, ch->geo, &ch->fn)) != WSM_OK) {
        cleanup();
        return st;
    }
    *out = ch.release();
    g_err.clear();
    return WSM_OK;
}

wsm_status wsm_chain_run(wsm_chain *ch, wsm_stream_t stream_) {
    if (!ch) return fail(WSM_ERR_INVALID, "chain is null");
    if (!ch->parts.empty()) {
        for (wsm_chain *part : ch->parts) {
            wsm_status st = wsm_chain_run(part, stream_);
            if (st != WSM_OK) return st;
        }
        return WSM_OK;
    }
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int dev = 0;
    WSM_CUDA(cudaGetDevice(&dev));
    if (dev != ch->device) return fail(WSM_ERR_INVALID, "chain was prepared on device %d, current is %d", ch->device, dev);
    if (ch->needs_reset) {
        WSM_CUDA(cudaMemsetAsync(ch->d_counters, 0, ch->counter_bytes, stream));
        WSM_CUDA(cudaMemsetAsync(ch->d_run_ctl, 0, 2 * sizeof(unsigned int), stream));
        ch->needs_reset = false;
    }
    if (ch->d_trace && ch->trace_mode != 2) WSM_CUDA(cudaMemsetAsync(ch->d_trace, 0, ch->trace_elems * 8, stream));
    KParams kp;
    memset(&kp, 0, sizeof kp);
    kp.tasks = ch->d_table;
    kp.n_tasks = ch->n;
    kp.stages = ch->geo.stages;
    kp.stage_bytes = ch->geo.stage_bytes;
    kp.x_off = ch->geo.x_off;
    kp.kps = ch->geo.kps;
    kp.x_stride = ch->geo.x_stride;
    kp.wide = ch->geo.wide;
    kp.k_rotate = ch->k_rotate;
    kp.dep_ring_stages = ch->dep_ring_stages;
    kp.pdl = ch->pdl;
    kp.prefetch_stages = ch->prefetch_stages;
    kp.run_ctl = ch->d_run_ctl;
    kp.dep_target_extra = ch->dep_target_extra;
    kp.status = ch->d_status;
    kp.dep_timeout_ns = ch->dep_timeout_ns;
    kp.wait_timeout_ns = ch->dep_timeout_ns + kPipeTimeoutNs;
    kp.trace = ch->d_trace;
    kp.debug_stall_ns = take_stall();
    kp.cluster = ch->cluster;
    kp.xbuf_off = ch->geo.stages * ch->geo.stage_bytes;
    kp.xrow = ch->geo.x_stride / (kUmmaBK * 2) + 4;
    kp.sm_die = ch->d_sm_die;
    return launch(ch->fn, ch->geo, kp, stream, ch->any_dep, ch->cluster ? (size_t)ch->xbuf_bytes : 0);
}

wsm_status wsm_chain_status(wsm_chain *ch, wsm_stream_t stream_, int *failed_task) {
    if (!ch) return fail(WSM_ERR_INVALID, "chain is null");
    if (!ch->parts.empty()) {
        wsm_status first = WSM_OK;
        if (failed_task) *failed_task = -1;
        for (size_t k = 0; k < ch->parts.size(); ++k) {
            int ft = -1;
            wsm_status st = wsm_chain_status(ch->parts[k], stream_, &ft);
            if (st != WSM_OK && first == WSM_OK) {
                first = st;
                if (failed_task) *failed_task = ft < 0 ? -1 : ch->part_first[k] + ft;
            }
        }
        return first;
    }
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    WSM_CUDA(cudaStreamSynchronize(stream));
    int h[kStatusWords] = {};
    WSM_CUDA(cudaMemcpy(h, ch->d_status, sizeof h, cudaMemcpyDeviceToHost));
    if (failed_task) *failed_task = -1;
    if (h[0] == 0) return WSM_OK;
    if (failed_task) *failed_task = h[1];
    WSM_CUDA(cudaMemset(ch->d_status, 0, sizeof h));
    ch->needs_reset = true;
    return fail(WSM_ERR_TIMEOUT, "chain wait ran out at task %d (cta %d, site %d)", h[1], h[2], h[3]);
}

wsm_status wsm_chain_task_plan(wsm_chain *ch, int task, wsm_plan_info *out) {
    if (!ch || !out) return fail(WSM_ERR_INVALID, "chain and out must be non-null");
    if (task < 0 || task >= ch->n) return fail(WSM_ERR_INVALID, "task %d out of range (n = %d)", task, ch->n);
    if (!ch->parts.empty()) {
        size_t k = ch->parts.size() - 1;
        while (ch->part_first[k] > task) --k;
        return wsm_chain_task_plan(ch->parts[k], task - ch->part_first[k], out);
    }
    fill_plan_info(ch->task_geo[task], out);
    out->workspace_bytes = 0;  // the chain owns its scratch
    g_err.clear();
    return WSM_OK;
}

size_t wsm_chain_trace(wsm_chain *ch, wsm_stream_t stream_, unsigned long long *out, size_t capacity) {
    if (!ch || !ch->d_trace) return 0;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (cudaStreamSynchronize(stream) != cudaSuccess) return 0;
    if (out && capacity >= ch->trace_elems) {
        if (cudaMemcpy(out, ch->d_trace, ch->trace_elems * 8, cudaMemcpyDeviceToHost) != cudaSuccess) return 0;
    }
    return ch->trace_elems;
}

void wsm_chain_destroy(wsm_chain *ch) {
    if (!ch) return;
    if (!ch->parts.empty()) {
        for (wsm_chain *part : ch->parts) wsm_chain_destroy(part);
        delete ch;
        return;
    }
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(ch->device);
    cudaDeviceSynchronize();
    cudaFree(ch->d_buf);
    cudaFree(ch->d_table);
    if (ch->d_trace) cudaFree(ch->d_trace);
    cudaSetDevice(prev);
    delete ch;
}

wsm_status gemm_chain(const wsm_task *tasks, int n_tasks, wsm_stream_t stream) {
    wsm_status st = validate_tasks(tasks, n_tasks);
    if (st != WSM_OK) return st;
    int dev = 0;
    WSM_CUDA(cudaGetDevice(&dev));
    // cache key from the fields (not the raw struct bytes, whose padding a caller may leave unset)
    std::string key;
    for (int i = 0; i < n_tasks; ++i) {
        const wsm_task &t = tasks[i];
        const uintptr_t f[] = {reinterpret_cast<uintptr_t>(t.X), reinterpret_cast<uintptr_t>(t.W),
                               reinterpret_cast<uintptr_t>(t.Y), reinterpret_cast<uintptr_t>(t.Yf32),
                               reinterpret_cast<uintptr_t>(t.R), (uintptr_t)(uint32_t)t.M, (uintptr_t)(uint32_t)t.N,
                               (uintptr_t)(uint32_t)t.K, (uintptr_t)(uint32_t)t.dep, (uintptr_t)(uint32_t)t.epilogue,
                               (uintptr_t)(t.dep_cols != 0), (uintptr_t)(uint32_t)t.m_tile};
        key.append(reinterpret_cast<const char *>(f), sizeof f);
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    WSM_CUDA(cudaStreamIsCapturing(s, &cs));
    const bool capturing = cs != cudaStreamCaptureStatusNone;
    // a cached chain is run under the lock, so no other thread can drop it in between (a run only
    // queues work and takes no lock itself)
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_chain_cache.find({dev, key});
        if (it != g_chain_cache.end()) {
            if (capturing) it->second.pinned = true;
            return wsm_chain_run(it->second.ch, stream);
        }
    }
    if (capturing)
        return fail(WSM_ERR_INVALID, "gemm_chain: this task list is not prepared yet and cannot be prepared during "
                                     "stream capture: run it once outside capture first (or use wsm_chain_create)");
    wsm_chain *ch = nullptr;
    if ((st = wsm_chain_create(tasks, n_tasks, nullptr, &ch)) != WSM_OK) return st;
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_chain_cache.find({dev, key});
    if (it != g_chain_cache.end()) {  // another thread prepared the same list meanwhile
        wsm_chain_destroy(ch);
        return wsm_chain_run(it->second.ch, stream);
    }
    size_t unpinned = 0;
    for (auto &kv : g_chain_cache) unpinned += kv.second.pinned ? 0 : 1;
    if (unpinned >= kChainCacheUnpinned) {
        // bounded cache: drop the unpinned chains (rare; a prepared chain is cheap to rebuild)
        for (auto i = g_chain_cache.begin(); i != g_chain_cache.end();) {
            if (i->second.pinned) {
                ++i;
                continue;
            }
            wsm_chain_destroy(i->second.ch);
            i = g_chain_cache.erase(i);
        }
    }
    g_chain_cache[{dev, key}] = CachedChain{ch, false};
    return wsm_chain_run(ch, stream);
}

wsm_status gemm_chain_status(wsm_stream_t stream, int *failed_task) {
    if (failed_task) *failed_task = -1;
    int dev = 0;
    WSM_CUDA(cudaGetDevice(&dev));
    WSM_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
    wsm_status first = WSM_OK;
    std::string msg;
    // under the lock: no other thread drops a cached chain meanwhile
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto &kv : g_chain_cache) {
        if (kv.first.first != dev) continue;
        int ft = -1;
        const wsm_status st = wsm_chain_status(kv.second.ch, stream, &ft);
        if (st != WSM_OK && first == WSM_OK) {
            first = st;
            msg = g_err;
            if (failed_task) *failed_task = ft;
        }
    }
    if (first != WSM_OK) return fail(first, "gemm_chain: %s", msg.c_str());
    g_err.clear();
    return WSM_OK;
}

}  // extern "C"
