"""gemm_chain: one persistent kernel runs a list of GEMMs with readiness
counters.  Checked against the per-task oracle: a data-dependent chain (task
t reads task t-1's Y, so a counter that fails to order them gives a wrong
result, not an invisible race), independent tasks at the real layer shapes,
both kernel paths, repeated runs (epoch counters), the bounded dependency
wait (a target nothing reaches must end in WSM_ERR_TIMEOUT, not a hang), the
trace stamps, and the one-shot entry point."""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_streaming_megakernel_b200 as wsm
from parity import check_full, check_sampled

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def dependent_chain(M, dims, seed=0):
    """Task t: Y_t = Y_{t-1} . W_t^T with W_t [dims[t+1], dims[t]]."""
    x0 = synth.make_x(M, dims[0], seed).to(DEV)
    ws = [synth.make_w(dims[t + 1], dims[t], 1000 + seed + t).to(DEV) for t in range(len(dims) - 1)]
    ys = [torch.full((M, dims[t + 1]), float("nan"), dtype=torch.bfloat16, device=DEV) for t in range(len(ws))]
    yfs = [torch.empty(M, dims[t + 1], dtype=torch.float32, device=DEV) for t in range(len(ws))]
    tasks = []
    for t in range(len(ws)):
        x = x0 if t == 0 else ys[t - 1]
        tasks.append(wsm.Task(x, ws[t], ys[t], dep=t - 1, yf32=yfs[t]))
    return x0, ws, ys, yfs, tasks


def check_dependent(x0, ws, ys, yfs):
    x = x0
    for t in range(len(ws)):
        # each task against the oracle on the GPU's own input, so errors do not compound
        check_full(x.cpu(), ws[t].cpu(), ys[t], yfs[t], what=f"task {t}")
        x = ys[t]


@pytest.mark.parametrize("path,M,k_order", [(wsm.PATH_UMMA, 16, 0), (wsm.PATH_UMMA, 16, 1), (wsm.PATH_UMMA, 64, 0),
                                            (wsm.PATH_UMMA, 64, 1), (wsm.PATH_STREAM, 4, 0), (wsm.PATH_STREAM, 1, 0),
                                            (wsm.PATH_STREAM, 4, 2)])
def test_dependent_chain(path, M, k_order):
    """Data-dependent chain (task t reads task t - 1's output), in both K
    orders (auto: rotated on the tensor-core path, increasing on the FMA
    path)."""
    dims = [1024, 2048, 1024, 3072, 512, 1024, 4096, 1024]
    x0, ws, ys, yfs, tasks = dependent_chain(M, dims, seed=M)
    ch = wsm.Chain(tasks, path=path, k_order=k_order)
    ch.run()
    code, failed = ch.status()
    assert code == wsm.WSM_OK, (code, failed, wsm.last_error())
    check_dependent(x0, ws, ys, yfs)
    # run again (next epoch) after poisoning the outputs
    for y in ys:
        y.fill_(float("nan"))
    ch.run()
    assert ch.status()[0] == wsm.WSM_OK
    check_dependent(x0, ws, ys, yfs)
    ch.close()


@pytest.mark.parametrize("path,M", [(wsm.PATH_UMMA, 16), (wsm.PATH_UMMA, 48), (wsm.PATH_STREAM, 4)])
def test_dependent_chain_ahead_of_dependency(path, M):
    """How far a dependent task streams ahead of its dependency (W stages in
    the ring, L2 prefetch) changes only timing: every setting gives the same
    bits, and they pass the oracle."""
    dims = [1024, 3072, 1024, 2048, 1024]
    outs = []
    for ring, pf in ((1, 4), (2, -1), (-1, 8), (0, 0)):
        x0, ws, ys, yfs, tasks = dependent_chain(M, dims, seed=3)
        ch = wsm.Chain(tasks, path=path, dep_ring_stages=ring, l2_prefetch_stages=pf)
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK, wsm.last_error()
        ch.close()
        if not outs:
            check_dependent(x0, ws, ys, yfs)
        outs.append(torch.cat([y.view(torch.int16).flatten() for y in ys]))
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


@pytest.mark.parametrize("deps", [False, True])
def test_chain_units_grow_with_overlapping_work(deps):
    """Independent tasks followed by much more work take longer units (whole
    tiles when there is enough); the last task, with nothing after it, and
    tasks that wait on a dependency keep the single-call choice; an explicit
    unit_stages applies to every task.  Results pass the oracle either way."""
    shapes = [(16, 24576, 4096)] * 4 + [(16, 4096, 12288)]
    tasks = []
    for i, (M, N, K) in enumerate(shapes):
        x, w = synth.make_xw(M, N, K, seed=40 + i)
        tasks.append(wsm.Task(x.to(DEV), w.to(DEV), torch.empty(M, N, dtype=torch.bfloat16, device=DEV),
                              dep=(i - 1) if deps else -1, yf32=torch.empty(M, N, dtype=torch.float32, device=DEV)))
    single = [wsm.plan(M, N, K) for M, N, K in shapes]
    ch = wsm.Chain(tasks)
    plans = [ch.task_plan(i) for i in range(len(tasks))]
    if deps:
        assert [p["unit_stages"] for p in plans] == [p["unit_stages"] for p in single]
    else:
        # later work over 148 CTAs (X tiles of 16 rows): 3 gate_up + down = 10752 stages and 4608 ->
        # whole tiles (alone: 2 units of 8); 1536 (the down) -> units of up to 10 stages -> 2 units of
        # 8; nothing -> as alone
        assert plans[0]["unit_stages"] == plans[0]["k_iters"] == 16
        assert plans[2]["unit_stages"] == 16 > single[2]["unit_stages"]
        assert plans[3]["unit_stages"] == max(8, single[3]["unit_stages"])
        assert plans[4]["unit_stages"] == single[4]["unit_stages"]
    assert all(p["grid"] == plans[0]["grid"] for p in plans)
    ch.run()
    assert ch.status()[0] == wsm.WSM_OK, wsm.last_error()
    rng = np.random.default_rng(2)
    for i, t in enumerate(tasks):
        ms = rng.integers(0, t.x.shape[0], 1024)
        ns = rng.integers(0, t.w.shape[0], 1024)
        check_sampled(t.x, t.w, t.y, t.yf32, ms, ns, what=f"task {i}")
    with pytest.raises(wsm.WsmError):
        ch.task_plan(len(tasks))
    ch.close()
    ch = wsm.Chain(tasks, unit_stages=2)
    assert all(ch.task_plan(i)["unit_stages"] == 2 for i in range(len(tasks)))
    ch.close()


@pytest.mark.parametrize("rows,M", [(0, 1), (0, 2), (16, 2), (32, 4), (32, 8)])
def test_dependent_chain_fma_tile_rows(rows, M):
    """FMA-path chains on either tile height (automatic: one height for the
    whole chain), twice (counters reset per run)."""
    dims = [1024, 2048, 1032, 3072, 520, 4096, 1024]
    x0, ws, ys, yfs, tasks = dependent_chain(M, dims, seed=60 + M + rows)
    ch = wsm.Chain(tasks, path=wsm.PATH_STREAM, tile_rows=rows)
    heights = {ch.task_plan(i)["tile_rows"] for i in range(len(tasks))}
    assert heights == {rows} if rows else len(heights) == 1 and heights <= {16, 32}
    for _ in range(2):
        for y in ys:
            y.fill_(float("nan"))
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK, wsm.last_error()
        check_dependent(x0, ws, ys, yfs)
    ch.close()


@pytest.mark.parametrize("path,M", [(wsm.PATH_UMMA, 16), (wsm.PATH_STREAM, 4)])
def test_dependent_chain_tail_units(path, M):
    """Tail units in every task of a data-dependent chain, run twice (the
    claim counters are reset at the end of each run)."""
    dims = [1024, 2048, 1024, 3072, 512]
    x0, ws, ys, yfs, tasks = dependent_chain(M, dims, seed=30 + M)
    ch = wsm.Chain(tasks, path=path, unit_stages=3, tail_tiles=6, tail_unit_stages=1, l2_prefetch_stages=8)
    for _ in range(2):
        for y in ys:
            y.fill_(float("nan"))
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK
        check_dependent(x0, ws, ys, yfs)
    ch.close()


@pytest.mark.parametrize("path,M,groups", [(wsm.PATH_UMMA, 16, 2), (wsm.PATH_UMMA, 16, 7), (wsm.PATH_UMMA, 48, 3),
                                           (wsm.PATH_STREAM, 2, 2), (wsm.PATH_STREAM, 8, 5)])
def test_two_level_readiness(path, M, groups):
    """Two-level readiness counters (group counters, then one global bump per
    group): a data-dependent chain still orders every task after its
    dependency, over repeated runs and CUDA-graph replays."""
    dims = [1024, 2048, 1024, 3072, 512, 4096, 1024]
    x0, ws, ys, yfs, tasks = dependent_chain(M, dims, seed=50 + groups)
    ch = wsm.Chain(tasks, path=path, counter_groups=groups, flags=wsm.FLAG_W_READONLY)
    for _ in range(2):
        for y in ys:
            y.fill_(float("nan"))
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK, wsm.last_error()
        check_dependent(x0, ws, ys, yfs)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    ch.run(s)
    s.synchronize()
    with torch.cuda.graph(g, stream=s):
        ch.run(s)
    for _ in range(2):
        for y in ys:
            y.fill_(float("nan"))
        g.replay()
        s.synchronize()
        assert ch.status(s)[0] == wsm.WSM_OK
        check_dependent(x0, ws, ys, yfs)
    del g
    ch.close()


def test_two_level_rejects_column_dependencies():
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(64, 64, dtype=torch.bfloat16, device=DEV)
    y0 = torch.empty(4, 64, dtype=torch.bfloat16, device=DEV)
    y1 = torch.empty(4, 64, dtype=torch.bfloat16, device=DEV)
    tasks = [wsm.Task(x, w, y0), wsm.Task(y0, w, y1, dep=0, dep_cols=True)]
    with pytest.raises(wsm.WsmError) as e:
        wsm.Chain(tasks, counter_groups=2)
    assert e.value.code == wsm.WSM_ERR_UNSUPPORTED


@pytest.mark.parametrize("M", [16, 64])
def test_dependent_chain_wide_tiles(M):
    """A data-dependent chain on wide tiles (two 128-row halves per tile),
    with whole-task and per-column dependencies."""
    dims = [1024, 2048, 1024, 3072, 768]
    x0, ws, ys, yfs, tasks = dependent_chain(M, dims, seed=70 + M)
    for cols in (False, True):
        for i, t in enumerate(tasks):
            t.dep_cols = cols and i > 0
        ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, tile_rows=256)
        for _ in range(2):
            for y in ys:
                y.fill_(float("nan"))
            ch.run()
            assert ch.status()[0] == wsm.WSM_OK, wsm.last_error()
            check_dependent(x0, ws, ys, yfs)
        ch.close()


def test_dependent_chain_small_grid_and_empty_ctas():
    """A grid larger than some tasks' stage counts (CTAs with no work for a
    task) and a tiny grid (long per-CTA ranges)."""
    dims = [64, 128, 64, 256]
    for grid in (148, 3):
        x0, ws, ys, yfs, tasks = dependent_chain(16, dims, seed=grid)
        ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, grid=grid)
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK
        check_dependent(x0, ws, ys, yfs)
        ch.close()
        x0, ws, ys, yfs, tasks = dependent_chain(2, dims, seed=grid)
        ch = wsm.Chain(tasks, path=wsm.PATH_STREAM, grid=grid)
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK
        check_dependent(x0, ws, ys, yfs)
        ch.close()


def test_layer_shapes_chain():
    """Two layers of the Qwen3-8B-shaped chain at M = 16, ordering-only
    dependencies (task t waits for task t-1), inputs independent per task."""
    cases = synth.chain_layout(layers=2, M=16)
    tasks, refs = [], []
    for t, c in enumerate(cases):
        x = synth.make_x(c.M, c.K, c.seed).to(DEV)
        w = synth.make_w(c.N, c.K, 10000 + c.seed).to(DEV)
        y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV)
        yf = torch.empty(c.M, c.N, dtype=torch.float32, device=DEV)
        tasks.append(wsm.Task(x, w, y, dep=t - 1, yf32=yf))
    ch = wsm.Chain(tasks, trace=True)
    ch.run()
    assert ch.status()[0] == wsm.WSM_OK
    rng = np.random.default_rng(1)
    for t, task in enumerate(tasks):
        ms = rng.integers(0, 16, 2048)
        ns = rng.integers(0, task.w.shape[0], 2048)
        check_sampled(task.x, task.w, task.y, task.yf32, ms, ns, what=f"task {t}")
    tr = ch.trace()
    assert tr is not None and tr.shape[1] == len(tasks) and tr.shape[2] == 8
    started = tr[:, :, 0]
    assert (started[:, 0] > 0).any()
    # tensor-core path: every task's first stage reached the MMA issuer and an accumulator the
    # epilogue; a CTA's stamps of one task come in order
    for t in range(len(tasks)):
        assert (tr[:, t, 7] > 0).any() and (tr[:, t, 4] > 0).any()
        worked = tr[:, t, 2] > 0
        assert (tr[worked, t, 4] <= tr[worked, t, 2]).all()
        assert (tr[worked, t, 0] <= tr[worked, t, 2]).all()
    ch.close()


def test_bounded_dependency_wait_times_out():
    """A dependency target nothing reaches: each wait runs out after the
    timeout, the run ends, and the status names the waiting task."""
    dims = [256, 256, 256]
    x0, ws, ys, yfs, tasks = dependent_chain(16, dims, seed=5)
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, timeout_ns=20_000_000, debug_unmet_dependency=True)
    t0 = time.time()
    ch.run()
    code, failed = ch.status()
    elapsed = time.time() - t0
    assert code == wsm.WSM_ERR_TIMEOUT and failed in (1, 2)
    assert elapsed < 10.0
    ch.close()
    # the context is still usable and a normal chain still works
    x0, ws, ys, yfs, tasks = dependent_chain(16, dims, seed=6)
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA)
    ch.run()
    assert ch.status()[0] == wsm.WSM_OK
    check_dependent(x0, ws, ys, yfs)
    ch.close()


def test_gemm_chain_one_shot():
    dims = [512, 1024, 512]
    x0, ws, ys, yfs, tasks = dependent_chain(8, dims, seed=11)
    wsm.gemm_chain(tasks)
    torch.cuda.synchronize()
    check_dependent(x0, ws, ys, yfs)
    for y in ys:
        y.fill_(0)
    wsm.gemm_chain(tasks)  # cached prepared chain, next epoch
    torch.cuda.synchronize()
    check_dependent(x0, ws, ys, yfs)


@pytest.mark.parametrize("kernels", [wsm.CHAIN_KERNELS_AUTO, wsm.CHAIN_KERNELS_SPLIT])
def test_chain_plan_matches_prepared_chain(kernels):
    """wsm_chain_plan, computed on the host alone, reports the plan that
    wsm_chain_create makes on this GPU, task by task."""
    shapes = [(1, 1024, 4096, -1), (16, 3072, 1024, 0), (64, 1024, 3072, 1), (8, 2048, 1024, -1), (2, 512, 2048, 3)]
    tasks, specs = [], []
    for i, (M, N, K, dep) in enumerate(shapes):
        x = synth.make_x(M, K, 50 + i).to(DEV)
        w = synth.make_w(N, K, 60 + i).to(DEV)
        tasks.append(wsm.Task(x, w, torch.empty(M, N, dtype=torch.bfloat16, device=DEV), dep=dep))
        specs.append(dict(M=M, N=N, K=K, dep=dep))
    ch = wsm.Chain(tasks, kernels=kernels)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plans, n_kernels = wsm.chain_plan(specs, num_sms=sms, kernels=kernels)
    assert n_kernels == (3 if kernels == wsm.CHAIN_KERNELS_SPLIT else 1)
    for i, p in enumerate(plans):
        tp = ch.task_plan(i)
        assert all(tp[k] == p[k] for k in tp), (i, tp, p)
    ch.close()


@pytest.mark.filterwarnings("ignore:The CUDA Graph is empty")
def test_gemm_chain_in_graph_survives_cache_drop():
    """gemm_chain inside a CUDA graph: a list met for the first time during
    capture is refused (it cannot be prepared there); prepared by a call
    outside capture, it is captured, and the graph still replays correctly
    after more distinct lists than the cache keeps have dropped the others."""
    # shapes no other test passes to gemm_chain: the cache is keyed by pointers and shapes, and
    # freed buffers come back at the same addresses
    dims = [256, 768, 512]
    x0, ws, ys, yfs, tasks = dependent_chain(4, dims, seed=12)
    s = torch.cuda.Stream()
    g0 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g0, stream=s):
        with pytest.raises(wsm.WsmError) as ei:
            wsm.gemm_chain(tasks, stream=s)
    assert ei.value.code == wsm.WSM_ERR_INVALID and "capture" in str(ei.value)
    del g0
    wsm.gemm_chain(tasks, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        wsm.gemm_chain(tasks, stream=s)
    # 20 other lists (distinct output buffers) fill the cache past its bound
    extra = [torch.empty(4, 768, dtype=torch.bfloat16, device=DEV) for _ in range(20)]
    for yx in extra:
        wsm.gemm_chain([wsm.Task(x0, ws[0], yx)], stream=s)
    s.synchronize()
    for y in ys:
        y.fill_(0)
    with torch.cuda.stream(s):
        g.replay()
        g.replay()
    s.synchronize()
    check_dependent(x0, ws, ys, yfs)
    check_full(x0.cpu(), ws[0].cpu(), extra[-1], what="the last extra list")


@pytest.mark.parametrize("deps", [False, True])
@pytest.mark.parametrize("kernels", [wsm.CHAIN_KERNELS_SPLIT, wsm.CHAIN_KERNELS_ONE, wsm.CHAIN_KERNELS_AUTO])
def test_mixed_m_chain(deps, kernels):
    """Tasks of M = 1, 16, 33 and 64 in one chain on the tensor-core path,
    with and without ordering dependencies: as one kernel sharing one stage
    geometry (the widest X tile decides it), and with hybrid dispatch (one
    kernel per run of tasks of one kind, dependencies across kernels met by
    stream order)."""
    tasks = []
    for t, (M, N, K) in enumerate([(16, 1024, 4096), (64, 2048, 2048), (1, 640, 3072), (33, 1000, 1032),
                                   (64, 512, 8192), (16, 4096, 1024)]):
        x, w = synth.make_xw(M, N, K, seed=40 + t)
        tasks.append(wsm.Task(x.to(DEV), w.to(DEV), torch.full((M, N), float("nan"), dtype=torch.bfloat16,
                                                               device=DEV),
                              dep=(t - 1) if deps else -1,
                              yf32=torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)))
    one = kernels != wsm.CHAIN_KERNELS_SPLIT   # AUTO keeps these small tasks in one kernel
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, kernels=kernels, trace=one)
    for _ in range(2):
        for t in tasks:
            t.y.fill_(float("nan"))
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK, wsm.last_error()
        for t in tasks:
            check_full(t.x.cpu(), t.w.cpu(), t.y, t.yf32)
    assert (ch.trace() is not None) == one   # split chains keep no trace
    # each task's plan, from whichever kernel runs it: one kernel sizes every X tile's stages for
    # the widest (64 rows: 2 stages of 96 KB); split, the M <= 32 kernels keep their own ring
    plans = [ch.task_plan(i) for i in range(len(tasks))]
    for t, p in zip(tasks, plans):
        M = t.x.shape[0]
        assert p["m_tile"] >= M and p["m_tile"] % 16 == 0 and p["path"] == wsm.PATH_UMMA
        assert p["n_tiles"] == -(-t.w.shape[0] // 128) and p["k_iters"] * p["tile_k"] >= t.x.shape[1]
    narrow = [p["stages"] for t, p in zip(tasks, plans) if t.x.shape[0] <= 16]
    assert all(n == (2 if one else 3) for n in narrow), narrow
    ch.close()


def test_hybrid_chain_data_dependencies_across_kernels():
    """Hybrid dispatch with data dependencies between its kernels: an M = 16
    task writes the first 16 rows of the M = 64 task's input, whose output's
    first 16 rows feed the next M = 16 task (three kernels; each dependency
    is met by stream order).  Inputs are poisoned before every run."""
    K = 512
    B = synth.make_x(64, K, 81).to(DEV)          # rows 16..63 stay as drawn
    x0 = synth.make_x(16, K, 82).to(DEV)
    ws = [synth.make_w(K, K, 83 + t).to(DEV) for t in range(3)]
    y1 = torch.empty(64, K, dtype=torch.bfloat16, device=DEV)
    y2 = torch.empty(16, K, dtype=torch.bfloat16, device=DEV)
    f = [torch.empty(16, K, device=DEV), torch.empty(64, K, device=DEV), torch.empty(16, K, device=DEV)]
    tasks = [wsm.Task(x0, ws[0], B[0:16], yf32=f[0]),
             wsm.Task(B, ws[1], y1, dep=0, yf32=f[1]),
             wsm.Task(y1[0:16], ws[2], y2, dep=1, yf32=f[2])]
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, kernels=wsm.CHAIN_KERNELS_SPLIT)
    for _ in range(2):
        B[0:16].fill_(float("nan"))
        y1.fill_(float("nan"))
        y2.fill_(float("nan"))
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK
        for t in tasks:
            check_full(t.x.cpu(), t.w.cpu(), t.y, t.yf32)
    ch.close()


def test_independent_tasks_no_deps():
    tasks = []
    for t in range(5):
        M, N, K = [1, 3, 8, 5, 2][t], [4096, 100, 2112, 33, 640][t], [4096, 7168, 512, 8, 1032][t]
        x, w = synth.make_xw(M, N, K, seed=t)
        tasks.append(wsm.Task(x.to(DEV), w.to(DEV), torch.empty(M, N, dtype=torch.bfloat16, device=DEV),
                              yf32=torch.empty(M, N, dtype=torch.float32, device=DEV)))
    ch = wsm.Chain(tasks)
    ch.run()
    assert ch.status()[0] == wsm.WSM_OK
    for t in tasks:
        check_full(t.x.cpu(), t.w.cpu(), t.y, t.yf32)
    ch.close()


@pytest.mark.parametrize("path,M", [(wsm.PATH_UMMA, 16), (wsm.PATH_STREAM, 2)])
def test_dependent_chain_graph_replays(path, M):
    """A chain captured once in a CUDA graph and replayed many times: the
    dependency targets come from a device-side run counter, so every replay
    still orders task t after task t-1."""
    dims = [1024, 3072, 1024, 2048, 4096]
    x0, ws, ys, yfs, tasks = dependent_chain(M, dims, seed=21)
    ch = wsm.Chain(tasks, path=path, flags=wsm.FLAG_W_READONLY)
    s = torch.cuda.Stream()
    ch.run(s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ch.run(s)
    for rep in range(4):
        for y in ys:
            y.fill_(float("nan"))
        g.replay()
        s.synchronize()
        assert ch.status(s)[0] == wsm.WSM_OK
        check_dependent(x0, ws, ys, yfs)
    del g
    ch.close()


@pytest.mark.parametrize("config", ["qwen3_decode", "skinny", "l2_reuse"])
def test_benchmark_chain_full_size_sampled(config):
    """The chain bench.py times for a workload -- every GEMM of the step as an
    independent task of one kernel, full sizes, the weights flagged read-only
    -- checked on sampled outputs of every task, including the ragged end of
    N.  Its tasks run with chain-position work units (longer than the same
    GEMM alone), which this covers at the sizes that use them."""
    cases = getattr(synth, f"config_{config}")()
    tasks = []
    for c in cases:
        g = torch.Generator(device=DEV)
        g.manual_seed(1000 + c.seed + c.M * 7 + c.N)
        x = torch.randn(c.M, c.K, generator=g, device=DEV).to(torch.bfloat16)
        w = (torch.randn(c.N, c.K, generator=g, device=DEV) / c.K ** 0.5).to(torch.bfloat16)
        tasks.append(wsm.Task(x, w, torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV),
                              yf32=torch.empty(c.M, c.N, dtype=torch.float32, device=DEV)))
    ch = wsm.Chain(tasks, flags=wsm.FLAG_W_READONLY)
    plans = [ch.task_plan(i) for i in range(len(tasks))]
    for _ in range(2):  # the second run reuses the counters and partial slots of the first
        ch.run()
    assert ch.status()[0] == wsm.WSM_OK, wsm.last_error()
    rng = np.random.default_rng(5)
    for c, t, p in zip(cases, tasks, plans):
        ms = rng.integers(0, c.M, 1024)
        ns = rng.integers(0, c.N, 1024)
        ns[:32] = np.arange(c.N - 32, c.N)
        check_sampled(t.x, t.w, t.y, t.yf32, ms, ns, what=f"{c.name} (unit_stages {p['unit_stages']})")
    ch.close()
    del tasks
    torch.cuda.empty_cache()


def test_layer_chain_full_36_layers_sampled():
    """The 36 x 4 layer chain at M = 16 exactly as the benchmark runs it:
    task t waits for task t - 1 (ordering only; every task has its own X),
    the weights flagged read-only, 13.9 GB of weights in one kernel; two
    runs (the second on the counters the first left), then sampled outputs
    of every task against the oracle."""
    cases = synth.chain_layout()
    assert len(cases) == 144
    tasks = []
    for t, c in enumerate(cases):
        g = torch.Generator(device=DEV)
        g.manual_seed(3000 + t)
        x = torch.randn(c.M, c.K, generator=g, device=DEV).to(torch.bfloat16)
        w = (torch.randn(c.N, c.K, generator=g, device=DEV) / c.K ** 0.5).to(torch.bfloat16)
        tasks.append(wsm.Task(x, w, torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV), dep=t - 1,
                              yf32=torch.empty(c.M, c.N, dtype=torch.float32, device=DEV)))
    ch = wsm.Chain(tasks, flags=wsm.FLAG_W_READONLY)
    for _ in range(2):
        for t in tasks:
            t.y.fill_(float("nan"))
        ch.run()
    assert ch.status()[0] == wsm.WSM_OK, wsm.last_error()
    rng = np.random.default_rng(11)
    for i, (c, t) in enumerate(zip(cases, tasks)):
        ms = rng.integers(0, c.M, 256)
        ns = rng.integers(0, c.N, 256)
        ns[:16] = np.arange(c.N - 16, c.N)
        check_sampled(t.x, t.w, t.y, t.yf32, ms, ns, what=f"layer chain task {i} ({c.name})")
        assert not torch.isnan(t.y.float()).any(), f"task {i}: unwritten outputs"
    ch.close()
    del tasks
    torch.cuda.empty_cache()
