"""Device-side time-outs reach the caller on every entry point, and the call
after one computes correct results.

Every wait inside the kernels is bounded.  These tests make one run out on
demand with the library's stall hook (wsm_debug_stall: CTA 0 of the next
launch waits on a flag that nothing sets until a short limit passes, records
WSM_ERR_TIMEOUT and abandons its work -- no fault, every other wait stays
bounded).  The abandoned work leaves claim, tile and readiness counters
mid-count; the launch's last CTA repairs them.  Each test checks that the
status query reports the time-out exactly once and that the next call on the
same scratch (stream workspace, caller workspace, one-shot chain, prepared
chain) matches the fp64 oracle."""
import time

import pytest
import torch

import synth
import weight_streaming_megakernel_b200 as wsm
from parity import check_full

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
STALL_NS = 50_000_000


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    wsm.debug_stall(0)


def _inputs(M, N, K, seed):
    x, w = synth.make_xw(M, N, K, seed=seed)
    return x, w, x.to(DEV), w.to(DEV)


# (path, M, N, K): split tiles on both paths, so abandoned units leave tile arrival counters mid-count
SPLIT_CASES = [(wsm.PATH_UMMA, 16, 6144, 4096), (wsm.PATH_STREAM, 1, 1024, 8192), (wsm.PATH_UMMA, 64, 2048, 4096)]


@pytest.mark.parametrize("path,M,N,K", SPLIT_CASES)
def test_stream_workspace_timeout_reported_once_then_correct(path, M, N, K):
    p = wsm.plan(M, N, K, path=path)
    assert p["units"] > p["n_tiles"] * p["m_tiles"], "the case must split tiles"
    x, w, xd, wd = _inputs(M, N, K, seed=M + N)
    s = torch.cuda.Stream()
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    s.wait_stream(torch.cuda.current_stream())
    wsm.skinny_gemm(xd, wd, y, path=path, stream=s)  # sizes the stream's workspace
    assert wsm.stream_status(s) == 0
    wsm.debug_stall(1, STALL_NS)
    t0 = time.time()
    wsm.skinny_gemm(xd, wd, y, path=path, stream=s)
    # the next call, queued before anyone looks at the status, runs on the repaired counters
    with torch.cuda.stream(s):
        y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        yf2 = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    wsm.skinny_gemm(xd, wd, y2, path=path, yf32=yf2, stream=s)
    assert wsm.stream_status(s) == wsm.WSM_ERR_TIMEOUT
    assert time.time() - t0 < 5.0
    assert "site 6" in wsm.last_error()
    assert wsm.stream_status(s) == 0, "a time-out is reported once"
    check_full(x, w, y2, yf2, what="the call queued after the time-out")
    with torch.cuda.stream(s):
        y.fill_(float("nan"))
        yf = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    wsm.skinny_gemm(xd, wd, y, path=path, yf32=yf, stream=s)
    assert wsm.stream_status(s) == 0
    check_full(x, w, y, yf, what="a later call")


@pytest.mark.parametrize("path,M,N,K", SPLIT_CASES[:2])
def test_caller_workspace_timeout_reported_once_then_correct(path, M, N, K):
    x, w, xd, wd = _inputs(M, N, K, seed=3 * M + N)
    nbytes = wsm.workspace_bytes(M, N, K, path=path)
    ws = torch.zeros(nbytes // 4 + 64, dtype=torch.int32, device=DEV)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    wsm.debug_stall(1, STALL_NS)
    wsm.skinny_gemm(xd, wd, y, path=path, workspace=ws)
    yf = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    y.fill_(float("nan"))
    wsm.skinny_gemm(xd, wd, y, path=path, yf32=yf, workspace=ws)
    assert wsm.workspace_status(ws) == wsm.WSM_ERR_TIMEOUT
    assert wsm.workspace_status(ws) == 0
    # the time-out was on the caller's buffer, not on the stream's own workspace
    assert wsm.stream_status() == 0
    check_full(x, w, y, yf, what="the call queued after the time-out")


def test_timeout_before_workspace_growth_is_reported():
    """The call after a time-out needs a larger stream workspace: the time-out
    recorded in the outgrown buffer is still reported."""
    x, w, xd, wd = _inputs(16, 512, 1024, seed=4)
    X, W, Xd, Wd = _inputs(64, 8192, 8192, seed=5)
    s = torch.cuda.Stream()
    y = torch.empty(16, 512, dtype=torch.bfloat16, device=DEV)
    with torch.cuda.stream(s):
        Y = torch.full((64, 8192), float("nan"), dtype=torch.bfloat16, device=DEV)
    wsm.skinny_gemm(xd, wd, y, stream=s)
    assert wsm.stream_status(s) == 0
    assert wsm.workspace_bytes(64, 8192, 8192) > (1 << 20), "the second call must outgrow the first workspace"
    wsm.debug_stall(1, STALL_NS)
    wsm.skinny_gemm(xd, wd, y, stream=s)
    wsm.skinny_gemm(Xd, Wd, Y, stream=s)
    assert wsm.stream_status(s) == wsm.WSM_ERR_TIMEOUT
    assert wsm.stream_status(s) == 0
    check_full(X, W, Y, what="the call on the grown workspace")


def _dependent_tasks(M, dims, seed):
    x0 = synth.make_x(M, dims[0], seed).to(DEV)
    ws = [synth.make_w(dims[t + 1], dims[t], 500 + seed + t).to(DEV) for t in range(len(dims) - 1)]
    ys = [torch.empty(M, dims[t + 1], dtype=torch.bfloat16, device=DEV) for t in range(len(ws))]
    yfs = [torch.empty(M, dims[t + 1], dtype=torch.float32, device=DEV) for t in range(len(ws))]
    tasks = [wsm.Task(x0 if t == 0 else ys[t - 1], ws[t], ys[t], dep=t - 1, yf32=yfs[t]) for t in range(len(ws))]
    return x0, ws, ys, yfs, tasks


def _check_dependent(x0, ws, ys, yfs, what):
    x = x0
    for t in range(len(ws)):
        check_full(x.cpu(), ws[t].cpu(), ys[t], yfs[t], what=f"{what}: task {t}")
        x = ys[t]


@pytest.mark.parametrize("M", [16, 2])
def test_one_shot_chain_timeout_reported_once_then_correct(M):
    """gemm_chain (cached prepared chain): the time-out is reported by
    gemm_chain_status, and the next run of the same cached chain -- whose
    done counters the abandoned run left short -- orders its tasks again."""
    x0, ws, ys, yfs, tasks = _dependent_tasks(M, [1024, 3072, 1024, 2048], seed=M)
    wsm.gemm_chain(tasks)
    assert wsm.gemm_chain_status() == (wsm.WSM_OK, -1)
    wsm.debug_stall(1, STALL_NS)
    t0 = time.time()
    wsm.gemm_chain(tasks)
    for rep in range(2):
        # rep 0 is queued before anyone looks at the status: it runs on the counters the
        # abandoned run repaired on the device
        for y in ys:
            y.fill_(float("nan"))
        wsm.gemm_chain(tasks)
        code, failed = wsm.gemm_chain_status()
        if rep == 0:
            assert code == wsm.WSM_ERR_TIMEOUT and failed == -1, (code, failed)
            assert time.time() - t0 < 5.0
        else:
            assert code == wsm.WSM_OK
        _check_dependent(x0, ws, ys, yfs, f"run {rep} after the time-out")


@pytest.mark.parametrize("cluster", [wsm.CHAIN_CLUSTER_OFF, wsm.CHAIN_CLUSTER_ON])
def test_prepared_chain_graph_replays_after_timeout(cluster):
    """A prepared chain captured in a CUDA graph: a time-out in an eager run
    is reported once by wsm_chain_status, and later graph replays (which read
    the run counter from device memory) stay ordered and correct.  With
    cluster reduction the abandoned CTA's peers give up on their exchanges
    (tasks split 2 and 4 ways), and the waits of the failed run stop ordering
    its tasks; the exchange must stay well defined through all of that."""
    x0, ws, ys, yfs, tasks = _dependent_tasks(16, [512, 2048, 512, 1024, 512], seed=9)
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, cluster=cluster)
    if cluster == wsm.CHAIN_CLUSTER_ON:
        nus = {ch.task_plan(t)["units"] // ch.task_plan(t)["n_tiles"] for t in range(len(tasks))}
        assert nus == {2, 4}
    s = torch.cuda.Stream()
    ch.run(s)
    assert ch.status(s)[0] == wsm.WSM_OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ch.run(s)
    wsm.debug_stall(1, STALL_NS)
    ch.run(s)
    assert ch.status(s) == (wsm.WSM_ERR_TIMEOUT, -1)
    assert ch.status(s)[0] == wsm.WSM_OK
    for rep in range(3):
        with torch.cuda.stream(s):
            for y in ys:
                y.fill_(float("nan"))
            g.replay()
        s.synchronize()
        assert ch.status(s)[0] == wsm.WSM_OK
        _check_dependent(x0, ws, ys, yfs, f"replay {rep}")
    del g
    ch.close()


def test_two_level_chain_heals_group_counters():
    """Two-level readiness (group counters) after a time-out."""
    x0, ws, ys, yfs, tasks = _dependent_tasks(16, [1024, 2048, 1024], seed=21)
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, counter_groups=4)
    wsm.debug_stall(1, STALL_NS)
    ch.run()
    for rep in range(2):
        for y in ys:
            y.fill_(float("nan"))
        ch.run()
        code = ch.status()[0]
        assert code == (wsm.WSM_ERR_TIMEOUT if rep == 0 else wsm.WSM_OK)
        _check_dependent(x0, ws, ys, yfs, f"run {rep}")
    ch.close()


def test_stall_hook_arguments():
    with pytest.raises(wsm.WsmError):
        wsm.debug_stall(-1)
    with pytest.raises(wsm.WsmError):
        wsm.debug_stall(1, 0)
    wsm.debug_stall(0)
