"""Cluster reduction in linear dependent chains (wsm_chain_opts.cluster =
ON), against the fp64 oracle and against the global-memory reduction.

In a chain where every task waits for the one before it, the tensor-core
kernel can run as clusters of 4 CTAs and reduces the split tiles of each task's
first round through distributed shared memory.  The sum is taken in unit
order, the order of the global-memory reduction, so with the same split (same
work units on the same grid) the two must give the same bits.  Checked: data
chains at several X widths (16-row to 64-row tiles, padded M), the fused
SiLU*mul and residual epilogues, multi-round tasks whose later units fall back
to global partials, repeated runs and CUDA-graph replays, and the plan the
chain reports."""
import pytest
import torch

import oracle
import synth
import weight_streaming_megakernel_b200 as wsm
from parity import bf16_bits, check_bounded, check_full

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def _data_chain(M, dims, seed):
    x0 = synth.make_x(M, dims[0], seed).to(DEV)
    ws = [synth.make_w(dims[t + 1], dims[t], 700 + seed + t).to(DEV) for t in range(len(dims) - 1)]
    ys = [torch.full((M, dims[t + 1]), float("nan"), dtype=torch.bfloat16, device=DEV) for t in range(len(ws))]
    yfs = [torch.full((M, dims[t + 1]), float("nan"), dtype=torch.float32, device=DEV) for t in range(len(ws))]
    tasks = [wsm.Task(x0 if t == 0 else ys[t - 1], ws[t], ys[t], dep=t - 1, yf32=yfs[t]) for t in range(len(ws))]
    return x0, ws, ys, yfs, tasks


def _check(x0, ws, ys, yfs, what):
    x = x0
    for t in range(len(ws)):
        check_full(x.cpu(), ws[t].cpu(), ys[t], yfs[t], what=f"{what}: task {t}")
        x = ys[t]


@pytest.mark.parametrize("M", [16, 5, 17, 32, 64])
def test_cluster_chain_matches_oracle_and_global_reduction(M):
    dims = [4096, 6144, 4096, 4096, 12288, 4096, 1024]
    x0, ws, ys, yfs, tasks = _data_chain(M, dims, seed=M)
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, cluster=wsm.CHAIN_CLUSTER_ON)
    plans = [ch.task_plan(t) for t in range(len(tasks))]
    specs = [dict(M=M, N=dims[t + 1], K=dims[t], dep=t - 1) for t in range(len(tasks))]
    host, _ = wsm.chain_plan(specs, path=wsm.PATH_UMMA, cluster=wsm.CHAIN_CLUSTER_ON)
    grid = plans[0]["grid"]
    assert grid % 4 == 0 and all(h["cluster"] == 4 for h in host)
    for h, p in zip(host, plans):
        assert (h["grid"], h["units"], h["unit_stages"]) == (p["grid"], p["units"], p["unit_stages"])
    assert any(p["units"] > p["n_tiles"] * p["m_tiles"] for p in plans), "some task must split its tiles"
    ch.run()
    assert ch.status()[0] == wsm.WSM_OK
    _check(x0, ws, ys, yfs, f"cluster M={M}")
    got = [bf16_bits(y).copy() for y in ys]
    gotf = [yf.cpu().clone() for yf in yfs]
    ch.close()
    # the same split on the same grid without clusters: every partial goes through global memory
    for t in range(len(tasks)):
        ys[t].fill_(float("nan"))
        yfs[t].fill_(float("nan"))
    for t in range(len(tasks)):
        one = wsm.Chain([wsm.Task(tasks[t].x, ws[t], ys[t], yf32=yfs[t])], path=wsm.PATH_UMMA, grid=grid,
                        unit_stages=plans[t]["unit_stages"], tail_tiles=-1, cluster=wsm.CHAIN_CLUSTER_OFF,
                        k_order=wsm.K_ORDER_ROTATED)
        assert one.task_plan(0)["units"] == plans[t]["units"]
        one.run()
        assert one.status()[0] == wsm.WSM_OK
        one.close()
        assert (bf16_bits(ys[t]) == got[t]).all(), f"task {t}: bf16 bits differ from the cluster reduction"
        assert torch.equal(yfs[t].cpu().view(torch.int32), gotf[t].view(torch.int32)), f"task {t}: fp32 bits differ"


def test_cluster_chain_fused_epilogues_repeated_runs_and_graph():
    """o (+R in place) -> gate_up (SiLU*mul) -> down, repeated: whole-task
    data dependencies with fused epilogues, eagerly and in a graph."""
    M, d, ff = 16, 4096, 6144
    x0 = synth.make_x(M, d, seed=3).to(DEV)
    w_o = synth.make_w(d, d, seed=4).to(DEV)
    w_gu = synth.make_w(2 * ff, d, seed=5).to(DEV)
    w_dn = synth.make_w(d, ff, seed=6).to(DEV)
    r = synth.make_x(M, d, seed=7).to(DEV)
    h0 = r.clone()
    h1 = torch.empty(M, ff, dtype=torch.bfloat16, device=DEV)
    h2 = torch.empty(M, d, dtype=torch.bfloat16, device=DEV)
    f2 = torch.empty(M, d, dtype=torch.float32, device=DEV)
    tasks = [wsm.Task(x0, w_o, h0, epilogue=wsm.EPI_RESIDUAL, r=h0),
             wsm.Task(h0, w_gu, h1, dep=0, epilogue=wsm.EPI_SILU_MUL),
             wsm.Task(h1, w_dn, h2, dep=1, yf32=f2)]
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, cluster=wsm.CHAIN_CLUSTER_ON)
    assert ch.task_plan(0)["grid"] % 4 == 0
    s = torch.cuda.Stream()

    def check(what):
        Y0, S0 = oracle.residual_ref(x0.cpu(), w_o.cpu(), r.cpu())
        check_bounded(h0, None, Y0, oracle.fused_bounds("residual", S=S0, Y=Y0), f"{what} o")
        H, G, U, Sg, Su = oracle.silu_mul_ref(h0.cpu(), w_gu.cpu())
        check_bounded(h1, None, H, oracle.fused_bounds("silu_mul", G=G, U=U, Sg=Sg, Su=Su), f"{what} gate_up")
        check_full(h1.cpu(), w_dn.cpu(), h2, f2, what=f"{what} down")

    for rep in range(2):
        with torch.cuda.stream(s):
            h0.copy_(r)
        ch.run(s)
        assert ch.status(s)[0] == wsm.WSM_OK
        check(f"run {rep}")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ch.run(s)
    for rep in range(2):
        with torch.cuda.stream(s):
            h0.copy_(r)
            h1.fill_(float("nan"))
            h2.fill_(float("nan"))
            g.replay()
        s.synchronize()
        assert ch.status(s)[0] == wsm.WSM_OK
        check(f"replay {rep}")
    del g
    ch.close()
