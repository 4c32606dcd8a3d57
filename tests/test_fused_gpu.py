"""Fused epilogues and per-column readiness, against the fp64 oracle.

* SiLU*mul: the fused gate+up GEMM (gate and up rows interleaved in blocks of
  8) writes H = silu(gate) * up; checked with oracle.silu_mul_ref and the
  propagated bound oracle.fused_bounds("silu_mul").
* Residual: Y = X W^T + R, including Y written over R in place; exact on
  small-integer inputs.
* Chains whose tasks read the previous task's output per column (dep_cols):
  a layer-like chain o(+R) -> gate_up(SiLU*mul) -> down(+R), each task checked
  against the oracle on the GPU's own input, on both kernel paths, over
  repeated runs and CUDA-graph replays; and the bounded per-column wait.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_streaming_megakernel_b200 as wsm
from parity import check_bounded, bf16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def check_silu(x, w_gu, h, hf32, what=""):
    H, G, U, Sg, Su = oracle.silu_mul_ref(x.cpu(), w_gu.cpu())
    b = oracle.fused_bounds("silu_mul", G=G, U=U, Sg=Sg, Su=Su)
    return check_bounded(h, hf32, H, b, what)


def check_residual(x, w, r, y, yf32, what=""):
    Y, S = oracle.residual_ref(x.cpu(), w.cpu(), r.cpu())
    return check_bounded(y, yf32, Y, oracle.fused_bounds("residual", S=S, Y=Y), what)


def run(x, w, epilogue, r=None, **kw):
    M, K = x.shape
    N = w.shape[0]
    ny = N // 2 if epilogue == wsm.EPI_SILU_MUL else N
    y = torch.full((M, ny), float("nan"), dtype=torch.bfloat16, device=DEV)
    yf = torch.full((M, ny), float("nan"), dtype=torch.float32, device=DEV)
    wsm.skinny_gemm(x.to(DEV), w.to(DEV), y, yf32=yf, epilogue=epilogue,
                    r=None if r is None else r.to(DEV), **kw)
    torch.cuda.synchronize()
    assert wsm.stream_status() == 0
    return y, yf


SILU_CASES = [(1, 64, 256), (2, 1040, 1032), (4, 4096, 4096), (8, 2048, 7168), (16, 3072, 4096),
              (33, 1024, 2048), (64, 2048, 1024)]


@pytest.mark.parametrize("M,N,K", SILU_CASES)
def test_silu_mul(M, N, K):
    x, w = synth.make_xw(M, N, K, seed=M + N)
    paths = [wsm.PATH_UMMA] + ([wsm.PATH_STREAM] if M <= 8 else [])
    for path in paths:
        for grid in (0, 7):
            h, hf = run(x, w, wsm.EPI_SILU_MUL, path=path, grid=grid)
            check_silu(x, w, h, hf, what=f"path={path} grid={grid}")


@pytest.mark.parametrize("rows", [16, 32])
@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_fused_epilogues_fma_tile_rows(rows, M):
    """SiLU*mul (gate/up pairs 8 lanes apart in either tile height) and the
    residual add on both tile heights of the FMA path, whole tiles and split."""
    x, w = synth.make_xw(M, 2080, 1544, seed=90 + M + rows)
    r = synth.make_x(M, 2080, seed=91 + M)
    for us in (0, 1):
        h, hf = run(x, w, wsm.EPI_SILU_MUL, path=wsm.PATH_STREAM, tile_rows=rows, unit_stages=us)
        check_silu(x, w, h, hf, what=f"silu rows={rows} M={M} unit_stages={us}")
        y, yf = run(x, w, wsm.EPI_RESIDUAL, r=r, path=wsm.PATH_STREAM, tile_rows=rows, unit_stages=us)
        check_residual(x, w, r, y, yf, what=f"residual rows={rows} M={M} unit_stages={us}")


def test_silu_mul_auto_and_split_patterns():
    M, N, K = 4, 6144, 4096
    x, w = synth.make_xw(M, N, K, seed=9)
    h0, _ = run(x, w, wsm.EPI_SILU_MUL)
    check_silu(x, w, h0, None)
    for path, us in ((wsm.PATH_UMMA, 1), (wsm.PATH_UMMA, 5), (wsm.PATH_STREAM, 1)):
        h, hf = run(x, w, wsm.EPI_SILU_MUL, path=path, unit_stages=us)
        check_silu(x, w, h, hf, what=f"path={path} unit_stages={us}")


def test_silu_mul_saturates_without_nan():
    """Large gate values: silu(g) -> g for g >> 0 and -> -0 for g << 0."""
    M, N, K = 2, 256, 512
    x, w = synth.make_xw(M, N, K, seed=3)
    w = (w.float() * 40).to(torch.bfloat16)
    for path in (wsm.PATH_STREAM, wsm.PATH_UMMA):
        h, hf = run(x, w, wsm.EPI_SILU_MUL, path=path)
        assert not torch.isnan(hf).any()
        check_silu(x, w, h, hf, what=f"path={path}")


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 1), (wsm.PATH_STREAM, 8), (wsm.PATH_UMMA, 16),
                                    (wsm.PATH_UMMA, 64)])
def test_residual(path, M):
    N, K = 1000, 3072
    x, w = synth.make_xw(M, N, K, seed=M)
    r = synth.make_x(M, N, seed=100 + M)
    y, yf = run(x, w, wsm.EPI_RESIDUAL, r=r, path=path)
    check_residual(x, w, r, y, yf, what=f"path={path}")


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 4), (wsm.PATH_UMMA, 16)])
def test_residual_exact_on_integers_and_in_place(path, M):
    """Small integers: the sum and the added residual are exact in fp32, so
    the fp32 output equals the oracle exactly; then the same with Y = R."""
    N, K = 600, 2048
    x, w = synth.make_int_xw(M, N, K, seed=5)
    r = (torch.randint(-50, 51, (M, N), generator=torch.Generator().manual_seed(6))).to(torch.bfloat16)
    Y, _ = oracle.residual_ref(x, w, r)
    for grid in (0, 5):
        y, yf = run(x, w, wsm.EPI_RESIDUAL, r=r, path=path, grid=grid)
        assert np.array_equal(yf.cpu().double().numpy(), Y)
    yr = r.to(DEV).clone()
    wsm.skinny_gemm(x.to(DEV), w.to(DEV), yr, epilogue=wsm.EPI_RESIDUAL, r=yr, path=path)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(yr), oracle.round_bf16(Y))


def test_epilogue_argument_errors():
    x = torch.zeros(2, 64, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(24, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(wsm.WsmError) as e:
        wsm.skinny_gemm(x, w, torch.empty(2, 12, dtype=torch.bfloat16, device=DEV), epilogue=wsm.EPI_SILU_MUL)
    assert e.value.code == wsm.WSM_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        wsm.skinny_gemm(x, w, epilogue=wsm.EPI_RESIDUAL)


# --------------------------------------------------------------------------- per-column chains


def layer_chain(M, d, dff, layers, seed, dep_cols=True):
    """Per layer: h1 = o(a) + h0; g = silu_mul(gate_up(h1)); h2 = down(g) + h1.
    o reads an independent input a (attention is outside this chain); the
    gate_up and down tasks read the previous task's output."""
    gen = torch.Generator().manual_seed(seed)
    h = synth.make_x(M, d, seed).to(DEV)
    tasks, specs = [], []
    for l in range(layers):
        a = synth.make_x(M, d, seed + 1000 + l).to(DEV)
        wo = synth.make_w(d, d, seed + 2000 + l).to(DEV)
        wgu = synth.make_w(2 * dff, d, seed + 3000 + l).to(DEV)
        wd = synth.make_w(d, dff, seed + 4000 + l).to(DEV)
        h1 = torch.full((M, d), float("nan"), dtype=torch.bfloat16, device=DEV)
        g = torch.full((M, dff), float("nan"), dtype=torch.bfloat16, device=DEV)
        h2 = torch.full((M, d), float("nan"), dtype=torch.bfloat16, device=DEV)
        t0 = len(tasks)
        tasks.append(wsm.Task(a, wo, h1, dep=t0 - 1, epilogue=wsm.EPI_RESIDUAL, r=h,
                              yf32=torch.empty(M, d, device=DEV)))
        tasks.append(wsm.Task(h1, wgu, g, dep=t0, dep_cols=dep_cols, epilogue=wsm.EPI_SILU_MUL,
                              yf32=torch.empty(M, dff, device=DEV)))
        tasks.append(wsm.Task(g, wd, h2, dep=t0 + 1, dep_cols=dep_cols, epilogue=wsm.EPI_RESIDUAL, r=h1,
                              yf32=torch.empty(M, d, device=DEV)))
        specs += ["o", "gate_up", "down"]
        h = h2
    del gen
    return tasks, specs


def check_layer_chain(tasks, specs):
    for t, (task, kind) in enumerate(zip(tasks, specs)):
        if kind == "gate_up":
            check_silu(task.x, task.w, task.y, task.yf32, what=f"task {t} gate_up")
        else:
            check_residual(task.x, task.w, task.r, task.y, task.yf32, what=f"task {t} {kind}")


@pytest.mark.parametrize("path,M", [(wsm.PATH_UMMA, 16), (wsm.PATH_UMMA, 40), (wsm.PATH_STREAM, 2),
                                    (wsm.PATH_STREAM, 8)])
def test_column_dependent_layer_chain(path, M):
    tasks, specs = layer_chain(M, 1024, 2048, layers=3, seed=M)
    ch = wsm.Chain(tasks, path=path)
    for rep in range(3):
        for t in tasks:
            t.y.fill_(float("nan"))
        ch.run()
        code, failed = ch.status()
        assert code == wsm.WSM_OK, (code, failed, wsm.last_error())
        check_layer_chain(tasks, specs)
    ch.close()


def test_column_chain_matches_whole_task_chain_bitwise():
    """Per-column waits change when work runs, not what it computes: the same
    chain with whole-task dependencies gives the same bits (same plan: the
    K order is fixed, since the automatic one differs between the two)."""
    outs = []
    for dep_cols in (True, False):
        tasks, specs = layer_chain(16, 1024, 1536, layers=2, seed=3, dep_cols=dep_cols)
        ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, unit_stages=2, k_order=1)
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK
        outs.append([t.y.clone() for t in tasks])
        ch.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_column_chain_small_grids_and_graph_replay():
    tasks, specs = layer_chain(16, 512, 1024, layers=2, seed=8)
    for grid in (1, 3, 37):
        ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, grid=grid)
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK
        check_layer_chain(tasks, specs)
        ch.close()
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, flags=wsm.FLAG_W_READONLY)
    s = torch.cuda.Stream()
    ch.run(s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ch.run(s)
    for _ in range(3):
        for t in tasks:
            t.y.fill_(float("nan"))
        g.replay()
        s.synchronize()
        assert ch.status(s)[0] == wsm.WSM_OK
        check_layer_chain(tasks, specs)
    del g
    ch.close()


def test_column_wait_times_out():
    """A per-column target nothing reaches: the wait runs out after the
    timeout and the status names a waiting task; the context stays usable."""
    tasks, specs = layer_chain(16, 512, 512, layers=1, seed=4)
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, timeout_ns=20_000_000, debug_unmet_dependency=True)
    t0 = time.time()
    ch.run()
    code, failed = ch.status()
    assert code == wsm.WSM_ERR_TIMEOUT and failed in (1, 2)
    assert time.time() - t0 < 10.0
    ch.close()
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA)
    ch.run()
    assert ch.status()[0] == wsm.WSM_OK
    check_layer_chain(tasks, specs)
    ch.close()
