"""Independent single calls (WSM_FLAG_INDEPENDENT), against the fp64 oracle.

Such a call streams whole tiles in a fixed round-robin (no claim counters, no
partial slots), loads and stores without waiting for the kernel before it, lets
the next kernel launch at once and waits for its predecessor only on exit.
The tests check the results and the stream-order contract of the flag:

- back-to-back independent calls on unrelated buffers, both kernel paths, at
  full and reduced grids (consecutive calls then share the GPU);
- a producer GEMM, then q without the flag and k, v with it, all three
  reading the producer's output (the flag allows k and v to run beside q,
  never beside the producer), then a consumer without the flag reading v's
  output and a plain torch op reading k's: the waits that remain must still
  order every read after its write;
- a chain of independent calls followed by a normal call that overwrites
  their X: the overwrite must wait for every one of them;
- the flag with split tiles asked for explicitly (it is then ignored);
- a device-side time-out inside an independent call (the stall hook)."""
import numpy as np
import pytest
import torch

import synth
import weight_streaming_megakernel_b200 as wsm
from parity import check_full, check_sampled

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
IND = wsm.FLAG_INDEPENDENT


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    wsm.debug_stall(0)


def _nan(M, N, dtype=torch.bfloat16):
    return torch.full((M, N), float("nan"), dtype=dtype, device=DEV)


@pytest.mark.parametrize("grid", [0, 74, 37])
@pytest.mark.parametrize("path,M,N,K", [(wsm.PATH_STREAM, 1, 4096, 4096), (wsm.PATH_STREAM, 4, 2112, 7168),
                                        (wsm.PATH_UMMA, 16, 6144, 4096), (wsm.PATH_UMMA, 40, 1000, 2048),
                                        (wsm.PATH_UMMA, 64, 4096, 1032), (wsm.PATH_AUTO, 3, 6144, 4096)])
def test_back_to_back_independent_calls(path, M, N, K, grid):
    p = wsm.plan(M, N, K, path=path, grid=grid, flags=IND)
    assert p["units"] == p["n_tiles"] * p["m_tiles"], "an independent call plans whole tiles"
    n = 6
    xs, ws = zip(*[synth.make_xw(M, N, K, seed=100 * i + M + grid) for i in range(n)])
    xds = [x.to(DEV) for x in xs]
    wds = [w.to(DEV) for w in ws]
    ys = [_nan(M, N) for _ in range(n)]
    yfs = [_nan(M, N, torch.float32) for _ in range(n)]
    wo = synth.make_w(K, K, seed=7)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(n):
            wsm.skinny_gemm(xds[i], wds[i], ys[i], yf32=yfs[i], path=path, grid=grid, flags=IND, stream=s)
        # a call without the flag may write what the independent calls read: X of the first one
        wsm.skinny_gemm(xds[1], wo.to(DEV), xds[0], path=path, stream=s)
    assert wsm.stream_status(s) == 0
    for i in range(n):
        check_full(xs[i], ws[i], ys[i], yfs[i], what=f"independent call {i} path={path} M={M} grid={grid}")
    check_full(xs[1], wo, xds[0], what="the call after them")


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 2), (wsm.PATH_UMMA, 16)])
def test_group_after_producer_keeps_stream_order(path, M):
    """x -> P (large, no flag) -> y_p; q (no flag), k, v (flag) read y_p;
    D (no flag) reads v's output; a torch op reads k's output."""
    d, n_kv = 2048, 512
    x, wp = synth.make_xw(M, d, 28672, seed=M)          # a slow producer: 112 MiB of weights
    wq = synth.make_w(d, d, seed=M + 1)
    wk = synth.make_w(n_kv, d, seed=M + 2)
    wv = synth.make_w(n_kv, d, seed=M + 3)
    wd = synth.make_w(d, n_kv, seed=M + 4)
    xd, wpd, wqd, wkd, wvd, wdd = (t.to(DEV) for t in (x, wp, wq, wk, wv, wd))
    s = torch.cuda.Stream()
    for rep in range(3):
        y_p, y_q, y_k, y_v, y_d = _nan(M, d), _nan(M, d), _nan(M, n_kv), _nan(M, n_kv), _nan(M, d)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            wsm.skinny_gemm(xd, wpd, y_p, path=path, stream=s)
            wsm.skinny_gemm(y_p, wqd, y_q, path=path, stream=s)
            wsm.skinny_gemm(y_p, wkd, y_k, path=path, grid=48, flags=IND, stream=s)
            wsm.skinny_gemm(y_p, wvd, y_v, path=path, grid=48, flags=IND, stream=s)
            wsm.skinny_gemm(y_v, wdd, y_d, path=path, stream=s)
            k_copy = y_k.clone()
        assert wsm.stream_status(s) == 0
        yp = y_p.cpu()
        check_full(x, wp, y_p, what=f"rep {rep} producer")
        check_full(yp, wq, y_q, what=f"rep {rep} q")
        check_full(yp, wk, y_k, what=f"rep {rep} k (independent)")
        check_full(yp, wv, y_v, what=f"rep {rep} v (independent)")
        check_full(y_v.cpu(), wd, y_d, what=f"rep {rep} consumer of v")
        assert torch.equal(k_copy.view(torch.int16), y_k.view(torch.int16)), "torch op read k before it was written"


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 1), (wsm.PATH_UMMA, 32)])
def test_normal_call_after_independent_calls_waits_for_all(path, M):
    """Four independent calls read X; the normal call after them overwrites X
    (its own output).  Every independent call must have read X before then."""
    N, K = 4096, 4096
    x, _ = synth.make_xw(M, K, K, seed=5)
    ws = [synth.make_w(N, K, seed=10 + i) for i in range(4)]
    w_over = synth.make_w(K, K, seed=20)
    w_dev = [w.to(DEV) for w in ws]
    wo = w_over.to(DEV)
    s = torch.cuda.Stream()
    for rep in range(3):
        xd = x.to(DEV)
        x_in = xd.clone()
        ys = [_nan(M, N) for _ in ws]
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for wd, y in zip(w_dev, ys):
                wsm.skinny_gemm(xd, wd, y, path=path, grid=64, flags=IND, stream=s)
            wsm.skinny_gemm(x_in, wo, xd, path=path, stream=s)  # overwrites X
        assert wsm.stream_status(s) == 0
        for i, (w, y) in enumerate(zip(ws, ys)):
            check_full(x, w, y, what=f"rep {rep} independent call {i}")
        check_full(x, w_over, xd, what=f"rep {rep} overwrite of X")


@pytest.mark.parametrize("path,M,N,K", [(wsm.PATH_UMMA, 16, 6144, 4096), (wsm.PATH_STREAM, 1, 1024, 8192)])
def test_flag_with_explicit_split_tiles(path, M, N, K):
    p = wsm.plan(M, N, K, path=path, flags=IND, unit_stages=2)
    assert p["units"] > p["n_tiles"] * p["m_tiles"]
    x, w = synth.make_xw(M, N, K, seed=N)
    xd, wd = x.to(DEV), w.to(DEV)
    y = _nan(M, N)
    yf = _nan(M, N, torch.float32)
    wsm.skinny_gemm(xd, wd, y, yf32=yf, path=path, flags=IND, unit_stages=2)
    wsm.skinny_gemm(xd, wd, y, yf32=yf, path=path, flags=IND, unit_stages=2)
    assert wsm.stream_status() == 0
    check_full(x, w, y, yf, what="split plan with the flag")


@pytest.mark.parametrize("path,M,N,K", [(wsm.PATH_UMMA, 16, 6144, 4096), (wsm.PATH_STREAM, 1, 4096, 4096)])
def test_independent_timeout_reported_once_then_correct(path, M, N, K):
    x, w = synth.make_xw(M, N, K, seed=3 + M)
    xd, wd = x.to(DEV), w.to(DEV)
    s = torch.cuda.Stream()
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    y2 = _nan(M, N)
    yf2 = _nan(M, N, torch.float32)
    y3 = _nan(M, N)
    s.wait_stream(torch.cuda.current_stream())
    wsm.skinny_gemm(xd, wd, y, path=path, flags=IND, stream=s)
    assert wsm.stream_status(s) == 0
    wsm.debug_stall(1, 50_000_000)
    wsm.skinny_gemm(xd, wd, y, path=path, flags=IND, stream=s)
    # runs beside the stalled call and finishes its work long before the stall's limit
    wsm.skinny_gemm(xd, wd, y2, yf32=yf2, path=path, flags=IND, stream=s)
    wsm.skinny_gemm(xd, wd, y3, path=path, stream=s)  # a normal call on the same workspace after it
    assert wsm.stream_status(s) == wsm.WSM_ERR_TIMEOUT
    assert wsm.stream_status(s) == 0
    check_full(x, w, y2, yf2, what="independent call after the time-out")
    check_full(x, w, y3, what="normal call after the time-out")


def test_chain_rejects_the_flag():
    x, w = synth.make_xw(16, 512, 512, seed=1)
    y = torch.empty(16, 512, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(wsm.WsmError):
        wsm.Chain([wsm.Task(x.to(DEV), w.to(DEV), y)], flags=IND)


@pytest.mark.parametrize("config", ["qwen3_decode", "single", "l2_reuse"])
def test_full_size_independent_launches_sampled(config):
    """The benchmark's independent-launch configurations at full size: every
    GEMM of the set launched back to back with the flag and the automatic
    grid (the weights flagged read-only too), on two weight copies so that
    calls of the same shape run side by side; sampled outputs of every call,
    the ragged end of N included, and no output left unwritten."""
    cases = getattr(synth, f"config_{config}")(**({"m_tiles": (0,)} if config == "l2_reuse" else {}))
    calls = []
    for r in range(2):
        for c in cases:
            g = torch.Generator(device=DEV)
            g.manual_seed(5000 + 97 * r + c.seed + c.M * 7 + c.N)
            x = torch.randn(c.M, c.K, generator=g, device=DEV).to(torch.bfloat16)
            w = (torch.randn(c.N, c.K, generator=g, device=DEV) / c.K ** 0.5).to(torch.bfloat16)
            calls.append((c, x, w, _nan(c.M, c.N), _nan(c.M, c.N, torch.float32)))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for c, x, w, y, yf in calls:
            p = wsm.plan(c.M, c.N, c.K, flags=IND | wsm.FLAG_W_READONLY)
            assert p["units"] == p["n_tiles"] * p["m_tiles"] and p["grid"] <= 37
            wsm.skinny_gemm(x, w, y, yf32=yf, flags=IND | wsm.FLAG_W_READONLY, stream=s)
    assert wsm.stream_status(s) == 0
    rng = np.random.default_rng(9)
    for i, (c, x, w, y, yf) in enumerate(calls):
        ms = rng.integers(0, c.M, 1024)
        ns = rng.integers(0, c.N, 1024)
        ns[:32] = np.arange(c.N - 32, c.N)
        check_sampled(x, w, y, yf, ms, ns, what=f"independent call {i} ({c.name})")
        assert not torch.isnan(y.float()).any(), f"call {i}: unwritten outputs"
    del calls
    torch.cuda.empty_cache()


def test_random_mix_of_independent_calls():
    """40 seeded random calls back to back with the flag -- both paths and
    AUTO, M 1..64 (M-tiles where the path has them), ragged N and K, the
    three epilogues, grids automatic or given -- many of them running side
    by side; then a call without the flag that reads one of their outputs.
    Every output against the oracle."""
    import oracle
    from parity import check_bounded
    rng = np.random.default_rng(2024)
    calls = []
    for i in range(40):
        path = int(rng.choice([wsm.PATH_AUTO, wsm.PATH_STREAM, wsm.PATH_UMMA]))
        M = int(rng.integers(1, 9)) if path == wsm.PATH_STREAM else int(rng.integers(1, 65))
        epi = int(rng.choice([wsm.EPI_NONE, wsm.EPI_NONE, wsm.EPI_SILU_MUL, wsm.EPI_RESIDUAL]))
        N = int(rng.integers(1, 40)) * 16 if epi == wsm.EPI_SILU_MUL else int(rng.integers(1, 700))
        if i == 0:
            epi, N = wsm.EPI_NONE, 8 * int(rng.integers(1, 80))  # read by the last call: K % 8 == 0 there
        K = int(rng.integers(1, 320)) * 8
        grid = int(rng.choice([0, 0, 5, 16, 37, 148]))
        m_tile = int(rng.choice([0, 16, 32])) if path == wsm.PATH_UMMA and M > 16 else 0
        x, w = synth.make_xw(M, N, K, seed=7000 + i)
        out_n = N // 2 if epi == wsm.EPI_SILU_MUL else N
        r = synth.make_x(M, N, seed=8000 + i) if epi == wsm.EPI_RESIDUAL else None
        calls.append(dict(path=path, M=M, N=N, K=K, epi=epi, grid=grid, m_tile=m_tile, x=x, w=w, r=r,
                          xd=x.to(DEV), wd=w.to(DEV), rd=None if r is None else r.to(DEV),
                          y=_nan(M, out_n), yf=_nan(M, out_n, torch.float32)))
    wd_last = synth.make_w(96, calls[0]["y"].shape[1], seed=9000)
    y_last = _nan(calls[0]["M"], 96)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for c in calls:
            wsm.skinny_gemm(c["xd"], c["wd"], c["y"], path=c["path"], yf32=c["yf"], grid=c["grid"],
                            m_tile=c["m_tile"], flags=IND, epilogue=c["epi"], r=c["rd"], stream=s)
        wsm.skinny_gemm(calls[0]["y"], wd_last.to(DEV), y_last, stream=s)
    assert wsm.stream_status(s) == 0
    for i, c in enumerate(calls):
        what = f"call {i}: path {c['path']} M {c['M']} N {c['N']} K {c['K']} epi {c['epi']} grid {c['grid']}"
        if c["epi"] == wsm.EPI_NONE:
            check_full(c["x"], c["w"], c["y"], c["yf"], what=what)
        elif c["epi"] == wsm.EPI_SILU_MUL:
            H, G, U, Sg, Su = oracle.silu_mul_ref(c["x"], c["w"])
            check_bounded(c["y"], c["yf"], H, oracle.fused_bounds("silu_mul", G=G, U=U, Sg=Sg, Su=Su), what)
        else:
            Y, S = oracle.residual_ref(c["x"], c["w"], c["r"])
            check_bounded(c["y"], c["yf"], Y, oracle.fused_bounds("residual", S=S, Y=Y), what)
    check_full(calls[0]["y"].cpu(), wd_last, y_last, what="the call after them")
