"""Parity of skinny_gemm (both kernel paths) with the fp64 oracle, through the
C ABI, on seeded inputs: small shapes spanning several tiles with ragged
tails, every M, integer and permutation cases that must be exact, split
patterns (grid sizes), M-tiling orders, caller workspace, determinism, CUDA
graph capture, and the full-size workloads on sampled outputs."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_streaming_megakernel_b200 as wsm
from parity import check_full, check_sampled, bf16_bits

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def run(x, w, **kw):
    M, K = x.shape
    N = w.shape[0]
    xd, wd = x.to(DEV), w.to(DEV)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    yf = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    wsm.skinny_gemm(xd, wd, y, yf32=yf, **kw)
    torch.cuda.synchronize()
    assert wsm.stream_status() == 0
    return y, yf


SHAPES = [(1, 8), (17, 40), (300, 1000), (129, 4104), (1024, 4096), (2112, 7168)]


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("N,K", SHAPES)
def test_stream_path_small(M, N, K):
    x, w = synth.make_xw(M, N, K, seed=M * 7 + N)
    y, yf = run(x, w, path=wsm.PATH_STREAM)
    check_full(x, w, y, yf, what=f"stream M={M} N={N} K={K}")


@pytest.mark.parametrize("rows", [16, 32])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("N,K", [(17, 40), (300, 1000), (129, 4104), (2112, 7168)])
def test_stream_path_tile_rows(rows, M, N, K):
    """Both tile heights of the FMA path (16 rows: 2 row groups x 4 K-slices;
    32 rows: 4 x 2), ragged N and K, whole tiles and K split over units."""
    x, w = synth.make_xw(M, N, K, seed=M * 11 + N + rows)
    for us in (0, 1):
        y, yf = run(x, w, path=wsm.PATH_STREAM, tile_rows=rows, unit_stages=us)
        check_full(x, w, y, yf, what=f"stream rows={rows} M={M} N={N} K={K} unit_stages={us}")
    p = wsm.plan(M, N, K, path=wsm.PATH_STREAM, tile_rows=rows)
    assert p["tile_rows"] == rows and p["tile_k"] == (1024 if rows == 16 else 512)


@pytest.mark.parametrize("M", [1, 8, 16, 17, 32, 40, 64])
@pytest.mark.parametrize("N,K", SHAPES)
def test_umma_path_small(M, N, K):
    x, w = synth.make_xw(M, N, K, seed=M * 5 + N)
    y, yf = run(x, w, path=wsm.PATH_UMMA)
    check_full(x, w, y, yf, what=f"umma M={M} N={N} K={K}")


@pytest.mark.parametrize("path,ms", [(wsm.PATH_STREAM, range(1, 9)), (wsm.PATH_UMMA, range(1, 65))])
def test_every_m(path, ms):
    N, K = 520, 1032
    for M in ms:
        x, w = synth.make_xw(M, N, K, seed=100 + M)
        y, yf = run(x, w, path=path)
        check_full(x, w, y, yf, what=f"path={path} M={M}")


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 1), (wsm.PATH_STREAM, 7), (wsm.PATH_UMMA, 16),
                                    (wsm.PATH_UMMA, 64)])
def test_integer_inputs_exact(path, M):
    """Small integers: every partial sum is exact in fp32, so the fp32 output
    must equal the oracle exactly whatever the split."""
    N, K = 777, 4096
    x, w = synth.make_int_xw(M, N, K, seed=M)
    Y_ref, _ = oracle.gemm_ref(x, w)
    for grid in (0, 1, 5, 37):
        y, yf = run(x, w, path=path, grid=grid)
        assert np.array_equal(yf.cpu().double().numpy(), Y_ref), f"grid={grid}"
        assert np.array_equal(bf16_bits(y), oracle.round_bf16(Y_ref))


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 4), (wsm.PATH_UMMA, 16)])
def test_identity_and_permutation(path, M):
    K = 512
    x, _ = synth.make_xw(M, K, K, seed=3)
    I = torch.eye(K, dtype=torch.bfloat16)
    y, yf = run(x, I, path=path)
    assert torch.equal(y.cpu(), x)
    P, p = synth.make_permutation_w(K, seed=4)
    y, yf = run(x, P, path=path)
    assert torch.equal(y.cpu(), x[:, p])
    xo, idx = synth.make_onehot_x(M, K, seed=5)
    _, w = synth.make_xw(1, 300, K, seed=6)
    y, _ = run(xo, w, path=path)
    assert torch.equal(y.cpu(), w[:, idx].T.contiguous())


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 1), (wsm.PATH_STREAM, 8), (wsm.PATH_UMMA, 16),
                                    (wsm.PATH_UMMA, 48)])
@pytest.mark.parametrize("grid", [1, 2, 3, 7, 64, 148])
def test_split_patterns(path, M, grid):
    """Different grids put the split points (and the in-order reductions) in
    different places; every one must satisfy the bound."""
    N, K = 1000, 6144
    x, w = synth.make_xw(M, N, K, seed=grid)
    y, yf = run(x, w, path=path, grid=grid)
    check_full(x, w, y, yf, what=f"grid={grid}")


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 2), (wsm.PATH_UMMA, 16)])
@pytest.mark.parametrize("pf", [-1, 1, 64])
def test_l2_prefetch_back_to_back(path, M, pf):
    """The L2 prefetch issued while a launch waits for the previous kernel
    (W read-only flag) is only a hint: back-to-back launches give the same
    bits for every prefetch depth."""
    N, K = 3000, 4096
    x, w = synth.make_xw(M, N, K, seed=60 + M)
    xd, wd = x.to(DEV), w.to(DEV)
    ref = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    wsm.skinny_gemm(xd, wd, ref, path=path, l2_prefetch_stages=-1)
    ys = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV) for _ in range(4)]
    for y in ys:
        wsm.skinny_gemm(xd, wd, y, path=path, flags=wsm.FLAG_W_READONLY, l2_prefetch_stages=pf)
    torch.cuda.synchronize()
    assert wsm.stream_status() == 0
    for y in ys:
        assert torch.equal(y, ref)
    check_full(x, w, ys[-1], None, what=f"pf={pf}")


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 2), (wsm.PATH_STREAM, 8), (wsm.PATH_UMMA, 16),
                                    (wsm.PATH_UMMA, 64)])
def test_tail_units(path, M):
    """Tail tiles split into smaller units than the head tiles: exact on
    small-integer inputs (bitwise equal to the unsplit result) and within the
    bound on random inputs, for several tail sizes, unit sizes and grids."""
    N, K = 1000, 6144
    xi, wi = synth.make_int_xw(M, N, K, seed=40 + M)
    Y_ref, _ = oracle.gemm_ref(xi, wi)
    x, w = synth.make_xw(M, N, K, seed=50 + M)
    for tail_tiles, tus, grid in [(1, 1, 0), (5, 2, 0), (1000, 1, 0), (7, 3, 37), (3, 1, 5)]:
        y, yf = run(xi, wi, path=path, grid=grid, tail_tiles=tail_tiles, tail_unit_stages=tus)
        assert np.array_equal(yf.cpu().double().numpy(), Y_ref), (tail_tiles, tus, grid)
        y, yf = run(x, w, path=path, grid=grid, tail_tiles=tail_tiles, tail_unit_stages=tus)
        check_full(x, w, y, yf, what=f"tail_tiles={tail_tiles} tail_unit_stages={tus} grid={grid}")


def test_all_ones_closed_form():
    for path, M in ((wsm.PATH_STREAM, 3), (wsm.PATH_UMMA, 20)):
        K = 256
        x = torch.ones(M, K, dtype=torch.bfloat16)
        w = torch.ones(130, K, dtype=torch.bfloat16)
        y, yf = run(x, w, path=path)
        assert (yf.cpu() == K).all() and (y.cpu().float() == K).all()


@pytest.mark.parametrize("M,tm", [(32, 16), (64, 16), (64, 32), (40, 16)])
@pytest.mark.parametrize("order", [wsm.ORDER_M_MAJOR, wsm.ORDER_NAIVE])
def test_m_tiling(M, tm, order):
    N, K = 1100, 2048
    x, w = synth.make_xw(M, N, K, seed=M + tm)
    y, yf = run(x, w, path=wsm.PATH_UMMA, m_tile=tm, order=order)
    check_full(x, w, y, yf, what=f"M={M} tm={tm} order={order}")
    xi, wi = synth.make_int_xw(M, N, K, seed=1)
    Y_ref, _ = oracle.gemm_ref(xi, wi)
    y, yf = run(xi, wi, path=wsm.PATH_UMMA, m_tile=tm, order=order)
    assert np.array_equal(yf.cpu().double().numpy(), Y_ref)


@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 4), (wsm.PATH_UMMA, 32)])
def test_deterministic(path, M):
    N, K = 4096, 4096
    x, w = synth.make_xw(M, N, K, seed=9)
    y1, f1 = run(x, w, path=path)
    y2, f2 = run(x, w, path=path)
    assert torch.equal(y1, y2) and torch.equal(f1.view(torch.int32), f2.view(torch.int32))


def test_l2_policy_options_same_result():
    x, w = synth.make_xw(16, 2000, 3000, seed=1)
    outs = []
    for pol in (wsm.L2_EVICT_FIRST, wsm.L2_NORMAL):
        y, yf = run(x, w, path=wsm.PATH_UMMA, l2_policy=pol)
        outs.append(yf)
    assert torch.equal(outs[0], outs[1])


def test_caller_workspace():
    M, N, K = 8, 4096, 4096
    x, w = synth.make_xw(M, N, K, seed=2)
    need = wsm.workspace_bytes(M, N, K)
    ws = torch.zeros(need // 4 + 64, dtype=torch.int32, device=DEV)
    y, yf = run(x, w, workspace=ws)
    check_full(x, w, y, yf)
    y2, yf2 = run(x, w, workspace=ws)  # left reusable by the first call
    assert torch.equal(yf, yf2)
    with pytest.raises(wsm.WsmError) as e:
        run(x, w, workspace=ws[:8])
    assert e.value.code == wsm.WSM_ERR_NOMEM


def test_argument_errors():
    x = torch.zeros(2, 64, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(64, 64, dtype=torch.bfloat16, device=DEV)
    y = torch.zeros(2, 64, dtype=torch.bfloat16, device=DEV)
    L = wsm.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert L.skinny_gemm(0, w.data_ptr(), y.data_ptr(), 2, 64, 64, s) == wsm.WSM_ERR_INVALID
    assert L.skinny_gemm(x.data_ptr() + 2, w.data_ptr(), y.data_ptr(), 2, 64, 64, s) == wsm.WSM_ERR_ALIGN
    assert L.skinny_gemm(x.data_ptr(), w.data_ptr(), y.data_ptr(), 2, 64, 60, s) == wsm.WSM_ERR_UNSUPPORTED
    assert L.skinny_gemm(x.data_ptr(), w.data_ptr(), y.data_ptr(), 65, 64, 64, s) == wsm.WSM_ERR_UNSUPPORTED
    assert "unsupported" in wsm.last_error()


def test_cuda_graph_capture():
    M, N, K = 16, 4096, 4096
    x, w = synth.make_xw(M, N, K, seed=4)
    xd, wd = x.to(DEV), w.to(DEV)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        wsm.skinny_gemm(xd, wd, y)  # sizes the stream's workspace outside capture
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        wsm.skinny_gemm(xd, wd, y, stream=s)
    y.fill_(0)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    check_full(x, w, y)


def test_graph_survives_workspace_growth():
    """A graph captured with the stream's workspace still replays correctly
    after a larger call on that stream has outgrown the workspace (the
    library keeps the outgrown buffer, which the graph still points at)."""
    M, N, K = 16, 1024, 4096
    M2, N2, K2 = 64, 2048, 16384
    assert wsm.workspace_bytes(M2, N2, K2) > max(1 << 20, 2 * wsm.workspace_bytes(M, N, K))
    x, w = synth.make_xw(M, N, K, seed=5)
    x2, w2 = synth.make_xw(M2, N2, K2, seed=6)
    xd, wd, x2d, w2d = x.to(DEV), w.to(DEV), x2.to(DEV), w2.to(DEV)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    y2 = torch.empty(M2, N2, dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        wsm.skinny_gemm(xd, wd, y)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        wsm.skinny_gemm(xd, wd, y, stream=s)
    with torch.cuda.stream(s):
        wsm.skinny_gemm(x2d, w2d, y2)  # grows the stream's workspace
        y.fill_(0)
        g.replay()
        g.replay()
    s.synchronize()
    assert wsm.stream_status(s) == 0
    check_full(x, w, y, what="graph after workspace growth")
    rng = np.random.default_rng(0)
    ms = rng.integers(0, M2, 2048)
    ns = rng.integers(0, N2, 2048)
    check_sampled(x2, w2, y2, None, ms, ns, what="the call that grew the workspace")


def test_empty_ranges_when_fewer_stages_than_ctas():
    """T < grid: the plan clamps the grid, and a forced-large grid on a chain
    covers it in-kernel (see the chain tests)."""
    x, w = synth.make_xw(3, 40, 64, seed=1)
    y, yf = run(x, w, path=wsm.PATH_STREAM, grid=148)
    check_full(x, w, y, yf)
    x, w = synth.make_xw(20, 130, 128, seed=1)
    y, yf = run(x, w, path=wsm.PATH_UMMA, grid=148)
    check_full(x, w, y, yf)


# ----------------------------------------------------------- full-size workloads

def _full_cases():
    cases = []
    cases += synth.config_single()
    cases += synth.config_qwen3_decode()
    cases += synth.config_skinny()
    cases += synth.config_l2_reuse()
    return cases


@pytest.mark.parametrize("case", _full_cases(), ids=lambda c: c.name)
def test_full_size_sampled(case):
    """The benchmark's shapes and launch configuration (default plan; M-tile
    where the config names one), checked on 4096 sampled outputs."""
    g = torch.Generator(device=DEV)
    g.manual_seed(case.seed)
    x = torch.randn(case.M, case.K, generator=g, device=DEV).to(torch.bfloat16)
    w = (torch.randn(case.N, case.K, generator=g, device=DEV) / case.K ** 0.5).to(torch.bfloat16)
    y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device=DEV)
    yf = torch.empty(case.M, case.N, dtype=torch.float32, device=DEV)
    kw = {"m_tile": case.m_tile} if case.m_tile else {}
    wsm.skinny_gemm(x, w, y, yf32=yf, **kw)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    ms = rng.integers(0, case.M, 4096)
    ns = rng.integers(0, case.N, 4096)
    ns[:64] = np.arange(case.N - 64, case.N)  # the ragged end of N
    check_sampled(x, w, y, yf, ms, ns, what=case.name)


def test_workspace_reused_across_shapes():
    """One scratch buffer (the stream's, then a caller's) serves shapes with
    very different tile counts and partial sizes in turn: the counters of
    one shape must never sit on another shape's partial sums."""
    seq = [(64, 1000, 8192, wsm.PATH_UMMA), (1, 8192, 4096, wsm.PATH_STREAM), (48, 300, 12288, wsm.PATH_UMMA),
           (2, 16384, 1024, wsm.PATH_STREAM), (8, 4096, 7168, wsm.PATH_STREAM), (64, 6000, 2048, wsm.PATH_UMMA)]
    for M, N, K, path in seq:
        x, w = synth.make_xw(M, N, K, seed=N)
        y, yf = run(x, w, path=path)
        check_full(x, w, y, yf, what=f"stream workspace M={M} N={N} K={K}")
    need = max(wsm.workspace_bytes(M, N, K, path=path) for M, N, K, path in seq)
    ws = torch.zeros(need // 4, dtype=torch.int32, device=DEV)
    for M, N, K, path in seq:
        x, w = synth.make_xw(M, N, K, seed=N + 1)
        y, yf = run(x, w, path=path, workspace=ws)
        check_full(x, w, y, yf, what=f"caller workspace M={M} N={N} K={K}")


@pytest.mark.parametrize("flags", [0, wsm.FLAG_W_READONLY, wsm.FLAG_NO_PDL])
@pytest.mark.parametrize("path,M", [(wsm.PATH_STREAM, 2), (wsm.PATH_UMMA, 16)])
def test_back_to_back_dependent_calls(flags, path, M):
    """Calls queued back to back on one stream, each reading the previous
    call's Y as its X: the programmatic-dependent-launch waits must keep
    stream order for X, Y and the scratch (W may be streamed early only
    with FLAG_W_READONLY, and W is never written here)."""
    dims = [2048, 4096, 1024, 6144, 2048, 4096]
    xs = [synth.make_x(M, dims[0], 1).to(DEV)]
    ws = [synth.make_w(dims[i + 1], dims[i], 50 + i).to(DEV) for i in range(len(dims) - 1)]
    ys = [torch.full((M, dims[i + 1]), float("nan"), dtype=torch.bfloat16, device=DEV) for i in range(len(ws))]
    for rep in range(3):
        for y in ys:
            y.fill_(float("nan"))
        x = xs[0]
        for i, w in enumerate(ws):
            wsm.skinny_gemm(x, w, ys[i], path=path, flags=flags)
            x = ys[i]
        torch.cuda.synchronize()
        assert wsm.stream_status() == 0
        x = xs[0]
        for i, w in enumerate(ws):
            check_full(x.cpu(), w.cpu(), ys[i], what=f"rep {rep} call {i} flags {flags}")
            x = ys[i]


# --------------------------------------------------------------------------- wide tiles


@pytest.mark.parametrize("M", [1, 16, 33, 64])
@pytest.mark.parametrize("N,K", [(1000, 1032), (129, 4104), (4096, 4096), (300, 256)])
def test_wide_tiles(M, N, K):
    """Tiles of two 128-row W halves sharing each X stage (two accumulators):
    ragged N (the second half may lie past N), every grid split."""
    x, w = synth.make_xw(M, N, K, seed=M * 7 + N)
    for grid in (0, 5):
        y, yf = run(x, w, path=wsm.PATH_UMMA, tile_rows=256, grid=grid)
        check_full(x, w, y, yf, what=f"wide M={M} grid={grid}")


@pytest.mark.parametrize("M", [16, 64])
def test_wide_tiles_integer_exact_and_options(M):
    N, K = 1000, 3072
    x, w = synth.make_int_xw(M, N, K, seed=M)
    Y_ref, _ = oracle.gemm_ref(x, w)
    for kw in (dict(), dict(unit_stages=1), dict(stage_k=64), dict(stage_k=256), dict(m_tile=16),
               dict(tail_tiles=2, tail_unit_stages=1)):
        y, yf = run(x, w, path=wsm.PATH_UMMA, tile_rows=256, **kw)
        assert np.array_equal(yf.cpu().double().numpy(), Y_ref), kw
        assert np.array_equal(bf16_bits(y), oracle.round_bf16(Y_ref)), kw


def test_wide_tiles_fused_epilogues():
    M, N, K = 32, 1024, 2048
    x, w = synth.make_xw(M, N, K, seed=91)
    y = torch.full((M, N // 2), float("nan"), dtype=torch.bfloat16, device=DEV)
    yf = torch.full((M, N // 2), float("nan"), dtype=torch.float32, device=DEV)
    wsm.skinny_gemm(x.to(DEV), w.to(DEV), y, yf32=yf, path=wsm.PATH_UMMA, tile_rows=256, epilogue=wsm.EPI_SILU_MUL)
    torch.cuda.synchronize()
    H, G, U, Sg, Su = oracle.silu_mul_ref(x, w)
    from parity import check_bounded
    check_bounded(y, yf, H, oracle.fused_bounds("silu_mul", G=G, U=U, Sg=Sg, Su=Su), "wide silu")
    r = synth.make_x(M, N, 92)
    y, yf = run(x, w, path=wsm.PATH_UMMA, tile_rows=256, epilogue=wsm.EPI_RESIDUAL, r=r.to(DEV))
    Yr, S = oracle.residual_ref(x, w, r)
    check_bounded(y, yf, Yr, oracle.fused_bounds("residual", S=S, Y=Yr), "wide residual")


@pytest.mark.parametrize("path,M", [(wsm.PATH_UMMA, 1), (wsm.PATH_UMMA, 16), (wsm.PATH_UMMA, 64),
                                    (wsm.PATH_STREAM, 1), (wsm.PATH_STREAM, 8)])
def test_rotated_k_order(path, M):
    """Units walking their K stages from a tile-dependent offset: exact on
    small integers, within the bound on random inputs, deterministic."""
    N, K = 1000, 6144
    xi, wi = synth.make_int_xw(M, N, K, seed=3 + M)
    Y_ref, _ = oracle.gemm_ref(xi, wi)
    for kw in (dict(), dict(unit_stages=5), dict(grid=7)):
        y, yf = run(xi, wi, path=path, k_order=2, **kw)
        assert np.array_equal(yf.cpu().double().numpy(), Y_ref), kw
    x, w = synth.make_xw(M, N, K, seed=4 + M)
    y1, yf1 = run(x, w, path=path, k_order=2, unit_stages=7)
    check_full(x, w, y1, yf1)
    y2, yf2 = run(x, w, path=path, k_order=2, unit_stages=7)
    assert torch.equal(yf1, yf2)


@pytest.mark.parametrize("M", [16, 32, 64])
@pytest.mark.parametrize("stage_k", [64, 128, 192, 256])
def test_stage_widths_exact(M, stage_k):
    """Every stage width, including 192 (three 64-wide boxes: K = 4104 leaves
    a last stage of one partial box and two boxes past K, zero-filled)."""
    N, K = 700, 4104
    x, w = synth.make_int_xw(M, N, K, seed=stage_k + M)
    Y_ref, _ = oracle.gemm_ref(x, w)
    y, yf = run(x, w, path=wsm.PATH_UMMA, stage_k=stage_k)
    assert np.array_equal(yf.cpu().double().numpy(), Y_ref)
    assert np.array_equal(bf16_bits(y), oracle.round_bf16(Y_ref))
