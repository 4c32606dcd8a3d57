"""C-ABI library checks that need no GPU: it loads, exports every function
include/wsm.h declares, and its pure host logic (planning, task-list
validation) behaves as documented."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import weight_streaming_megakernel_b200 as wsm
from weight_streaming_megakernel_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wsm.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    yield


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while", "sizeof")))


def test_header_parse_sees_all_entry_points():
    names = header_functions()
    assert set(names) == set(wsm.HEADER_SYMBOLS), names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(wsm.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), f"{name} declared in wsm.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", wsm.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in header_functions():
        assert name in exported


def test_abi_version():
    assert wsm.abi_version() == 2


def test_status_queries_and_stall_hook_check_arguments_on_the_host():
    """The time-out queries and the stall test hook reject bad arguments
    before any CUDA call (so this runs without a GPU)."""
    L = wsm.lib()
    code = ctypes.c_int(-7)
    assert L.wsm_workspace_status(None, 1 << 20, None, ctypes.byref(code)) == wsm.WSM_ERR_INVALID
    assert code.value == 0
    assert L.wsm_workspace_status(ctypes.c_void_p(0x1008), 1 << 20, None, ctypes.byref(code)) == wsm.WSM_ERR_ALIGN
    assert L.wsm_workspace_status(ctypes.c_void_p(0x1000), 256, None, ctypes.byref(code)) == wsm.WSM_ERR_INVALID
    assert L.wsm_debug_stall(-1, 1000) == wsm.WSM_ERR_INVALID
    assert L.wsm_debug_stall(1, 0) == wsm.WSM_ERR_INVALID
    assert L.wsm_debug_stall(1, 20_000_000_000) == wsm.WSM_ERR_INVALID
    assert L.wsm_debug_stall(2, 1_000_000) == wsm.WSM_OK
    assert L.wsm_debug_stall(0, 0) == wsm.WSM_OK


def test_plan_paths_and_geometry():
    p = wsm.plan(1, 4096, 4096, num_sms=148)
    assert p["path"] == wsm.PATH_STREAM and p["tile_rows"] == 32 and p["m_tile"] == 1
    assert p["n_tiles"] == 128 and p["k_iters"] == 4096 // p["tile_k"]
    assert p["iters"] == p["n_tiles"] * p["k_iters"] and p["grid"] == 128   # one CTA per (whole-tile) unit
    p = wsm.plan(1, 4096, 4096, num_sms=148, tile_rows=16)
    assert p["tile_rows"] == 16 and p["n_tiles"] == 256 and p["grid"] == 148
    p = wsm.plan(16, 4096, 4096, num_sms=148)
    assert p["path"] == wsm.PATH_UMMA and p["tile_rows"] == 128 and p["tile_k"] == 256 and p["m_tile"] == 16
    assert p["n_tiles"] == 32 and p["k_iters"] == 16 and p["m_tiles"] == 1
    p = wsm.plan(16, 4096, 4096, num_sms=148, stage_k=64)
    assert p["tile_k"] == 64 and p["k_iters"] == 64
    p = wsm.plan(48, 4096, 4096, num_sms=148)
    assert p["tile_k"] == 256 and p["m_tile"] == 48 and p["stages"] == 2
    p = wsm.plan(17, 100, 1000, num_sms=148)          # 32-row X tiles: 192-wide stages
    assert p["m_tile"] == 32 and p["n_tiles"] == 1 and p["tile_k"] == 192 and p["k_iters"] == 6
    p = wsm.plan(8, 4096, 4096, num_sms=148, path=wsm.PATH_UMMA)
    assert p["path"] == wsm.PATH_UMMA and p["m_tile"] == 16


def test_auto_path_crossovers():
    """AUTO: FMA path for M <= 2 at any size, M <= 4 up to 64 MiB of weights;
    tensor cores otherwise."""
    S, U = wsm.PATH_STREAM, wsm.PATH_UMMA
    cases = [(1, 4096, 4096, S), (1, 4096, 12288, S), (1, 10240, 8192, S), (1, 24576, 4096, S), (1, 57344, 8192, S),
             (2, 4096, 12288, S), (2, 10240, 8192, S), (2, 24576, 4096, S), (4, 4096, 4096, S),
             (4, 4096, 7168, S), (4, 4096, 12288, U), (3, 6144, 4096, S), (5, 64, 64, U), (8, 4096, 4096, U),
             (16, 64, 64, U), (3, 24576, 4096, U)]
    for M, N, K, want in cases:
        assert wsm.plan(M, N, K)["path"] == want, (M, N, K)
    # exactly at the threshold for M = 3, 4
    assert wsm.plan(4, 4096, 8192)["path"] == S           # 64 MiB
    assert wsm.plan(4, 4097, 8192)["path"] == U
    assert wsm.plan(3, 4097, 8192)["path"] == U


def test_independent_calls_plan():
    """WSM_FLAG_INDEPENDENT: whole tiles (no split-K) unless split units are
    asked for; grid 0 = at most a quarter of the SMs in even rounds of units,
    a given grid as it is (at most one CTA per unit); the tensor cores from
    M = 3 (the FMA path up to M = 2)."""
    IND = wsm.FLAG_INDEPENDENT
    for M, N, K in [(1, 4096, 4096), (16, 6144, 4096), (16, 4096, 4096), (64, 8192, 2048), (2, 1024, 8192),
                    (1, 24576, 4096)]:
        for grid in (0, 37, 74):
            p = wsm.plan(M, N, K, flags=IND, grid=grid)
            u = p["units"]
            assert u == p["n_tiles"] * p["m_tiles"], (M, N, K, grid)
            if grid:
                assert p["grid"] == min(grid, u)
            else:  # at most a quarter of the SMs, in even rounds
                rounds = -(-u // 37)
                assert p["grid"] == -(-u // rounds) and p["grid"] <= 37, (M, N, K, p["grid"])
    assert wsm.plan(1, 4096, 4096, flags=IND)["grid"] == 32      # 128 units: 4 rounds of 32
    assert wsm.plan(16, 6144, 4096, flags=IND)["grid"] == 24     # 48 units: 2 rounds of 24
    assert wsm.plan(16, 4096, 4096, flags=IND)["grid"] == 32     # 32 units: 1 round
    assert wsm.plan(16, 4096, 4096)["units"] > wsm.plan(16, 4096, 4096)["n_tiles"]  # without the flag: split
    p = wsm.plan(16, 6144, 4096, flags=IND, unit_stages=2)
    assert p["units"] > p["n_tiles"]
    S, U = wsm.PATH_STREAM, wsm.PATH_UMMA
    for M, want in ((1, S), (2, S), (3, U), (4, U), (8, U)):
        assert wsm.plan(M, 4096, 4096, flags=IND)["path"] == want, M
    assert wsm.plan(4, 4096, 4096)["path"] == S


def test_fma_tile_rows():
    """FMA path tile height: 32 rows (16 KB boxes, the faster stream per SM)
    unless that leaves too few tiles (fewer than half the CTAs: K split in
    two); an explicit tile_rows of 16 or 32 is taken as given, anything else
    refused on this path.  Units: whole tiles from half as many tiles as CTAs
    up, 2 per tile below."""
    def rows(M, N, K, **kw):
        p = wsm.plan(M, N, K, num_sms=148, path=wsm.PATH_STREAM, **kw)
        assert p["tile_k"] == (1024 if p["tile_rows"] == 16 else 512)
        nu = -(-p["k_iters"] // p["unit_stages"])
        assert nu == (1 if p["n_tiles"] * 2 >= 148 else 2) or p["k_iters"] == 1
        return p["tile_rows"]
    assert rows(1, 4096, 4096) == 32          # o: 128 whole 32-row tiles, one round
    assert rows(1, 4096, 7168) == 32
    assert rows(1, 6144, 4096) == 32          # qkv: 192 tiles of 32 rows
    assert rows(1, 24576, 4096) == 32         # gate_up
    assert rows(1, 4096, 12288) == 32         # down
    assert rows(1, 2112, 7168) == 16          # 66 tiles of 32 rows would split K: 132 whole 16-row tiles
    assert rows(2, 57344, 8192) == 32
    assert rows(1, 4096, 4096, tile_rows=32) == 32
    assert rows(1, 24576, 4096, tile_rows=16) == 16
    with pytest.raises(wsm.WsmError):
        wsm.plan(1, 4096, 4096, path=wsm.PATH_STREAM, tile_rows=128)
    with pytest.raises(wsm.WsmError):
        wsm.plan(16, 4096, 4096, path=wsm.PATH_UMMA, tile_rows=32)


def test_plan_ring_fits_shared_memory():
    for M in (1, 2, 3, 4, 8, 16, 33, 64):
        p = wsm.plan(M, 4096, 4096, num_sms=148)
        assert 2 <= p["stages"] <= 16
        assert p["smem_bytes"] <= 232448 - 4096


def test_plan_grid_clamped_to_work():
    p = wsm.plan(1, 16, 8, num_sms=148)
    assert p["iters"] == 1 and p["grid"] == 1
    p = wsm.plan(1, 4096, 4096, num_sms=148, grid=7)
    assert p["grid"] == 7
    p = wsm.plan(1, 8192, 4096, num_sms=148, grid=1000)
    assert p["grid"] == 148
    p = wsm.plan(1, 4096, 4096, num_sms=148, grid=1000)
    assert p["grid"] == p["units"] == 128


def test_plan_m_tiling_and_l2_policy():
    p = wsm.plan(64, 24576, 4096, num_sms=148, m_tile=16)
    assert p["m_tiles"] == 4 and p["m_tile"] == 16 and p["l2_policy"] == wsm.L2_NORMAL
    assert p["order"] == wsm.ORDER_M_MAJOR
    p = wsm.plan(64, 24576, 4096, num_sms=148, m_tile=32, order=wsm.ORDER_NAIVE)
    assert p["m_tiles"] == 2 and p["order"] == wsm.ORDER_NAIVE
    p = wsm.plan(32, 4096, 12288, num_sms=148)
    assert p["m_tiles"] == 1 and p["l2_policy"] == wsm.L2_EVICT_FIRST


def test_plan_workspace_formula():
    p = wsm.plan(16, 4096, 4096, num_sms=148)
    nu = -(-p["k_iters"] // p["unit_stages"])
    assert p["units"] == p["n_tiles"] * p["m_tiles"] * nu
    counters = (2 + p["n_tiles"] * p["m_tiles"]) * 4
    partials = p["units"] * 128 * 16 * 4 if nu > 1 else 0
    assert p["workspace_bytes"] >= 256 + counters + partials
    assert p["workspace_bytes"] % 256 == 0


def test_auto_units_per_tile():
    """The automatic split of tiles into units on the tensor-core path (the
    cost model fitted to measured B200 times): many-tile shapes split less,
    few-tile shapes more, wider X tiles (larger partials) less."""
    def nu(M, N, K):
        p = wsm.plan(M, N, K, num_sms=148, path=wsm.PATH_UMMA)
        return -(-p["k_iters"] // p["unit_stages"])
    assert nu(16, 4096, 4096) == 4          # 32 tiles: 128 units, one round
    assert nu(16, 4096, 12288) == 4
    assert nu(16, 18432, 7168) == 1         # 144 tiles: one unit per CTA
    assert nu(16, 10240, 8192) == 3         # 80 tiles: 240 units
    assert nu(16, 57344, 8192) == 4         # 448 tiles: many rounds, small tail
    assert nu(64, 24576, 4096) == 2         # 192 tiles at M = 64: three rounds of 8 stages
    assert nu(64, 57344, 8192) == 2
    assert nu(16, 6144, 4096) == 3
    assert nu(16, 24576, 4096) == 2         # 192 tiles: 384 units in three whole rounds (measured
    assert nu(8, 24576, 4096) == 2          # 40.0 us against 42.7 with 4 units per tile)
    assert nu(32, 24576, 4096) == 2


def test_plan_units():
    """At most 4 units per tile on the tensor-core path, 2 on the FMA path;
    the units cover every stage of a tile exactly once."""
    for M, N, K in [(1, 4096, 4096), (16, 4096, 4096), (1, 57344, 8192), (16, 24576, 4096), (4, 2112, 7168),
                    (16, 4096, 12288), (64, 300, 72)]:
        for path in (wsm.PATH_STREAM, wsm.PATH_UMMA):
            if path == wsm.PATH_STREAM and M > 8:
                continue
            p = wsm.plan(M, N, K, num_sms=148, path=path)
            nu = -(-p["k_iters"] // p["unit_stages"])
            assert 1 <= p["unit_stages"] <= p["k_iters"]
            assert nu <= (4 if path == wsm.PATH_UMMA else 2)
            assert (nu - 1) * p["unit_stages"] < p["k_iters"] <= nu * p["unit_stages"]
            assert p["units"] == p["n_tiles"] * p["m_tiles"] * nu
    p = wsm.plan(16, 4096, 4096, num_sms=148, unit_stages=3)
    assert p["unit_stages"] == 3 and p["units"] == 32 * 6


def test_plan_tail_units():
    """The last tail_tiles tiles are split into units of tail_unit_stages
    stages; the head tiles keep unit_stages.  Units and workspace follow."""
    M, N, K = 16, 4096, 4096          # 32 tiles x 16 stages of 256
    base = wsm.plan(M, N, K, num_sms=148, path=wsm.PATH_UMMA, tail_tiles=-1)
    assert base["tail_tiles"] == 0 and base["units"] == 32 * 4
    p = wsm.plan(M, N, K, num_sms=148, path=wsm.PATH_UMMA, tail_tiles=10, tail_unit_stages=2)
    assert p["tail_tiles"] == 10 and p["tail_unit_stages"] == 2 and p["unit_stages"] == base["unit_stages"]
    assert p["units"] == 22 * 4 + 10 * 8
    assert p["workspace_bytes"] >= p["units"] * 128 * 16 * 4
    # uneven split: 16 stages in units of 3 -> 6 units per tail tile, the last one short
    p = wsm.plan(M, N, K, num_sms=148, path=wsm.PATH_UMMA, tail_tiles=5, tail_unit_stages=3)
    assert p["units"] == 27 * 4 + 5 * 6
    # more tail tiles than tiles: every tile is a tail tile
    p = wsm.plan(M, N, K, num_sms=148, path=wsm.PATH_UMMA, tail_tiles=1000, tail_unit_stages=1)
    assert p["tail_tiles"] == 32 and p["units"] == 32 * 16
    # the FMA path takes the same options
    p = wsm.plan(2, 2112, 7168, num_sms=148, path=wsm.PATH_STREAM, tail_tiles=20, tail_unit_stages=1)
    assert p["tail_tiles"] == 20 and p["units"] == (p["n_tiles"] - 20) * -(-p["k_iters"] // p["unit_stages"]) + 20 * p["k_iters"]
    for bad in (dict(tail_tiles=-2), dict(tail_unit_stages=-1), dict(unit_stages=-1), dict(l2_prefetch_stages=-2)):
        with pytest.raises(wsm.WsmError) as e:
            wsm.plan(M, N, K, **bad)
        assert e.value.code == wsm.WSM_ERR_INVALID


@pytest.mark.parametrize("M,N,K", [(0, 16, 16), (65, 16, 16), (1, 0, 16), (1, 16, 4), (1, 16, 12), (1, 16, 0)])
def test_plan_rejects_unsupported_shapes(M, N, K):
    with pytest.raises(wsm.WsmError) as e:
        wsm.plan(M, N, K)
    assert e.value.code == wsm.WSM_ERR_UNSUPPORTED


def test_plan_rejects_bad_options():
    with pytest.raises(wsm.WsmError) as e:
        wsm.plan(9, 64, 64, path=wsm.PATH_STREAM)
    assert e.value.code == wsm.WSM_ERR_UNSUPPORTED
    for tm in (8, 24, 80):
        with pytest.raises(wsm.WsmError) as e:
            wsm.plan(64, 64, 64, m_tile=tm)
        assert e.value.code == wsm.WSM_ERR_UNSUPPORTED
    with pytest.raises(wsm.WsmError) as e:
        wsm.plan(4, 64, 64, path=7)
    assert e.value.code == wsm.WSM_ERR_INVALID
    with pytest.raises(wsm.WsmError) as e:
        wsm.plan(4, 64, 64, grid=-1)
    assert e.value.code == wsm.WSM_ERR_INVALID


def _task(i, M=4, N=64, K=64, dep=-1, base=0x10000000):
    a = base + i * 0x100000
    return {"X": a, "W": a + 0x40000, "Y": a + 0x80000, "M": M, "N": N, "K": K, "dep": dep}


def test_chain_validation_accepts_good_lists():
    wsm.chain_validate([_task(0), _task(1, dep=0), _task(2, dep=0), _task(3, dep=2)])


@pytest.mark.parametrize("bad,code", [
    ({"dep": 3}, wsm.WSM_ERR_INVALID),      # forward dependency
    ({"dep": 1}, wsm.WSM_ERR_INVALID),      # self dependency
    ({"dep": -2}, wsm.WSM_ERR_INVALID),
    ({"X": 0}, wsm.WSM_ERR_INVALID),        # null pointer
    ({"Y": 0x10000008}, wsm.WSM_ERR_ALIGN),  # misaligned
    ({"K": 12}, wsm.WSM_ERR_UNSUPPORTED),
    ({"M": 65}, wsm.WSM_ERR_UNSUPPORTED),
])
def test_chain_validation_rejects(bad, code):
    tasks = [_task(0), _task(1, dep=0)]
    tasks[1].update(bad)
    with pytest.raises(wsm.WsmError) as e:
        wsm.chain_validate(tasks)
    assert e.value.code == code


def test_chain_validation_empty():
    with pytest.raises(wsm.WsmError) as e:
        wsm.chain_validate([])
    assert e.value.code == wsm.WSM_ERR_INVALID


def test_missing_library_fails_loudly(tmp_path):
    code = (
        "import weight_streaming_megakernel_b200 as w\n"
        f"w.LIB_PATH = {str(tmp_path / 'nope.so')!r}\n"
        "try:\n"
        "    w.lib()\n"
        "except RuntimeError as e:\n"
        "    print('RAISED', e)\n"
    )
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT)
    assert "RAISED" in out.stdout and "not built" in out.stdout


def test_product_never_touches_the_oracle():
    """The product package shares nothing with oracle/ and never imports it."""
    pkg = os.path.dirname(wsm.__file__)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "wsmo_" not in src, f
    oracle_src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    assert "wsm.h" not in oracle_src and "wsm_internal" not in oracle_src


def test_chain_validate_epilogues_and_column_deps():
    base = 0x20000000
    ok = [
        {"X": base, "W": base + 0x100000, "Y": base + 0x200000, "M": 4, "N": 64, "K": 64},
        {"X": base + 0x200000, "W": base + 0x300000, "Y": base + 0x400000, "M": 4, "N": 128, "K": 64, "dep": 0,
         "dep_cols": 1, "epilogue": wsm.EPI_SILU_MUL},
        {"X": base + 0x400000, "W": base + 0x500000, "Y": base + 0x600000, "M": 4, "N": 64, "K": 64, "dep": 1,
         "dep_cols": 1, "epilogue": wsm.EPI_RESIDUAL, "R": base + 0x200000},
    ]
    wsm.chain_validate(ok)

    def bad(i, code, **kv):
        ts = [dict(t) for t in ok]
        ts[i].update(kv)
        with pytest.raises(wsm.WsmError) as e:
            wsm.chain_validate(ts)
        assert e.value.code == code, kv

    bad(0, wsm.WSM_ERR_INVALID, epilogue=7)
    bad(1, wsm.WSM_ERR_UNSUPPORTED, N=120)                       # SiLU*mul needs N % 16 == 0
    bad(2, wsm.WSM_ERR_INVALID, R=None)                          # residual without R
    bad(2, wsm.WSM_ERR_INVALID, R=base + 0x200001)               # misaligned R
    bad(1, wsm.WSM_ERR_INVALID, dep=-1)                          # dep_cols without a dependency
    bad(1, wsm.WSM_ERR_INVALID, X=base + 0x700000)               # X is not the dep task's Y
    bad(2, wsm.WSM_ERR_INVALID, K=128)                           # K != dep's output columns (128 / 2)
    bad(2, wsm.WSM_ERR_INVALID, M=8)                             # M differs from the dep task's


def test_plan_accepts_epilogue_options():
    wsm.plan(4, 4096, 4096, epilogue=wsm.EPI_SILU_MUL)
    wsm.plan(4, 4096, 4096, epilogue=wsm.EPI_RESIDUAL)


# ----------------------------------------------------------- chain planning (pure host)

QWEN3_LAYER = ((4096, 6144), (4096, 4096), (4096, 24576), (12288, 4096))  # (K, N): qkv, o, gate_up, down


def test_chain_plan_independent_decode_step():
    """The decode step (20 independent GEMMs, M = 1..16) as one tensor-core
    kernel: units grow with the work after them (whole tiles while plenty
    follows), the last task keeps the single-call split; 12 prefetch stages
    (no dependencies, X tiles of 16 rows) and the rotated K order."""
    specs = [dict(M=m, N=n, K=k) for m in (1, 2, 4, 8, 16) for (k, n) in QWEN3_LAYER]
    plans, kernels = wsm.chain_plan(specs)
    assert kernels == 1
    for s, p in zip(specs, plans):
        assert p["path"] == wsm.PATH_UMMA and p["grid"] == 148 and p["kernel"] == 0
        assert p["l2_prefetch_stages"] == 12 and p["k_order"] == wsm.K_ORDER_ROTATED and p["dep_ring_stages"] == 1
        assert p["stages"] == 3 and p["m_tile"] == 16
        assert p["workspace_bytes"] == 0
    for p in plans[:12]:
        assert p["unit_stages"] == p["k_iters"], p  # whole tiles early in the step
    last = wsm.plan(16, 4096, 12288)
    assert plans[-1]["unit_stages"] == last["unit_stages"] and plans[-1]["units"] == last["units"]


def test_chain_plan_dependent_layers():
    """Task t waits for t - 1: nothing overlaps a task's end, so every task
    takes the single-call split on all 148 CTAs; 4 prefetch stages, one ring
    stage ahead of the dependency, rotated K order.  With cluster reduction
    requested: clusters of 4 CTAs (132 resident on 148 SMs), 1, 2 or 4 units
    per tile from the cost model (qkv: 2, o: 4, gate_up: 2, down: 4), no
    tail units."""
    specs = []
    for layer in range(3):
        for (k, n) in QWEN3_LAYER:
            specs.append(dict(M=16, N=n, K=k, dep=len(specs) - 1))
    plans, kernels = wsm.chain_plan(specs)
    assert kernels == 1
    for s, p in zip(specs, plans):
        single = wsm.plan(16, s["N"], s["K"])
        assert p["cluster"] == 0 and p["grid"] == 148
        assert p["unit_stages"] == single["unit_stages"] and p["units"] == single["units"], (s, p, single)
        assert p["l2_prefetch_stages"] == 4 and p["dep_ring_stages"] == 1 and p["k_order"] == wsm.K_ORDER_ROTATED
    plans, _ = wsm.chain_plan(specs, cluster=wsm.CHAIN_CLUSTER_ON)
    units_per_tile = {6144: 2, 4096: 4, 24576: 2}
    for s, p in zip(specs, plans):
        assert p["cluster"] == 4 and p["grid"] == 132, p
        nu = p["units"] // (p["n_tiles"] * p["m_tiles"])
        assert nu == units_per_tile[s["N"]], (s, p)
        assert p["unit_stages"] * nu >= p["k_iters"] > p["unit_stages"] * (nu - 1)
        assert p["tail_tiles"] == 0
    # explicit options pass through
    plans, _ = wsm.chain_plan(specs, l2_prefetch_stages=-1, dep_ring_stages=-1, k_order=wsm.K_ORDER_INCREASING)
    assert all(p["l2_prefetch_stages"] == 0 and p["dep_ring_stages"] == 0 and p["k_order"] == 1 for p in plans)


def test_chain_plan_cluster_reduction_applies_only_to_linear_dependent_chains():
    """Cluster reduction is used only on request, and only for a linear
    dependent tensor-core chain: independent tasks, a task that skips its
    predecessor, two-level counters, the FMA path, an explicit split of 8
    units per tile or tail units are refused with WSM_ERR_UNSUPPORTED; a grid
    option is rounded down to whole clusters."""
    ON = wsm.CHAIN_CLUSTER_ON
    lin = [dict(M=16, N=4096, K=4096, dep=i - 1) for i in range(4)]
    assert all(p["cluster"] == 0 for p in wsm.chain_plan(lin)[0])
    assert all(p["cluster"] == 0 for p in wsm.chain_plan(lin, cluster=wsm.CHAIN_CLUSTER_OFF)[0])
    assert all(p["cluster"] == 4 for p in wsm.chain_plan(lin, cluster=ON)[0])
    assert all(p["grid"] == 64 for p in wsm.chain_plan(lin, grid=66, cluster=ON)[0])
    assert all(p["cluster"] == 4 and p["unit_stages"] == 4 for p in wsm.chain_plan(lin, unit_stages=4, cluster=ON)[0])
    indep = [dict(M=16, N=4096, K=4096) for _ in range(4)]
    skip = [dict(M=16, N=4096, K=4096, dep=d) for d in (-1, 0, 0, 2)]
    lin_fma = [dict(M=2, N=4096, K=4096, dep=i - 1) for i in range(4)]
    for bad, kw in ((indep, {}), (skip, {}), (lin, dict(counter_groups=2)), (lin_fma, {}), (lin, dict(unit_stages=2)),
                    (lin, dict(tail_tiles=8))):
        with pytest.raises(wsm.WsmError) as e:
            wsm.chain_plan(bad, cluster=ON, **kw)
        assert e.value.code == wsm.WSM_ERR_UNSUPPORTED, kw
    with pytest.raises(wsm.WsmError) as e:
        wsm.chain_plan(lin, cluster=7)
    assert e.value.code == wsm.WSM_ERR_INVALID


def test_chain_plan_die_groups():
    """Die-grouped claims: each task's tiles split in two contiguous ranges
    (equal dies assumed by host-only planning), no tail units; refused on the
    FMA path, with two-level counters, cluster reduction or dep_cols."""
    specs = [dict(M=m, N=n, K=k, m_tile=0) for m in (32, 64) for (k, n) in QWEN3_LAYER[2:]]
    specs = [dict(M=s["M"], N=s["N"], K=s["K"]) for s in specs]
    plans, _ = wsm.chain_plan(specs, die_groups=wsm.DIE_GROUPS_ON)
    for p in plans:
        tiles = p["n_tiles"] * p["m_tiles"]
        assert p["die_split"] == tiles // 2 or p["die_split"] == (tiles + 1) // 2, p
        assert p["tail_tiles"] == 0
    assert all(p["die_split"] == 0 for p in wsm.chain_plan(specs)[0])  # no M-tiled task: auto leaves it off
    tiled = [dict(s, m_tile=16) for s in specs]
    assert all(p["die_split"] > 0 for p in wsm.chain_plan(tiled)[0])   # M-tiled: auto groups
    assert all(p["die_split"] == 0 for p in wsm.chain_plan(tiled, die_groups=wsm.DIE_GROUPS_OFF)[0])
    lin = [dict(M=16, N=4096, K=4096, dep=i - 1) for i in range(3)]
    for kw in (dict(path=wsm.PATH_STREAM, specs=[dict(M=2, N=4096, K=4096)]), dict(counter_groups=2),
               dict(cluster=wsm.CHAIN_CLUSTER_ON)):
        sp = kw.pop("specs", lin)
        with pytest.raises(wsm.WsmError) as e:
            wsm.chain_plan(sp, die_groups=wsm.DIE_GROUPS_ON, **kw)
        assert e.value.code == wsm.WSM_ERR_UNSUPPORTED, kw


def test_chain_plan_wide_x_and_fma():
    """M = 32 / 64 tasks keep 4 prefetch stages (wider X tiles); a chain of
    M = 1 GEMMs runs on the FMA path in increasing K order, without prefetch,
    its whole ring ahead of a dependency."""
    specs = [dict(M=m, N=n, K=k) for m in (32, 64) for (k, n) in QWEN3_LAYER[2:]]
    plans, _ = wsm.chain_plan(specs)
    for s, p in zip(specs, plans):
        assert p["path"] == wsm.PATH_UMMA and p["l2_prefetch_stages"] == 4 and p["m_tile"] == s["M"]
        assert p["stages"] == 2  # the ring is sized for the widest X tile
    specs = [dict(M=1, N=n, K=k, dep=i - 1) for i, (k, n) in enumerate(QWEN3_LAYER)]
    plans, kernels = wsm.chain_plan(specs)
    assert kernels == 1
    for p in plans:
        assert p["path"] == wsm.PATH_STREAM and p["k_order"] == wsm.K_ORDER_INCREASING
        assert p["l2_prefetch_stages"] == 0 and p["dep_ring_stages"] == 0 and p["tile_rows"] in (16, 32)


def test_chain_plan_hybrid_dispatch():
    """Tasks of M <= 32 and M > 32 in one chain: SPLIT gives one kernel per
    run of one X width (numbered in order), ONE a single kernel sized for the
    widest X tile; AUTO splits only when the narrow runs carry enough weight
    bytes per extra kernel."""
    specs = [dict(M=16, N=4096, K=4096), dict(M=16, N=6144, K=4096, dep=0), dict(M=64, N=4096, K=4096, dep=1),
             dict(M=64, N=4096, K=4096), dict(M=8, N=4096, K=4096, dep=3)]
    plans, kernels = wsm.chain_plan(specs, kernels=wsm.CHAIN_KERNELS_SPLIT)
    assert kernels == 3 and [p["kernel"] for p in plans] == [0, 0, 1, 1, 2]
    assert [p["m_tile"] for p in plans] == [16, 16, 64, 64, 16]
    assert plans[0]["stages"] == 3 and plans[2]["stages"] == 2
    plans, kernels = wsm.chain_plan(specs, kernels=wsm.CHAIN_KERNELS_ONE)
    assert kernels == 1 and all(p["stages"] == 2 and p["kernel"] == 0 for p in plans)
    _, kernels = wsm.chain_plan(specs)
    assert kernels == 1  # 0.1 GB of narrow weights: not worth two extra kernel boundaries


def test_chain_plan_column_dependencies_keep_increasing_order():
    specs = [dict(M=16, N=2048, K=1024), dict(M=16, N=1024, K=2048, dep=0, dep_cols=True)]
    plans, _ = wsm.chain_plan(specs)
    assert all(p["k_order"] == wsm.K_ORDER_INCREASING for p in plans)
    assert plans[1]["tail_tiles"] == 0


def test_chain_plan_errors():
    specs = [dict(M=16, N=4096, K=4096), dict(M=16, N=4096, K=4096, dep=0)]
    for kw, code in ((dict(path=3), wsm.WSM_ERR_INVALID), (dict(kernels=3), wsm.WSM_ERR_INVALID),
                     (dict(flags=4), wsm.WSM_ERR_INVALID), (dict(l2_prefetch_stages=-2), wsm.WSM_ERR_INVALID),
                     (dict(k_order=3), wsm.WSM_ERR_INVALID), (dict(dep_ring_stages=-2), wsm.WSM_ERR_INVALID),
                     (dict(counter_groups=-1), wsm.WSM_ERR_INVALID), (dict(tile_rows=64), wsm.WSM_ERR_UNSUPPORTED),
                     (dict(path=wsm.PATH_STREAM), wsm.WSM_ERR_UNSUPPORTED),  # M = 16 on the FMA path
                     (dict(num_sms=0), wsm.WSM_ERR_INVALID)):
        with pytest.raises(wsm.WsmError) as e:
            wsm.chain_plan(specs, **kw)
        assert e.value.code == code, kw
    with pytest.raises(wsm.WsmError) as e:
        wsm.chain_plan([dict(M=16, N=4096, K=4096, dep=0)])  # a task may not wait for itself
    assert e.value.code == wsm.WSM_ERR_INVALID
