"""The SM -> die map and die-grouped claims, and M-tiled chain tasks.

wsm_sm_die_map measures which die each SM sits on from L2-hit latencies;
checked for a clean two-way split (every SM labelled, both dies populated,
far lines slower than near ones) and for caching.  A chain with die_groups
claims each task's tiles from its die's range first and then helps with the
other range; the work units are the same as without grouping, so the results
must match the ungrouped chain bit for bit and the oracle element by element.
Chain tasks with an M-tile (X rows split into several tiles that share each
weight column) are checked against the oracle too."""
import pytest
import torch

import synth
import weight_streaming_megakernel_b200 as wsm
from parity import bf16_bits, check_full

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def test_sm_die_map():
    die, info = wsm.sm_die_map()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ids = [i for i, d in enumerate(die) if d >= 0]
    print("die probe:", info)
    assert len(ids) == sms == info["num_sms"]
    assert {die[i] for i in ids} <= {0, 1}
    if info["dies"] == 2:
        assert info["sms_die0"] + info["sms_die1"] == sms and min(info["sms_die0"], info["sms_die1"]) > 0
        assert info["agreement"] >= 0.75
        assert info["far_cycles"] > info["near_cycles"] > 0
        assert sum(1 for i in ids if die[i] == 1) == info["sms_die1"]
    else:
        assert all(die[i] == 0 for i in ids)
    assert wsm.sm_die_map()[0] == die


def _tasks(cases, seed):
    out = []
    for i, (M, N, K, tm) in enumerate(cases):
        x, w = synth.make_xw(M, N, K, seed=seed + i)
        out.append((x, w, wsm.Task(x.to(DEV), w.to(DEV), torch.full((M, N), float("nan"), dtype=torch.bfloat16,
                                                                     device=DEV),
                                   yf32=torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV),
                                   m_tile=tm)))
    return out


CASES = [(32, 3072, 4096, 16), (64, 2048, 1536, 16), (64, 1024, 6144, 32), (48, 4096, 1024, 16), (17, 520, 1032, 16)]


@pytest.mark.parametrize("deps", [False, True])
def test_die_grouped_chain_matches_oracle_and_ungrouped(deps):
    ts = _tasks(CASES, seed=11)
    tasks = [t for _, _, t in ts]
    if deps:
        for i, t in enumerate(tasks):
            t.dep = i - 1
    plain = wsm.Chain(tasks, path=wsm.PATH_UMMA, die_groups=wsm.DIE_GROUPS_OFF)
    plain.run()
    assert plain.status()[0] == wsm.WSM_OK
    ref = [(bf16_bits(t.y).copy(), t.yf32.cpu().clone()) for t in tasks]
    plans = [plain.task_plan(i) for i in range(len(tasks))]
    plain.close()
    for t in tasks:
        t.y.fill_(float("nan"))
        t.yf32.fill_(float("nan"))
    ch = wsm.Chain(tasks, path=wsm.PATH_UMMA, die_groups=wsm.DIE_GROUPS_ON)
    for i, (M, N, K, tm) in enumerate(CASES):
        p = ch.task_plan(i)
        assert p["units"] == plans[i]["units"] and p["m_tiles"] == -(-M // tm)
    s = torch.cuda.Stream()
    for rep in range(2):
        s.wait_stream(torch.cuda.current_stream())
        ch.run(s)
        assert ch.status(s)[0] == wsm.WSM_OK
        for i, ((x, w, t), (yb, yf)) in enumerate(zip(ts, ref)):
            check_full(x, w, t.y, t.yf32, what=f"die-grouped task {i} run {rep}")
            assert (bf16_bits(t.y) == yb).all(), f"task {i}: bits differ from ungrouped claims"
            assert torch.equal(t.yf32.cpu().view(torch.int32), yf.view(torch.int32))
            t.y.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ch.run(s)
    for rep in range(2):
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            g.replay()
        s.synchronize()
        assert ch.status(s)[0] == wsm.WSM_OK
        for i, (x, w, t) in enumerate(ts):
            check_full(x, w, t.y, t.yf32, what=f"die-grouped task {i} replay {rep}")
    del g
    ch.close()


@pytest.mark.parametrize("tm", [16, 32])
def test_m_tiled_chain_tasks_match_oracle(tm):
    """The M-tile of each chain task: X rows in tiles of tm, every weight
    column read by all of them (M-major), as in the L2-reuse configuration."""
    cases = [(M, N, K, tm) for (M, N, K, _) in CASES]
    ts = _tasks(cases, seed=40 + tm)
    ch = wsm.Chain([t for _, _, t in ts], path=wsm.PATH_UMMA)
    for i, (M, N, K, _) in enumerate(cases):
        assert ch.task_plan(i)["m_tiles"] == -(-M // tm)
    ch.run()
    assert ch.status()[0] == wsm.WSM_OK
    for i, (x, w, t) in enumerate(ts):
        check_full(x, w, t.y, t.yf32, what=f"m_tile {tm} task {i}")
    ch.close()
