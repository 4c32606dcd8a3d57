"""The column-parallel (N-sharded) path on the GPU, against the fp64 oracle.

Each rank of a column split streams a contiguous block of every weight's
rows with the library's kernels and the blocks are assembled into the full
Y.  One GPU stands in for the ranks: the shards of a 1-, 2- and 3-way split
are computed one after another through ShardedLinear (its default per-rank
compute is the library's skinny_gemm) or through one chain kernel per rank
(the benchmark's nshard step), then concatenated in shard order -- the
assembly the all-gather performs across GPUs -- and compared element by
element with the oracle, plain and with the fused SiLU*mul weight.  The
all-gather itself runs once through NCCL in a one-rank process group."""
import socket
from datetime import timedelta

import pytest
import torch

import oracle
import synth
import weight_streaming_megakernel_b200 as wsm
from parity import check_bounded, check_full
from weight_streaming_megakernel_b200.shard import ShardedLinear, column_shards, gather_columns

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def _assemble(parts, shards, M):
    out = torch.cat([p[:, : n1 - n0] for p, (n0, n1) in zip(parts, shards)], dim=1)
    assert out.shape[0] == M
    return out


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 6144, 4096), (8, 2112, 7168), (64, 1000, 2048)])
def test_sharded_linear_matches_oracle(world, M, N, K):
    x, w = synth.make_xw(M, N, K, seed=world * 100 + M)
    xd, wd = x.to(DEV), w.to(DEV)
    lins = [ShardedLinear(wd, r, world, align=128) for r in range(world)]
    parts = [lin.forward(xd, gather=False) for lin in lins]
    torch.cuda.synchronize()
    assert wsm.stream_status() == 0
    y = _assemble(parts, lins[0].out_shards, M)
    assert y.shape == (M, N)
    check_full(x, w, y, what=f"{world}-way column split M={M} N={N} K={K}")


@pytest.mark.parametrize("world,align", [(1, 16), (2, 16), (2, 128), (3, 32)])
@pytest.mark.parametrize("M", [2, 16])
def test_sharded_silu_mul_matches_oracle(world, align, M):
    """The fused gate+up weight split by output columns: every block holds
    whole gate/up pairs (align a multiple of 16), so each rank's SiLU*mul
    output is its slice of H."""
    N, K = 2 * 1040, 1032
    x, w = synth.make_xw(M, N, K, seed=world + align + M)
    xd, wd = x.to(DEV), w.to(DEV)

    def silu_gemm(xx, ww):
        return wsm.skinny_gemm(xx, ww, epilogue=wsm.EPI_SILU_MUL)

    lins = [ShardedLinear(wd, r, world, align=align, compute=silu_gemm, out_div=2) for r in range(world)]
    parts = [lin.forward(xd, gather=False) for lin in lins]
    torch.cuda.synchronize()
    h = _assemble(parts, lins[0].out_shards, M)
    H, G, U, Sg, Su = oracle.silu_mul_ref(x, w)
    check_bounded(h, None, H, oracle.fused_bounds("silu_mul", G=G, U=U, Sg=Sg, Su=Su),
                  f"{world}-way SiLU*mul split, align {align}")


@pytest.mark.parametrize("world", [1, 2])
def test_sharded_chain_step_matches_oracle(world):
    """The benchmark's nshard step: each rank runs one chain kernel over its
    blocks of every weight (here a decode layer's four GEMMs at M = 16)."""
    M = 16
    shapes = [(6144, 4096), (4096, 4096), (24576, 4096), (4096, 12288)]
    xs = [synth.make_x(M, K, seed=i) for i, (N, K) in enumerate(shapes)]
    ws = [synth.make_w(N, K, seed=50 + i) for i, (N, K) in enumerate(shapes)]
    xds = [x.to(DEV) for x in xs]
    wds = [w.to(DEV) for w in ws]
    outs = [[] for _ in shapes]
    for r in range(world):
        tasks = []
        for i, (N, K) in enumerate(shapes):
            n0, n1 = column_shards(N, world, 128)[r]
            tasks.append(wsm.Task(xds[i], wds[i][n0:n1].contiguous(),
                                  torch.full((M, n1 - n0), float("nan"), dtype=torch.bfloat16, device=DEV)))
        ch = wsm.Chain(tasks, flags=wsm.FLAG_W_READONLY)
        ch.run()
        assert ch.status()[0] == wsm.WSM_OK
        for i, t in enumerate(tasks):
            outs[i].append(t.y)
        ch.close()
    for i, (N, K) in enumerate(shapes):
        y = _assemble(outs[i], column_shards(N, world, 128), M)
        check_full(xs[i], ws[i], y, what=f"{world}-way chain task {i}")


def test_gather_columns_through_nccl_one_rank():
    """gather_columns through a real NCCL all-gather (a one-rank group): the
    padded exchange buffer and the reassembly keep every bit."""
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group already exists in this process")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60), device_id=torch.device(DEV))
    try:
        M, N, K = 16, 6144, 4096
        x, w = synth.make_xw(M, N, K, seed=77)
        xd, wd = x.to(DEV), w.to(DEV)
        lin = ShardedLinear(wd, 0, 1, align=128)
        y_local = lin.forward(xd, gather=False)
        y = gather_columns(y_local, lin.out_shards)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_local.view(torch.int16))
        check_full(x, w, y, what="gathered")
    finally:
        dist.destroy_process_group()
