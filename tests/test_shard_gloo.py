"""Column-parallel sharding across ranks (host logic, CPU only).

The shard boundaries are checked directly; the all-gather and the
max-over-ranks timing are run as two gloo processes on the CPU, with an exact
stand-in for the per-rank GEMM (fp64 products of small integers), so the
gathered result must equal the unsharded one bit for bit.  The same code runs
with NCCL and the library's GEMM on GPUs.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from weight_streaming_megakernel_b200.shard import ShardedLinear, column_shards, max_over_ranks


@pytest.mark.parametrize("N,world,align", [(4096, 2, 128), (4096, 8, 128), (1000, 2, 128), (1000, 3, 16),
                                           (24576, 8, 16), (100, 4, 128), (0, 2, 16), (6144, 7, 128)])
def test_column_shards_cover_once_aligned_balanced(N, world, align):
    sh = column_shards(N, world, align)
    assert len(sh) == world
    assert sh[0][0] == 0 and sh[-1][1] == N
    for (a0, a1), (b0, b1) in zip(sh, sh[1:]):
        assert a1 == b0 and a0 <= a1
    for n0, n1 in sh:
        assert (n0 % align == 0 or n0 == N) and (n1 % align == 0 or n1 == N)
    units = [-(-(n1 - n0) // align) for n0, n1 in sh]
    assert max(units) - min(units) <= 1


def _exact_compute(x, w):
    # exact for small-integer inputs: fp64 products and sums
    return (x.double() @ w.double().T).to(torch.float64)


def _exact_silu_pair(x, w):
    # the fused gate+up layout at block size 8: gate rows 16b..16b+7, up rows 16b+8..16b+15
    y = x.double() @ w.double().T
    gi, ui = oracle.gate_up_rows(y.shape[1] // 2)
    return y[:, gi] * y[:, ui]      # the product pairing only (silu itself is not sharding logic)


def _worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
        x, w = synth.make_int_xw(3, 1000, 256, seed=7)
        lin = ShardedLinear(w, rank, world, align=16, compute=_exact_compute)
        full = lin.forward(x)
        xg, wg = synth.make_int_xw(2, 96, 64, seed=8)
        lin2 = ShardedLinear(wg, rank, world, align=16, compute=_exact_silu_pair, out_div=2)
        h = lin2.forward(xg)
        t = max_over_ranks(1.5 + rank)
        q.put((rank, full.numpy(), h.numpy(), t))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, repr(e), None, None))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_linear_gathers_full_result(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, full, h, t = q.get(timeout=120)
        assert h is not None, full
        out[rank] = (full, h, t)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, w = synth.make_int_xw(3, 1000, 256, seed=7)
    ref = _exact_compute(x, w).numpy()
    xg, wg = synth.make_int_xw(2, 96, 64, seed=8)
    href = _exact_silu_pair(xg, wg).numpy()
    for rank, (full, h, t) in out.items():
        assert np.array_equal(full, ref), rank
        assert np.array_equal(h, href), rank
        assert t == 1.5 + (world - 1)
