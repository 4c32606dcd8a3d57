"""Benchmark of the weight-streaming decode GEMM on B200.

One step = every GEMM of the workload once (default: the Qwen3-8B-shaped decode
GEMMs -- fused QKV, o, fused gate_up, down -- at M = 1, 2, 4, 8, 16; 20 GEMMs,
each with its own weight matrix, 1.93 GB of distinct weights per step, so the
inputs are larger than L2 and no flush is needed).  The metric is achieved HBM
bandwidth: algorithmic bytes (W + X read once) / time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl wsm|reference]
                  [--workload qwen3_decode|single|skinny|l2_reuse|chain]

Prints ONE JSON line on rank 0.  With N > 1 (launched by torchrun) every rank
runs an independent replica of the workload on its own GPU (the GEMMs do not
shard across GPUs); value = all ranks' bytes / the slowest rank's time.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "achieved HBM GB/s (% of peak) and µs per bf16 decode GEMM at M=1–64 on 1 B200"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def kernel_source_hash():
    """sha256 over the CUDA sources (name + bytes, sorted): identifies the
    kernel build a stored DRAM-traffic figure was taken from."""
    import hashlib
    d = os.path.join(ROOT, "weight_streaming_megakernel_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(d)):
        if name.endswith((".cu", ".cuh")):
            h.update(name.encode())
            with open(os.path.join(d, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()


def stored_traffic(kernel, workload, mode):
    """DRAM bytes (read + write) of one launch of `kernel`, from the ncu
    summary under profiles/ -- only if it was taken from the current sources."""
    path = os.path.join(ROOT, "profiles", f"traffic_{kernel}_{workload}_{mode}.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("csrc_sha256") != kernel_source_hash():
            return None
        return int(kv["dram__bytes_read.sum"]) + int(kv["dram__bytes_write.sum"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_cases(name):
    if name == "qwen3_decode":
        return synth.config_qwen3_decode()
    if name == "single":
        return synth.config_single()
    if name == "skinny":
        return synth.config_skinny()
    if name == "l2_reuse":
        return synth.config_l2_reuse()
    if name == "l2_reuse_whole_m":
        return synth.config_l2_reuse(m_tiles=(0,))
    if name == "chain":
        return synth.chain_layout()
    raise SystemExit(f"unknown workload {name}")


L2_BYTES = 126 * 2 ** 20


def n_copies(cases, min_calls=1):
    """Weight copies a step cycles through so that consecutive steps touch at
    least 4x the L2 size (1 when one step's weights already do), and a GEMM's
    weights come back only after `min_calls` launches: independent launches
    run several at a time, and two of them on the same copy would share its
    weights through L2."""
    w = sum(2 * c.N * c.K for c in cases)
    return max(1, -(-4 * L2_BYTES // w), -(-min_calls // len(cases)))


# independent launches in flight at once: about SMs / grid (4-5 at a quarter of the SMs); a weight copy
# comes back only after twice that many
INDEPENDENT_REUSE_CALLS = 10


def alg_bytes(c):
    """Algorithmic bytes of one GEMM: W read once + X read once (bf16)."""
    return 2 * c.N * c.K + 2 * c.M * c.K


def out_bytes(c):
    return 2 * c.M * c.N


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        time.sleep(0.05)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm),
                "window": "loaded window containing the timed region"}


# ----------------------------------------------------------------------------- GPU arm

def setup_inputs(cases, dev, seed_base=0):
    """Seeded device inputs per GEMM (generated on the device: same recipe,
    X ~ N(0,1), W ~ N(0,1/K), fp32 rounded to bf16).  The X of all GEMMs are
    slices of one buffer and so are the Y (each slice 16-byte aligned), so a
    step's inputs and results move between host and device in one copy each."""
    def offsets(sizes):
        out, at = [], 0
        for n in sizes:
            out.append(at)
            at += -(-n // 8) * 8          # 8 bf16 = 16 bytes
        return out, at
    xo, xn = offsets([c.M * c.K for c in cases])
    yo, yn = offsets([c.M * c.N for c in cases])
    xbuf = torch.empty(xn, dtype=torch.bfloat16, device=dev)
    ybuf = torch.empty(yn, dtype=torch.bfloat16, device=dev)
    data = []
    for i, c in enumerate(cases):
        g = torch.Generator(device=dev)
        g.manual_seed(seed_base * 100003 + i * 7919 + c.seed)
        x = xbuf[xo[i]: xo[i] + c.M * c.K].view(c.M, c.K)
        x.copy_(torch.randn(c.M, c.K, generator=g, device=dev).to(torch.bfloat16))
        w = (torch.randn(c.N, c.K, generator=g, device=dev) * (1.0 / c.K ** 0.5)).to(torch.bfloat16)
        y = ybuf[yo[i]: yo[i] + c.M * c.N].view(c.M, c.N)
        data.append((c, x, w, y))
    return data


def packed(data, which):
    """The one buffer the X (which=1) or Y (which=3) of all GEMMs are slices of."""
    t = data[0][which]
    return t.as_strided((t.untyped_storage().nbytes() // 2,), (1,), 0)


def run_e2e(args, wsm, dev, datas, copies, mode, total_bytes, world, stream, n_steps):
    """The step through the public API with its inputs in pinned host memory:
    every step copies its X in (one copy of the packed X) and its Y out (one
    copy), inside the timed region.  The copies run on their own streams,
    double-buffered (two device X/Y buffer sets and two host buffer pairs),
    so step k's kernel overlaps step k + 1's input copy and step k - 1's
    result copy, as a serving loop would; the region ends when the last
    step's result is on the host."""
    slots = 2
    hx = [packed(datas[0], 1).cpu().pin_memory() for _ in range(slots)]
    hy = [torch.empty(packed(datas[0], 3).numel(), dtype=torch.bfloat16).pin_memory() for _ in range(slots)]
    h2d, d2h = hx[0].numel() * 2, hy[0].numel() * 2
    # device X / Y of each slot, laid out like the packed buffers, and the step's GEMMs bound to them
    xs = [torch.empty_like(packed(datas[0], 1)) for _ in range(slots)]
    ys = [torch.empty_like(packed(datas[0], 3)) for _ in range(slots)]

    def view(buf, ref):  # the slice of `buf` at the place `ref` has in its packed buffer
        off = ref.storage_offset()
        return buf[off: off + ref.numel()].view(ref.shape)

    s = stream.cuda_stream
    runs = {}
    for j in range(slots):
        for r in range(copies):
            gemms = [(c, view(xs[j], x), w, view(ys[j], y)) for c, x, w, y in datas[r]]
            if mode == "chain":
                deps = [(i - 1) if args.workload == "chain" else -1 for i in range(len(gemms))]
                ch = wsm.Chain([wsm.Task(x, w, y, dep=deps[i], m_tile=c.m_tile) for i, (c, x, w, y) in enumerate(gemms)],
                               flags=wsm.FLAG_W_READONLY, die_groups=args.die_groups, cluster=args.cluster)
                runs[j, r] = (lambda ch=ch: ch.run(s), ch)
            else:
                def go(gemms=gemms):
                    for c, x, w, y in gemms:
                        wsm.skinny_gemm(x, w, y, m_tile=c.m_tile, flags=wsm.FLAG_W_READONLY, stream=s)
                runs[j, r] = (go, None)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    x_in = [ev() for _ in range(slots)]     # slot's X landed
    done = [ev() for _ in range(slots)]     # slot's kernels finished (its X may be overwritten)
    y_out = [ev() for _ in range(slots)]    # slot's Y copied out (its Y may be overwritten)
    used = [False] * slots

    def e2e_step(k):
        j, r = k % slots, k % copies
        if used[j]:
            up.wait_event(done[j])
        with torch.cuda.stream(up):
            xs[j].copy_(hx[j], non_blocking=True)
            x_in[j].record(up)
        stream.wait_event(x_in[j])
        if used[j]:
            stream.wait_event(y_out[j])
        runs[j, r][0]()
        done[j].record(stream)
        down.wait_event(done[j])
        with torch.cuda.stream(down):
            hy[j].copy_(ys[j], non_blocking=True)
            y_out[j].record(down)
        used[j] = True

    for k in range(max(1, args.warmup)):
        e2e_step(k)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_event(a)
    for k in range(n_steps):
        e2e_step(k)
    for j in range(slots):
        stream.wait_event(y_out[j])
    b.record(stream)
    torch.cuda.synchronize(dev)
    e_ms = a.elapsed_time(b)
    if world > 1:
        tt = torch.tensor([e_ms], device=dev)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        e_ms = float(tt.item())
    for _, ch in runs.values():
        if ch is not None:
            if ch.status(s)[0] != 0:
                raise RuntimeError("device-side status in the e2e run")
            ch.close()
    return {"value": round(total_bytes * world / (e_ms / n_steps * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "overlap": "copies on their own streams, double-buffered across steps"}


def back_to_back_per_shape(args, dev, hbm_peak, independent, grid, launches=32, replays=3):
    """Each GEMM of the workload on its own: `launches` back-to-back
    skinny_gemm launches of that one shape in a CUDA graph, cycling through
    weight copies larger than 4x L2 together; device time per launch (CUDA
    events around `replays` replays) and its fraction of the measured peak.
    With `independent`, every launch carries WSM_FLAG_INDEPENDENT (the copies
    share no buffers) on `grid` CTAs."""
    import ctypes
    import weight_streaming_megakernel_b200 as wsm
    L = wsm.lib()
    stream = torch.cuda.Stream(dev)
    out = {}
    for c in workload_cases(args.workload):
        copies = n_copies([c], INDEPENDENT_REUSE_CALLS if independent else 1)
        datas = [setup_inputs([c], dev, seed_base=7 + r) for r in range(copies)]
        fl = wsm.FLAG_W_READONLY | (wsm.FLAG_INDEPENDENT if independent else 0)
        o = wsm._opts(m_tile=c.m_tile, flags=fl, grid=grid)
        ptrs = [(d[0][1].data_ptr(), d[0][2].data_ptr(), d[0][3].data_ptr()) for d in datas]

        def run():
            for i in range(launches):
                xp, wp, yp = ptrs[i % copies]
                if L.skinny_gemm_ex(xp, wp, yp, c.M, c.N, c.K, ctypes.byref(o), stream.cuda_stream) != 0:
                    raise RuntimeError(f"skinny_gemm failed: {wsm.last_error()}")

        stream.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(stream):
            run()                         # eager: sizes the stream's scratch before the capture
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g.replay()
            e0.record(stream)
            for _ in range(replays):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (replays * launches)
        out[c.name] = {"us": round(us, 2), "frac_of_peak": round(alg_bytes(c) / (us * 1e-6) / 1e9 / hbm_peak, 4)}
        del g, datas
    if wsm.stream_status(stream) != 0:
        raise RuntimeError("device-side status in the per-shape runs")
    return out


def run_gpu(args, rank, world, local_rank, mode=None, steps=None, extras=True):
    """Timed region: K steps, each one replay of a CUDA graph holding every
    GEMM launch of the step with an external timing event between launches
    (so per-launch durations come from the same timed replays)."""
    import ctypes
    import weight_streaming_megakernel_b200 as wsm

    mode = mode or args.mode
    n_steps = steps or args.steps
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cases = workload_cases(args.workload)
    if args.only:
        cases = [c for c in cases if c.name in args.only.split(",")]
        assert cases, f"no case named {args.only}"
    # Inputs larger than L2 between timed steps: a step whose weights fit in
    # L2 several times cycles through copies (step k uses copy k % copies).
    copies = n_copies(cases, INDEPENDENT_REUSE_CALLS if mode == "launches" and args.independent else 1)
    datas = [setup_inputs(cases, dev, seed_base=rank * 1000 + r) for r in range(copies)]
    data = datas[0]
    cur = [0]  # copy the next launches use
    L = wsm.lib()
    stream = torch.cuda.Stream(dev)
    s = stream.cuda_stream
    chain = None

    if mode == "chain":
        # the whole step is one persistent kernel; the layer chain orders task t after t-1
        deps = [(i - 1) if args.workload == "chain" else -1 for i in range(len(data))]
        chains = [wsm.Chain([wsm.Task(x, w, y, dep=deps[i], m_tile=c.m_tile) for i, (c, x, w, y) in enumerate(d)],
                            flags=wsm.FLAG_W_READONLY, die_groups=args.die_groups, cluster=args.cluster)
                  for d in datas]
        chain = chains[0]
        launches_per_step = 1

        def launch(i):
            chains[cur[0]].run(s)
    else:
        callsets = []
        for d in datas:
            calls = []
            for c, x, w, y in d:
                # independent launches: every GEMM of a step and every copy has its own X, W and Y
                fl = wsm.FLAG_W_READONLY | (wsm.FLAG_INDEPENDENT if args.independent else 0)
                o = wsm._opts(m_tile=c.m_tile, flags=fl, grid=args.grid)
                calls.append((x.data_ptr(), w.data_ptr(), y.data_ptr(), c.M, c.N, c.K, o))
            callsets.append(calls)
        launches_per_step = len(callsets[0])

        def launch(i):
            xp, wp, yp, M, N, K, o = callsets[cur[0]][i]
            rc = L.skinny_gemm_ex(xp, wp, yp, M, N, K, ctypes.byref(o), s) if o is not None else \
                L.skinny_gemm(xp, wp, yp, M, N, K, s)
            if rc != 0:
                raise RuntimeError(f"skinny_gemm failed: {wsm.last_error()}")

    def step(events=None):
        for i in range(launches_per_step):
            if events is not None:
                events[i].record(stream)
            launch(i)
        if events is not None:
            events[launches_per_step].record(stream)

    total_bytes = sum(alg_bytes(c) for c in cases)

    # eager warm-up (also sizes the stream's scratch before any capture)
    with torch.cuda.stream(stream):
        for k in range(max(args.warmup, copies)):
            cur[0] = k % copies
            step()
    stream.synchronize()

    # one graph per timed step, each with its own in-graph timing events
    nev = launches_per_step + 1
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(nev)] for _ in range(n_steps)]
    graphs = []
    for k in range(n_steps):
        cur[0] = k % copies
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(evs[k])
        graphs.append(g)
    plain = torch.cuda.CUDAGraph()  # all copies once each
    with torch.cuda.graph(plain, stream=stream):
        for r in range(copies):
            cur[0] = r
            step()
    # the timed region: the K steps back to back in ONE graph, no events inside (launches keep their
    # programmatic overlap across steps and pay one graph launch for all of them)
    timed = torch.cuda.CUDAGraph()
    with torch.cuda.graph(timed, stream=stream):
        for k in range(n_steps):
            cur[0] = k % copies
            step()
    with torch.cuda.stream(stream):
        timed.replay()
        for g in graphs[: min(3, len(graphs))]:
            g.replay()
    stream.synchronize()

    # clocks: the sampler runs over a loaded window that contains the timed region
    clocks = ClockSampler(local_rank)
    if extras:
        clocks.start()
    t_pre = time.time()
    with torch.cuda.stream(stream):
        while extras and len(clocks.lines) < 2 and time.time() - t_pre < 3.0:
            plain.replay()
            stream.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        timed.replay()
        t_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    # per-launch durations (outside the timed region): the instrumented graphs, events between launches
    with torch.cuda.stream(stream):
        for g in graphs:
            g.replay()
    stream.synchronize()
    # keep the load on briefly so the window closes under load
    t_post = time.time()
    with torch.cuda.stream(stream):
        while extras and time.time() - t_post < 0.3:
            plain.replay()
            stream.synchronize()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    if world > 1:
        tt = torch.tensor([total_ms], device=dev)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(tt.item())
    ms_per_step = total_ms / n_steps
    per_launch = [[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(launches_per_step)]
                  for k in range(n_steps)]

    # uninstrumented graph, for reference (not the headline)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(n_steps):
            plain.replay()
        b.record(stream)
    stream.synchronize()
    plain_ms = a.elapsed_time(b) / (n_steps * copies)

    # ---- e2e: public API, host buffers, H2D of X and D2H of Y inside the timed region
    e2e = None
    if extras and not args.no_e2e:
        e2e = run_e2e(args, wsm, dev, datas, copies, mode, total_bytes, world, stream, n_steps)

    status = wsm.stream_status(stream) if chain is None else max(c.status(s)[0] for c in chains)
    if status != 0:
        raise RuntimeError(f"device-side status {status}")
    del graphs, plain, timed
    return dict(cases=cases, total_bytes=total_bytes, ms_per_step=ms_per_step, per_launch=per_launch,
                clocks=clk, e2e=e2e, launches_per_step=launches_per_step, chain=chain is not None,
                plain_ms=plain_ms, copies=copies)


def run_nshard(args, rank, world, local_rank):
    """Column-parallel step (--parallel nshard): every rank streams its block
    of output columns of every weight (one chain kernel over the blocks), then
    one all-gather per GEMM assembles the full Y on every rank.  Timed eagerly
    (the collectives are not captured in a graph): K steps between a barrier
    and a synchronize, max over ranks."""
    import weight_streaming_megakernel_b200 as wsm
    from weight_streaming_megakernel_b200.shard import column_shards, gather_columns, max_over_ranks

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cases = workload_cases(args.workload)
    if args.only:
        cases = [c for c in cases if c.name in args.only.split(",")]
    full_bytes = sum(alg_bytes(c) for c in cases)
    shards = [column_shards(c.N, world, 128) for c in cases]
    local = []
    for c, sh in zip(cases, shards):
        n0, n1 = sh[rank]
        local.append(synth.Case(c.name, c.M, max(n1 - n0, 1), c.K, c.seed, c.m_tile))
    data = setup_inputs(local, dev, seed_base=rank)
    deps = [(i - 1) if args.workload == "chain" else -1 for i in range(len(data))]
    chain = wsm.Chain([wsm.Task(x, w, y, dep=deps[i], m_tile=c.m_tile) for i, (c, x, w, y) in enumerate(data)],
                      flags=wsm.FLAG_W_READONLY)
    stream = torch.cuda.Stream(dev)

    def step():
        chain.run(stream.cuda_stream)
        if world > 1:
            for (c, x, w, y), sh in zip(data, shards):
                gather_columns(y[:, : sh[rank][1] - sh[rank][0]], sh)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
    stream.synchronize()
    total_ms = a.elapsed_time(b)
    if world > 1:
        torch.distributed.barrier()
        total_ms = max_over_ranks(total_ms, device=dev)
    if chain.status(stream.cuda_stream)[0] != 0:
        raise RuntimeError("device-side status")
    chain.close()
    return full_bytes, total_ms / args.steps


def trace_boundaries(args):
    """Diagnostic (not a bench line for the driver): run the dependent layer
    chain once with per-CTA trace stamps and report, per GEMM kind, the median
    over layers of where a task's time goes, in microseconds from the moment
    its dependency was met (median over CTAs): the accumulators reaching the
    epilogue (median and last CTA), the last split-K arrival, the last
    reduction, the last outputs written, the next task's dependency met and
    its first stage at the MMA issuer.  Prints one JSON line."""
    import statistics
    import weight_streaming_megakernel_b200 as wsm
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cases = workload_cases(args.workload)
    data = setup_inputs(cases, dev)
    tasks = [wsm.Task(x, w, y, dep=i - 1, m_tile=c.m_tile) for i, (c, x, w, y) in enumerate(data)]
    ch = wsm.Chain(tasks, flags=wsm.FLAG_W_READONLY, trace=True, cluster=args.cluster)
    s = torch.cuda.Stream(dev)
    for _ in range(max(3, args.warmup)):
        ch.run(s)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        a.record(s)
        ch.run(s)
        b.record(s)
    s.synchronize()
    tr = ch.trace(s).double()
    if ch.status(s)[0] != 0:
        raise RuntimeError("device-side status")
    plan0 = ch.task_plan(0)
    ch.close()

    def col(t, i):
        v = tr[:, t, i]
        return v[v > 0]
    kinds = {}
    for t in range(1, len(cases) - 1):
        kind = cases[t].name.split("_", 1)[1] if "_" in cases[t].name else cases[t].name
        acc, dep, nxt, mma = col(t, 4), col(t, 1), col(t + 1, 1), col(t + 1, 7)
        if min(len(acc), len(dep), len(nxt), len(mma)) == 0:
            continue
        t0 = float(dep.median())
        us = lambda v: (float(v) - t0) / 1e3  # noqa: E731
        row = {"acc_median": us(acc.median()), "acc_last": us(acc.max()), "outputs_last": us(col(t, 2).max()),
               "next_dependency_met": us(nxt.median()), "next_first_stage_at_mma": us(mma.median())}
        if len(col(t, 5)):
            row["arrival_last"] = us(col(t, 5).max())
        if len(col(t, 6)):
            row["reduction_last"] = us(col(t, 6).max())
        kinds.setdefault(kind, []).append(row)
    out = {k: {f: round(statistics.median(r[f] for r in rows if f in r), 2) for f in rows[0]}
           for k, rows in kinds.items()}
    print(json.dumps({"diagnostic": "boundary_trace", "workload": args.workload, "cluster": args.cluster,
                      "grid": plan0["grid"], "chain_ms_traced": round(a.elapsed_time(b), 4),
                      "us_from_dependency_met": out}))


def trace_launches(args):
    """Diagnostic (not a bench line for the driver): back-to-back launches of
    each GEMM of the workload, each launch a one-task chain (the same kernels,
    plan and programmatic-launch overlap as skinny_gemm with the W read-only
    flag, plus per-CTA trace stamps that are never cleared between runs, so no
    memset separates the launches), cycling through weight copies larger
    than L2 and replayed as one CUDA graph.  Reports per GEMM, in
    microseconds, medians over the launches: the launch slot (last outputs of
    one launch to the last outputs of the next), the span from a launch's
    first CTA issuing its first stage to its last outputs, how long after the
    previous launch's last outputs its first CTA and its median CTA started,
    and each CTA's busy time (first stage to its last outputs).  Prints one
    JSON line."""
    import statistics
    import weight_streaming_megakernel_b200 as wsm
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    out = {}
    for case in workload_cases(args.workload):
        if args.only and case.name not in args.only.split(","):
            continue
        copies = n_copies([case])
        datas = [setup_inputs([case], dev, seed_base=r) for r in range(copies)]
        chains = [wsm.Chain([wsm.Task(x, w, y, m_tile=c.m_tile)], flags=wsm.FLAG_W_READONLY, trace=2)
                  for d in datas for (c, x, w, y) in d]
        s = torch.cuda.Stream(dev)
        n_launch = max(2 * copies, 16)
        for ch in chains:
            ch.run(s)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for k in range(n_launch):
                chains[k % copies].run(s)
        with torch.cuda.stream(s):
            g.replay()
        s.synchronize()
        # each chain's trace holds its last launch: the final `copies` launches of the replay, in order
        order = [(n_launch - copies + j) % copies for j in range(copies)]
        stamps = [chains[i].trace(s).double()[:, 0, :] for i in order]
        plan = chains[0].task_plan(0)
        for ch in chains:
            if ch.status(s)[0] != 0:
                raise RuntimeError("device-side status")
            ch.close()
        del g
        rows = []
        for j in range(1, copies):
            prev, cur = stamps[j - 1], stamps[j]
            pe = prev[:, 2][prev[:, 2] > 0].max()
            c0, c2 = cur[:, 0], cur[:, 2]
            ok = (c0 > 0) & (c2 > 0)
            rows.append({"slot": float(c2[ok].max() - pe) / 1e3,
                         "span": float(c2[ok].max() - c0[ok].min()) / 1e3,
                         "first_cta_start_after_prev_end": float(c0[ok].min() - pe) / 1e3,
                         "median_cta_start_after_prev_end": float(c0[ok].median() - pe) / 1e3,
                         "cta_busy_median": float((c2[ok] - c0[ok]).median()) / 1e3,
                         "ctas": int(ok.sum())})
        out[case.name] = {k: round(statistics.median(r[k] for r in rows), 2) for k in rows[0]}
        out[case.name].update(path="umma" if plan["path"] == 2 else "fma", units=plan["units"], grid=plan["grid"],
                              roofline_us=round(alg_bytes(case) / (peaks()[0] * 1e3), 2))
    print(json.dumps({"diagnostic": "launch_trace", "workload": args.workload, "us": out}))


# ----------------------------------------------------------------------------- CPU arm

def oracle_sample_rate(cases, budget_s, threads=0):
    """Time the fp64 oracle on a bounded sample of every GEMM of the workload:
    a fixed random subset of outputs per GEMM, sized to ~budget_s of CPU work.
    Returns (seconds per full step extrapolated, cores, description)."""
    import numpy as np
    import oracle

    cores = oracle.set_threads(threads or len(os.sched_getaffinity(0)))
    macs_step = sum(c.M * c.N * c.K for c in cases)
    # calibrate
    c0 = max(cases, key=lambda c: c.K)
    x, w = synth.make_xw(1, 64, c0.K, seed=0)
    t0 = time.perf_counter()
    oracle.gemm_ref(x, w)
    dt = max(time.perf_counter() - t0, 1e-6)
    rate = 64 * c0.K / dt  # MAC/s
    frac = min(1.0, budget_s * rate / macs_step)
    rng = np.random.default_rng(0)
    spent = 0.0
    done_macs = 0
    for i, c in enumerate(cases):
        n_out = max(8, int(c.M * c.N * frac))
        g = torch.Generator().manual_seed(i)
        xs = torch.randn(c.M, c.K, generator=g).to(torch.bfloat16)
        ws = (torch.randn(min(c.N, n_out), c.K, generator=g) / c.K ** 0.5).to(torch.bfloat16)
        ms = rng.integers(0, c.M, n_out)
        ns = rng.integers(0, ws.shape[0], n_out)
        t0 = time.perf_counter()
        oracle.gemm_ref_sampled(xs, ws, ms, ns)
        spent += time.perf_counter() - t0
        done_macs += n_out * c.K
    per_step = spent * macs_step / max(done_macs, 1)
    desc = (f"{done_macs / macs_step:.4%} of the step's outputs (random output positions of every GEMM), "
            f"fp64 oracle, {cores} OpenMP threads, extrapolated by MAC count")
    return per_step, cores, desc


# The five configurations of the metric, as (key, workload, mode, target fraction of the measured peak or
# None).  The default run reports every one of them beside its headline (the Qwen3-8B decode step).
CONFIGURATIONS = (
    ("c1_single_m1_4096x4096", "single", "launches", 0.80, {"steps": 64}),
    # back-to-back calls on unrelated buffers with WSM_FLAG_INDEPENDENT (automatic grid: at most a quarter
    # of the SMs each, so about four calls run at once); 64 launches per timed graph so that its start and
    # end (the first call alone, the last one draining) weigh little
    ("c1_single_m1_4096x4096_independent", "single", "launches", 0.80,
     {"independent": True, "grid": 0, "steps": 64}),
    ("c2_qwen3_8b_decode_gemms", "qwen3_decode", "chain", 0.80),
    ("c3_skinny_k7168_k8192", "skinny", "chain", 0.80),
    ("c4_l2_reuse_m32_m64", "l2_reuse", "chain", None),
    ("c4_l2_reuse_m32_m64_whole_m_tile", "l2_reuse_whole_m", "chain", None),
    # the same four GEMMs (gate_up, down at M = 32, 64, one M-tile each) as independent single launches
    ("c4_l2_reuse_m32_m64_independent_launches", "l2_reuse_whole_m", "launches", 0.80,
     {"independent": True, "grid": 0}),
    ("c5_chain_36x4_m16", "chain", "chain", 0.75),
)


def run_configurations(args, rank, world, local_rank, hbm_peak, headline):
    """Every configuration besides the headline one: device time per step of
    K' = min(K, 10) steps in one graph (same protocol as the headline; the
    single-GEMM lines take 64 launches), GB/s of algorithmic bytes, fraction
    of the measured peak."""
    out = {}
    for key, workload, mode, target, *over in CONFIGURATIONS:
        over = dict(over[0]) if over else {}
        own_steps = "steps" in over
        n_steps = over.pop("steps", min(args.steps, 10))
        if workload == args.workload and mode == args.mode and (not own_steps or n_steps == args.steps) and \
                all(getattr(args, k) == v for k, v in over.items()):
            r = headline
            n_steps = args.steps
        else:
            sub = argparse.Namespace(**vars(args))
            sub.workload, sub.mode, sub.only = workload, mode, ""
            sub.independent, sub.grid = False, 0
            for k, v in over.items():
                setattr(sub, k, v)
            r = run_gpu(sub, rank, world, local_rank, mode=mode, steps=n_steps, extras=False)
        gbs = r["total_bytes"] / (r["ms_per_step"] * 1e-3) / 1e9
        n = len(r["cases"])
        out[key] = {"workload": workload, "mode": mode, "gemms": n, "ms_per_step": round(r["ms_per_step"], 4),
                    "us_per_gemm": round(r["ms_per_step"] * 1e3 / n, 3), "GBps": round(gbs, 1),
                    "frac_of_peak": round(gbs / hbm_peak, 4), "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                    "target_frac": target, "steps": n_steps, **({"options": over} if over else {}),
                    "bytes_per_step": r["total_bytes"]}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="wsm", choices=["wsm", "reference"])
    ap.add_argument("--workload", default="qwen3_decode",
                    choices=["qwen3_decode", "single", "skinny", "l2_reuse", "l2_reuse_whole_m", "chain"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=10.0)
    ap.add_argument("--only", default="", help="comma-separated case names (profiling)")
    ap.add_argument("--mode", default=None, choices=["chain", "launches"],
                    help="chain: the step is one persistent gemm_chain kernel; launches: one skinny_gemm per GEMM "
                         "(default: launches for the single-GEMM workload, chain otherwise)")
    ap.add_argument("--no-breakdown", action="store_true", help="skip the per-GEMM single-launch breakdown")
    ap.add_argument("--trace-boundaries", action="store_true",
                    help="diagnostic: one traced run of the workload as a dependent chain; prints where each task's "
                         "time goes (not a bench line)")
    ap.add_argument("--trace-launches", action="store_true",
                    help="diagnostic: per-CTA timeline of back-to-back launches of each GEMM of the workload "
                         "(not a bench line)")
    ap.add_argument("--cluster", type=int, default=0, choices=[0, 1, 2],
                    help="chains' cluster reduction: 0 auto (off), 1 off, 2 on")
    ap.add_argument("--die-groups", type=int, default=0, choices=[0, 1, 2],
                    help="chains' die-grouped claims: 0 auto (M-tiled chains), 1 on, 2 off")
    ap.add_argument("--independent", action="store_true",
                    help="launches mode: WSM_FLAG_INDEPENDENT on every launch (the step's GEMMs share no buffers)")
    ap.add_argument("--grid", type=int, default=0, help="launches mode: persistent CTAs per launch (0 = auto)")
    ap.add_argument("--no-configurations", action="store_true",
                    help="skip the other four configurations (reported beside the default workload)")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "nshard"],
                    help="N > 1: independent replicas (weak scaling) or column blocks of every weight per rank "
                         "with an all-gather of each Y (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.mode is None:
        args.mode = "launches" if args.workload == "single" else "chain"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    hbm_peak, peak_kind = peaks()
    cases = workload_cases(args.workload)
    if args.only:
        cases = [c for c in cases if c.name in args.only.split(",")]
        if not cases:
            raise SystemExit(f"--only {args.only}: no case of workload {args.workload} has these names")
    n_cp = n_copies(cases, INDEPENDENT_REUSE_CALLS if args.mode == "launches" and args.independent else 1)
    config = {"workload": {"qwen3_decode": "qwen3_8b_decode_gemms", "single": "single_gemm_m1_4096x4096",
                           "skinny": "skinny_k7168_k8192", "l2_reuse": "l2_reuse_m32_m64",
                           "l2_reuse_whole_m": "l2_reuse_m32_m64_whole_m_tile",
                           "chain": "chain_36x4_m16"}[args.workload],
              "gemms_per_step": len(cases),
              "M": sorted({c.M for c in cases}),
              "shapes_KxN": sorted({f"{c.K}x{c.N}" for c in cases}),
              "weight_bytes_per_step": sum(2 * c.N * c.K for c in cases),
              "l2": "inputs larger than L2: every GEMM of a step has its own weights "
                    f"({sum(2 * c.N * c.K for c in cases) / 1e9:.3f} GB per step, L2 126 MB)"
                    + (f"; steps cycle through {n_cp} weight copies "
                       f"({n_cp * sum(2 * c.N * c.K for c in cases) / 1e9:.2f} GB)"
                       if n_cp > 1 else ""),
              "parallelism": f"replicas{world}" if world > 1 else "single",
              "mode": args.mode + (" (one persistent kernel per step, W read-only flag)" if args.mode == "chain"
                                   else " (one skinny_gemm launch per GEMM, W read-only flag"
                                        + (", independent flag" if args.independent else "")
                                        + (f", grid {args.grid}" if args.grid else "") + ")")}

    if args.impl == "reference":
        if rank != 0:
            return
        budget = max(2.0, min(args.cpu_budget_s, 60.0 / max(1, args.steps + args.warmup)))
        for _ in range(args.warmup):
            oracle_sample_rate(cases, budget / 4)
        per = []
        for _ in range(args.steps):
            sec, cores, desc = oracle_sample_rate(cases, budget)
            per.append(sec)
        per.sort()
        sec = per[len(per) // 2]
        tb = sum(alg_bytes(c) for c in cases)
        val = tb / sec / 1e9
        line = {"metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "impl": "reference",
                "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if args.trace_boundaries or args.trace_launches:
        if rank == 0:
            (trace_boundaries if args.trace_boundaries else trace_launches)(args)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", device_id=torch.device("cuda", local_rank),
                                             timeout=datetime.timedelta(seconds=120))
    if args.parallel == "nshard":
        full_bytes, ms = run_nshard(args, rank, world, local_rank)
        if rank == 0:
            config["parallelism"] = f"nshard{world}"
            print(json.dumps({"metric": METRIC, "value": round(full_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
                              "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
                              "frac_of_peak": round(full_bytes / (ms * 1e-3) / 1e9 / world / hbm_peak, 4),
                              "gpu_launches": args.steps, "roofline": None, "cpu_baseline": None, "e2e": None}))
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    r = run_gpu(args, rank, world, local_rank)
    breakdown = None
    if args.mode == "chain" and not args.no_breakdown and args.workload != "chain":
        # informational: the same GEMMs as separate skinny_gemm launches (graph-replayed)
        rb = run_gpu(args, rank, world, local_rank, mode="launches", steps=min(args.steps, 5), extras=False)
        import statistics as _st
        breakdown = {"ms_per_step": round(rb["ms_per_step"], 4),
                     "value_GBps": round(rb["total_bytes"] / (rb["ms_per_step"] * 1e-3) / 1e9, 1),
                     "frac_of_peak": round(rb["total_bytes"] / (rb["ms_per_step"] * 1e-3) / 1e9 / hbm_peak, 4),
                     "note": "ms_per_step: the launches back to back in one graph; us_per_gemm_isolated: each "
                             "launch alone between two events, without the overlap with its neighbours",
                     "us_per_gemm_isolated": {c.name: round(_st.median(row[i] for row in rb["per_launch"]) * 1e3, 2)
                                              for i, c in enumerate(rb["cases"])}}
        # the same launches with WSM_FLAG_INDEPENDENT (the step's GEMMs share no buffers; automatic grid:
        # at most a quarter of the SMs each): neighbouring launches run side by side
        sub = argparse.Namespace(**vars(args))
        sub.independent, sub.grid = True, 0
        ri = run_gpu(sub, rank, world, local_rank, mode="launches", steps=min(args.steps, 5), extras=False)
        gbs = ri["total_bytes"] / (ri["ms_per_step"] * 1e-3) / 1e9
        breakdown["independent_launches"] = {"ms_per_step": round(ri["ms_per_step"], 4), "value_GBps": round(gbs, 1),
                                             "frac_of_peak": round(gbs / hbm_peak, 4), "grid": "auto"}
        # every GEMM on its own, 32 launches of its shape back to back: plain, and independent
        dev = torch.device("cuda", local_rank)
        breakdown["per_shape_back_to_back"] = {
            "note": "32 launches of one shape back to back in a graph, weight copies > 4x L2 (independent: a "
                    "copy comes back after 10 launches at the earliest); us per launch; independent = "
                    "WSM_FLAG_INDEPENDENT with the automatic grid (at most a quarter of the SMs, even rounds)",
            "plain": back_to_back_per_shape(args, dev, hbm_peak, False, 0),
            "independent": back_to_back_per_shape(args, dev, hbm_peak, True, 0)}

    configurations = None
    if args.workload == "qwen3_decode" and args.mode == "chain" and not args.only and not args.no_configurations:
        configurations = run_configurations(args, rank, world, local_rank, hbm_peak, r)

    # roofline of the weight-streaming kernel: per-launch algorithmic bytes / duration
    import statistics
    per_case = []
    if r["chain"]:
        launch_ms = [row[0] for row in r["per_launch"]]
        med = statistics.median(launch_ms)
        fam_bytes, fam_ms = r["total_bytes"], med
        us_per_gemm = {"chain_us": round(med * 1e3, 2), "per_gemm_us_avg": round(med * 1e3 / len(cases), 3)}
        # the chain's path: FMA only if the automatic choice is FMA for every task at the largest M
        from weight_streaming_megakernel_b200 import plan
        mmax = max(c.M for c in cases)
        fma = all(plan(mmax, c.N, c.K)["path"] == 1 for c in cases)
        dominant = "wsm_stream_kernel" if fma else "wsm_umma_kernel"
    else:
        from weight_streaming_megakernel_b200 import plan
        fam = {}
        us_per_gemm = {}
        for i, c in enumerate(r["cases"]):
            ms = statistics.median(row[i] for row in r["per_launch"])
            p = plan(c.M, c.N, c.K, num_sms=torch.cuda.get_device_properties(0).multi_processor_count,
                     m_tile=c.m_tile)
            k = "wsm_umma_kernel" if p["path"] == 2 else "wsm_stream_kernel"
            b, t = fam.get(k, (0, 0.0))
            fam[k] = (b + alg_bytes(c), t + ms)
            us_per_gemm[c.name] = round(ms * 1e3, 2)
            per_case.append((c.name, ms))
        dominant = max(fam, key=lambda k: fam[k][1])
        fam_bytes, fam_ms = fam[dominant]
    achieved = fam_bytes / (fam_ms * 1e-3) / 1e9
    traffic = stored_traffic(dominant, config["workload"], args.mode) if r["chain"] and not args.only else None
    step_ms = sorted(sum(row) for row in r["per_launch"])

    def pct(q):
        return round(step_ms[min(len(step_ms) - 1, int(q * (len(step_ms) - 1) + 0.5))], 4)
    value = r["total_bytes"] * world / (r["ms_per_step"] * 1e-3) / 1e9

    cpu = cpu1 = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, cores, desc = oracle_sample_rate(cases, args.cpu_budget_s)
        cpu = {"value": round(r["total_bytes"] / sec / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": desc}
        sec, cores, desc = oracle_sample_rate(cases, args.cpu_budget_s / 2, threads=1)
        cpu1 = {"value": round(r["total_bytes"] / sec / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                "sample": desc}

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
                "frac_of_peak": round(value / world / hbm_peak, 4),
                "frac_of_8tbs": round(value / world / NOMINAL_HBM_GBS, 4),
                "roofline": {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1), "peak": hbm_peak,
                             "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                             "traffic": traffic,
                             "algorithmic_bytes_per_launch": fam_bytes if r["chain"] else None},
                "step_ms_p10_p50_p90": [pct(0.1), pct(0.5), pct(0.9)],
                "us_per_gemm": us_per_gemm,
                "single_launch_breakdown": breakdown,
                "configurations": configurations,
                "cpu_baseline": cpu,
                "cpu_baseline_1thread": cpu1,
                "e2e": r["e2e"],
                "gpu_launches": r["launches_per_step"] * args.steps,
                "ms_per_step_without_timing_events": round(r["plain_ms"], 4),
                "clocks": r["clocks"]}
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
