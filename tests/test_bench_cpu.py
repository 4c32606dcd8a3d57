"""bench.py on the host: its reference arm (the fp64 oracle timed on the host
cores) runs without a GPU and prints the one JSON line of the benchmark
contract, and its weight-copy rotation keeps timed weights out of L2."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--cpu-budget-s", "2"], capture_output=True, text=True, timeout=300,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"] == "qwen3_8b_decode_gemms"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the multi-GPU benchmark is (two ranks), rank 0 alone times
    the oracle and prints; the other rank exits 0 without work."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl",
           "reference", "--steps", "1", "--warmup", "3", "--cpu-budget-s", "2"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2


def test_weight_copies_keep_steps_and_concurrent_launches_apart():
    """Weight copies: consecutive steps touch at least 4x L2, and for
    independent launches (several run at once) a copy comes back only after
    INDEPENDENT_REUSE_CALLS launches, so no two calls in flight share weights
    through L2."""
    import bench
    import synth
    L2 = bench.L2_BYTES
    for name in ("qwen3_decode", "single", "skinny", "l2_reuse", "l2_reuse_whole_m", "chain"):
        cases = bench.workload_cases(name)
        w = sum(2 * c.N * c.K for c in cases)
        n = bench.n_copies(cases)
        assert n * w >= 4 * L2 or n == 1 and w >= 4 * L2
        ni = bench.n_copies(cases, bench.INDEPENDENT_REUSE_CALLS)
        assert ni >= n and ni * len(cases) >= bench.INDEPENDENT_REUSE_CALLS
    for c in synth.config_qwen3_decode():   # the per-shape runs: one GEMM per step
        n = bench.n_copies([c], bench.INDEPENDENT_REUSE_CALLS)
        assert n >= bench.INDEPENDENT_REUSE_CALLS and n * 2 * c.N * c.K >= 4 * L2
