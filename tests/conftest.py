import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU-side work")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The parity checks' ulp statistics over the session (when any ran)."""
    parity = sys.modules.get("parity")
    if parity is None or not parity.STATS["checks"]:
        return
    s = parity.STATS
    terminalreporter.write_line(
        f"parity: {s['checks']} checks, {s['elements']} bf16 elements; max ulp distance from round(Y_ref) "
        f"over elements held to 1 ulp: {s['max_ulp']}; cancellation window (|Y_ref| < fp32 bound): "
        f"{s['cancel_elements']} elements, max ulp there {s['cancel_max_ulp']}")
