import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "oracle: pins of the CPU oracle")
    config.addinivalue_line("markers", "slow: long-running")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Routing against the oracle, per case the GPU tests checked: tokens
    checked, tokens whose routing set differs from the oracle's (each one
    inside the 1e-5 tie window, or the test fails), and tokens inside the
    window at all."""
    mod = sys.modules.get("tests.gpu_util")
    rep = getattr(mod, "ROUTING_REPORT", None)
    if not rep:
        return
    tr = terminalreporter
    tr.write_sep("-", "routing against the oracle (tie window 1e-5)")
    tr.write_line(f"{'case':<44} {'tokens':>7} {'flips':>6} {'in window':>9}")
    for case in sorted(rep):
        n, flips, near = rep[case]
        tr.write_line(f"{case:<44} {n:>7} {flips:>6} {near:>9}")
