import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                yield line.split()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Near ties counted by the GPU parity tests: positions whose candidate
    differs from the oracle's float64 argmax only within the near-tie gap."""
    mod = sys.modules.get("gpu_util")
    ties = getattr(mod, "NEAR_TIES", None) if mod is not None else None
    if not ties:
        return
    terminalreporter.section("near ties (GPU parity)")
    for name, (n, m) in sorted(ties.items()):
        terminalreporter.write_line("near-ties %s: %d of %d positions compared" % (name, n, m))
