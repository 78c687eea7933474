import os
import sys

import pytest

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
for p in (_ROOT, os.path.dirname(os.path.abspath(__file__))):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


def pytest_terminal_summary(terminalreporter):
    """Print what the GPU parity tests recorded: per workload the queries whose routing was checked against the
    oracle (fp32 bit-exact, fp64 margin rule) with the counts of differences and small margins; per gradient the
    error ratio against its bound."""
    mod = sys.modules.get("gpu_parity")
    lines = getattr(mod, "PARITY_LOG", None)
    if lines:
        terminalreporter.section("parity against the oracle")
        for line in lines:
            terminalreporter.write_line(line)
