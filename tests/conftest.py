import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running check")


def pytest_terminal_summary(terminalreporter):
    """Print every recorded parity error (output, plain max-abs error, bound)."""
    try:
        import parity_report
    except ImportError:
        from tests import parity_report
    lines = parity_report.lines()
    if lines:
        terminalreporter.section("parity: plain max-abs error per output")
        for ln in lines:
            terminalreporter.write_line(ln)
