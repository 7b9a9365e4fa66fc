import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def root_dir():
    return ROOT


def pytest_terminal_summary(terminalreporter):
    """One line per workload: how many packed codes the GPU parity tests compared with
    the oracle and how many differed (each by one, at a rounding boundary); then the
    measurements the tests report without a bound."""
    try:
        import stq_testlib
    except ImportError:
        return
    if stq_testlib.FLIPS:
        terminalreporter.write_sep("-", "GPU vs oracle packed codes")
        for config, (n_diff, n_codes) in sorted(stq_testlib.FLIPS.items()):
            frac = n_diff / n_codes if n_codes else 0.0
            terminalreporter.write_line(f"{config}: {n_diff} of {n_codes} codes differ (fraction {frac:.3g})")
    if stq_testlib.REPORTS:
        terminalreporter.write_sep("-", "reported measurements (not gated)")
        for name, text in sorted(stq_testlib.REPORTS.items()):
            terminalreporter.write_line(f"{name}: {text}")
