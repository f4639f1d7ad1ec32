import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config._favor_parity = []


@pytest.fixture
def parity_report(request):
    """Appends one line to the parity summary printed at the end of the run."""
    return request.config._favor_parity.append


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    rows = getattr(config, "_favor_parity", [])
    if rows:
        terminalreporter.section("GPU output against the fp64 oracle")
        for r in rows:
            terminalreporter.write_line(r)


@pytest.fixture(scope="session")
def repo_root():
    return ROOT
