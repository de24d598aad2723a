import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU-side oracle work")


def pytest_terminal_summary(terminalreporter):
    """Print the parity margins the GPU tests measured (see tests/parity.py)."""
    import parity
    if not parity.MARGINS:
        return
    terminalreporter.write_sep("-", "parity margins (measured value, fraction of its bar)")
    for line in parity.summary_lines():
        terminalreporter.write_line(line)


@pytest.fixture(scope="session")
def repo_root():
    return ROOT
