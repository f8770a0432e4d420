import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def repo_root():
    return ROOT


def pytest_terminal_summary(terminalreporter):
    """Near-tie exclusions (oracle key_(k) - key_(k+1) < 1e-6) per workload
    the GPU parity tests compared, and how many compared tokens listed the
    same experts in another order."""
    try:
        import _parity
    except ImportError:
        return
    if not _parity.EXCLUSIONS:
        return
    terminalreporter.write_sep("-", "near-tie exclusions (GPU parity)")
    for name, (T, n, ordered) in sorted(_parity.EXCLUSIONS.items()):
        terminalreporter.write_line(
            f"{name}: excluded={n} of {T} tokens, ordered_list_mismatches={ordered}")
