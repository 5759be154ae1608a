import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running test")


@pytest.fixture(scope="session")
def oracle():
    import oracle as oracle_pkg

    return oracle_pkg.load()


def pytest_terminal_summary(terminalreporter):
    """The achieved figures of the GPU parity comparisons (tests/gpu_helpers.py RESULTS)."""
    mod = sys.modules.get("tests.gpu_helpers")
    res = getattr(mod, "RESULTS", None) if mod else None
    if not res:
        return
    terminalreporter.section("parity figures (GPU path against the oracle)")
    for what, kind, fig in res:
        terminalreporter.write_line(f"{kind:9s} {what}: {fig}")
