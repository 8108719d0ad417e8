import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large parity cases")


@pytest.fixture(scope="session")
def orc():
    from oracle import oracle
    oracle.lib()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Largest parity errors measured by the GPU tests of this session."""
    gh = sys.modules.get("gpuhelp")
    if gh is not None and getattr(gh, "MAX_ERR", None):
        items = ", ".join(f"{k} {v:.3e}" for k, v in sorted(gh.MAX_ERR.items()))
        terminalreporter.write_line(f"largest measured errors: {items}")
