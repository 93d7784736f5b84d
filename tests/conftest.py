import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # the in-tree libraries are built (or found up to date) before any test imports them
    from __graft_entry__ import load_builder
    load_builder().build()


@pytest.fixture(scope="session")
def repo_root():
    return ROOT


def pytest_terminal_summary(terminalreporter):
    """The largest attention error against the oracle per test (the bound is 1e-2)."""
    side = sys.modules.get("tests.oracle_side")
    if side is None or not side.ATTEND_MAX_ERR:
        return
    terminalreporter.write_sep("-", "attention: max |gpu - oracle| per test (bound 1e-2)")
    for key, err in sorted(side.ATTEND_MAX_ERR.items()):
        terminalreporter.write_line(f"{err:.3e}  {key}")
