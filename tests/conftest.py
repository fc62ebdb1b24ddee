import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# (test id, quantity, measured value, tolerance) of every parity comparison that reported
# itself; printed as a table at the end of the run so the margins are visible.
_PARITY = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture
def parity(request):
    """parity(quantity, value, tol=None): record a measured error (or count) of this test."""
    def record(what, value, tol=None):
        _PARITY.append((request.node.nodeid, what, float(value), tol))
    return record


def pytest_terminal_summary(terminalreporter):
    if not _PARITY:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity: measured values against their tolerances")
    for nodeid, what, v, tol in _PARITY:
        line = f"{nodeid} :: {what} = {v:.3e}"
        if tol:
            line += f"  (tol {tol:.1e}" + (f", margin {tol / v:.1f}x)" if v > 0 else ")")
        tr.write_line(line)
