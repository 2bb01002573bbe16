import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def pytest_terminal_summary(terminalreporter):
    """Worst per-tensor max-relative error and worst floored elementwise
    relative error of every test that compared outputs with the oracle."""
    try:
        from helpers import ELEM_FLOOR, REPORT
    except ImportError:
        return
    if not REPORT:
        return
    worst = {}
    for test, mr, er in REPORT:
        a, b = worst.get(test, (0.0, 0.0))
        worst[test] = (max(a, mr), max(b, er))
    terminalreporter.section("parity errors (max|x-ref|/max|ref|; elementwise with floor %g*max|ref|)" % ELEM_FLOOR)
    for test, (mr, er) in sorted(worst.items()):
        terminalreporter.write_line(f"{mr:10.3e} {er:10.3e}  {test}")
