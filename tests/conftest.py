import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_terminal_summary(terminalreporter):
    """Worst plain max|err|/RMS per kind of parity check in this run (the tests assert the
    element-wise allowance; these are the literal-metric figures beside it)."""
    try:
        from _util import RECORDS
    except ImportError:
        return
    if not RECORDS:
        return
    worst = {}
    for test, kind, e, tol in RECORDS:
        if kind not in worst or e > worst[kind][0]:
            worst[kind] = (e, tol, test)
    terminalreporter.write_line(f"parity: {len(RECORDS)} checks; worst plain max|err|/RMS per kind:")
    for kind, (e, tol, test) in sorted(worst.items()):
        terminalreporter.write_line(f"  {kind:14s} {e:.3e} (bound {tol:g}) in {test}")
