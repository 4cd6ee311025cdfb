import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def pytest_terminal_summary(terminalreporter):
    """Prints what the parity comparisons counted: codes that differed at a decision boundary (within
    1e-5), QJL signs that differed inside the rounding bound, and the worst score errors."""
    try:
        from tests.parity import REPORT
    except Exception:  # the comparison module was never imported
        return
    if not REPORT:
        return
    tr = terminalreporter
    tr.section("parity counts")
    totals = {}
    for test, kind, value, total in REPORT:
        tr.write_line("%-90s %-42s %s of %d" % (test[-90:], kind, ("%.3g" % value) if isinstance(value, float)
                                                else value, total))
        t = totals.setdefault(kind, [0, 0])
        if isinstance(value, float):
            t[0] = max(t[0], value)
        else:
            t[0] += value
        t[1] += total
    for kind, (v, n) in sorted(totals.items()):
        tr.write_line("TOTAL %-40s %s over %d" % (kind, ("max %.3g" % v) if isinstance(v, float) else v, n))
