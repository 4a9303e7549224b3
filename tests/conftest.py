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
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Measured parity errors against their bounds, smallest headroom first."""
    from helpers import HEADROOM
    if not HEADROOM:
        return
    rows = sorted(HEADROOM, key=lambda r: r[2] / r[3] if r[3] > 0 else 0.0, reverse=True)
    tr = terminalreporter
    tr.write_sep("-", f"parity headroom ({len(rows)} comparisons; measured / bound, largest first)")
    for what, qty, got, bound in rows[:25]:
        tr.write_line(f"{got / bound:6.3f}  {got:.3e} / {bound:.1e}  {qty:11s} {what}")
