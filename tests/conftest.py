import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")
    config.addinivalue_line("markers", "slow: long CPU case")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


GOLDEN = ROOT / "tests" / "golden"


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """O comparisons of the session: how many elements needed the half bf16 step
    beyond the plain 1e-2 bound (the bf16 output's own rounding)."""
    import parity
    if not parity.RECORDS:
        return
    tr = terminalreporter
    n = sum(r[1] for r in parity.RECORDS)
    k = sum(r[2] for r in parity.RECORDS)
    tr.write_sep("-", f"O comparisons: {len(parity.RECORDS)}, {n} elements, {k} beyond the plain 1e-2")
    for tag, elems, beyond, mx, mean in parity.RECORDS:
        if beyond:
            tr.write_line(f"  {tag}: {beyond} of {elems} elements beyond 1e-2 (max-abs {mx:.4g}, mean-abs {mean:.3g})")
    worst = max(parity.RECORDS, key=lambda r: r[3])
    tr.write_line(f"  largest max-abs: {worst[0]} {worst[3]:.4g}; largest mean-abs "
                  f"{max(r[4] for r in parity.RECORDS):.3g}")
