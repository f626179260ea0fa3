import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


# Errors that whole-tensor parity checks saw, printed at the end of the run
# (pytest captures the tests' own output): (where, O max-abs, O mean-abs,
# LSE max-abs, elements compared).
PARITY_LOG = []


def record_parity(where, o_max, o_mean, lse_max, n):
    PARITY_LOG.append((where, float(o_max), float(o_mean), float(lse_max), int(n)))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


def pytest_terminal_summary(terminalreporter):
    if not PARITY_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "whole-tensor parity against the fp64 oracle (errors seen)")
    for where, mx, mean, lmx, n in PARITY_LOG:
        tr.write_line(f"{where}: O max-abs {mx:.3e}, O mean-abs {mean:.3e}, LSE max-abs {lmx:.3e} "
                      f"over {n} outputs")


def read_golden(name):
    """Parse a tests/golden/*.txt fixture: 'key = v1 v2 ...' lines, '#' comments."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = (s.strip() for s in line.split("=", 1))
            vals = [float(t) for t in v.split()]
            out[k] = vals if len(vals) > 1 else vals[0]
    return out


@pytest.fixture(scope="session")
def golden():
    return read_golden
