import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size parity case")


def read_golden(name):
    """Parse a tests/golden/*.txt fixture: '# ...' comment lines, then
    'key: v1 v2 ...' lines.  Values stay strings; callers convert."""
    path = os.path.join(ROOT, "tests", "golden", name)
    out = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out


@pytest.fixture(scope="session")
def golden():
    return read_golden


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Reports, for every bf16 comparison of the run, how many elements were
    accepted by the fp32 accumulation bound rather than the 1-ulp bound."""
    try:
        from tests._util import FALLBACK_LOG
    except Exception:
        return
    if not FALLBACK_LOG:
        return
    tr = terminalreporter
    tot_fb = sum(r[2] for r in FALLBACK_LOG)
    tot = sum(r[3] for r in FALLBACK_LOG)
    tr.section("bf16 comparisons: elements accepted by the fp32 accumulation bound")
    tr.write_line(f"{len(FALLBACK_LOG)} comparisons, {tot} elements, {tot_fb} needed the fp32 bound "
                  f"({tot_fb / max(tot, 1):.2e} of all)")
    for test, what, nfb, n in FALLBACK_LOG:
        if nfb:
            tr.write_line(f"  {test} [{what}]: {nfb} / {n}")
