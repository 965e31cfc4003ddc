import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def read_golden(name: str) -> dict:
    """Parse a `key = value` fixture; '#' lines are the citation header."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (x.strip() for x in line.split("=", 1))
            parts = val.split()
            out[key] = [int(p) for p in parts] if len(parts) > 1 else int(parts[0])
    return out


@pytest.fixture
def golden():
    return read_golden


def pytest_terminal_summary(terminalreporter):
    """Observed attention error per comparison: max-abs and max-rel beside the
    allclose bound |gpu - ref| <= 2e-3 + 1e-2 |ref| the tests apply."""
    try:
        from _helpers import ERROR_LOG
    except ImportError:
        return
    if not ERROR_LOG:
        return
    tr = terminalreporter
    tr.section("attention error vs the fp64 oracle (bound: 2e-3 + 1e-2*|ref| per element)")
    tr.write_line(f"{'comparison':<56} {'elements':>9} {'max_abs':>9} {'max_rel':>9} {'rel|>=.2':>9} "
                  f"{'err/bound':>9}")
    for what, n, a, r, rb, q in ERROR_LOG:
        tr.write_line(f"{what[:56]:<56} {n:>9} {a:>9.3g} {r:>9.3g} {rb:>9.3g} {q:>9.3f}")
