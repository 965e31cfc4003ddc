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
