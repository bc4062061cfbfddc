import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.join(ROOT, "tests")
for _p in (ROOT, TESTS):
    if _p not in sys.path:
        sys.path.insert(0, _p)
GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name: str) -> dict:
    """Parse a tests/golden fixture: '# ...' comments, 'key: value' lines.

    Repeated keys accumulate into lists."""
    out: dict = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.rstrip("\n")
            if not line.strip() or line.startswith("#"):
                continue
            k, _, v = line.partition(":")
            out.setdefault(k.strip(), []).append(v.strip())
    return out


@pytest.fixture
def golden():
    return read_golden
