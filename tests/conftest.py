import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a tests/golden/*.txt fixture: '#' comments, whitespace-separated rows."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def golden_dict(name):
    return {r[0]: float(r[1]) for r in read_golden(name)}


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
