import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libwmtp.so")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session", autouse=True)
def _build_oracle():
    from oracle.build_oracle import build
    build()


def golden_path(name: str) -> str:
    return os.path.join(GOLDEN, name)


def read_golden(name: str):
    """Reads a golden fixture: '#' lines are comments (citations), the rest whitespace-split."""
    rows = []
    with open(golden_path(name)) as f:
        for line in f:
            s = line.strip()
            if not s or s.startswith("#"):
                continue
            rows.append(s.split())
    return rows
