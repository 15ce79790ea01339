import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")


def golden_path(name: str) -> str:
    return os.path.join(ROOT, "tests", "golden", name)


def read_golden(name: str):
    """Non-comment lines of a golden fixture as (key, [tokens]) pairs."""
    rows = []
    with open(golden_path(name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            rows.append((key, rest))
    return rows


@pytest.fixture
def golden():
    return read_golden


@pytest.fixture(scope="session", autouse=True)
def _library_built():
    """Compile the CUDA library (sm_100a) if it is missing or older than its sources."""
    from ternary_weight_a8_b200 import _build

    _build.build()
