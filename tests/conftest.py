import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_fixture(name):
    """Rows of a tests/golden text fixture, without '#' comment lines."""
    path = os.path.join(ROOT, "tests", "golden", name)
    with open(path, encoding="utf-8") as fh:
        return [ln.strip() for ln in fh if ln.strip() and not ln.startswith("#")]


@pytest.fixture
def fixture_rows():
    return read_fixture
