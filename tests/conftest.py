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
    """Parse a golden fixture: '# comment' lines are skipped, 'key: v v v' lines become lists."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            out[key.strip()] = val.split()
    return out


@pytest.fixture
def golden():
    return read_golden


@pytest.fixture(scope="session")
def ql():
    """The quantized_linear_b200 binding, building libqlinear.so first if it is missing or stale."""
    from quantized_linear_b200 import build as qlbuild
    qlbuild.build()
    import quantized_linear_b200
    return quantized_linear_b200
