import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload, minutes on one GPU")


def read_golden(name):
    """Parse a golden fixture: '#' lines are comments, every other line is
    'key v1 v2 ...' (hex bytes allowed)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = [int(v, 16) if v.startswith("0x") else float(v) for v in vals]
    return out


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _no_expired_device_waits(request):
    """After every GPU test: no kernel of the library gave up a bounded wait
    (such a kernel stops early and sets a device flag, read and cleared here)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    from sparse_long_context_03_b200 import dsa
    dsa.check_device_error()
