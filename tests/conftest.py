import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture
def knob():
    """Set library knobs (w1_set_knob) for one test; restored afterwards."""
    from pack_sign_g128_b200 import ops
    names = []

    def setter(name, value):
        ops.set_knob(name, value)
        names.append(name)

    yield setter
    for n in reversed(names):
        ops.set_knob(n, None)
