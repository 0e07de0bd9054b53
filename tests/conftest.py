import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built libbsq.so")
    config.addinivalue_line("markers", "slow: full-size oracle work (minutes on CPU)")


@pytest.fixture
def knobs():
    """Setter for the library's kernel-selection overrides
    (bsq_debug_kernel_choice); every knob set is restored to automatic at
    teardown."""
    from fp8_math_b200 import bsq
    touched = []

    def setter(knob, value):
        bsq.bsq_debug_kernel_choice(knob, value)
        touched.append(knob)

    yield setter
    for k in touched:
        bsq.bsq_debug_kernel_choice(k, -1)


@pytest.fixture(scope="session")
def ora():
    from oracle import oracle as o
    o.build()
    return o


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows
