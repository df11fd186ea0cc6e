"""Shared pytest configuration.

Tests marked ``gpu`` need a CUDA device (they call the C-ABI library's kernels);
everything else runs on the CPU: the oracle against its pins, the host-side
validation of the C ABI, symbol exports, and the multi-process (gloo) paths.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: larger CPU cases")


@pytest.fixture(scope="session", autouse=True)
def _built_oracle():
    import oracle
    oracle.build()
    yield
