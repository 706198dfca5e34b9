"""Shared pytest configuration.

``gpu`` tests call the CUDA library through its C ABI and need a B200; every
other test runs on the CPU (the oracle, host-side logic, ABI symbol checks and
world-size-2 gloo tests).
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle
