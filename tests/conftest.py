"""pytest configuration: the ``gpu`` marker and the import path.

Tests marked ``gpu`` need a CUDA device and the built CUDA library; everything
else runs on the CPU (oracle pins, host logic, library loading)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle():
    from oracle import oracle as O
    return O.get()
