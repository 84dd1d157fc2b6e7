"""Shared pytest set-up: the repository root on sys.path and the ``gpu`` marker.

Tests marked ``gpu`` need a B200 and the built CUDA library; everything else runs
on a CPU-only machine (``pytest -m "not gpu"``).
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libqkq")


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN
