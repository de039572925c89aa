"""Shared pytest set-up: markers, import path and cached synthetic inputs."""
import functools
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: a CPU test that takes more than a few seconds")


@functools.lru_cache(maxsize=2)
def workload_inputs(name):
    """Generated once per process: the named workload's bf16 inputs (CPU)."""
    import gen
    return gen.make_inputs(name)


@pytest.fixture
def inputs_of():
    return workload_inputs
