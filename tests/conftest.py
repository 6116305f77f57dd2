import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture
def mutation():
    """Plant one known mistake in the CPU oracle for the duration of a test."""
    import oracle

    def _set(m):
        oracle.set_mutation(m)

    yield _set
    oracle.set_mutation(oracle.MUT_NONE)
