import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The C-ABI library through its Python binding; fails loudly when absent."""
    from long_context_prefill_dca_b200 import q1m
    return q1m.library()


@pytest.fixture
def deterministic():
    """Deterministic mode for a test that compares two runs bit for bit (the attention
    kernel then walks every item's key blocks in a fixed order)."""
    from long_context_prefill_dca_b200 import q1m
    was = q1m.deterministic()
    q1m.set_deterministic(True)
    try:
        yield
    finally:
        q1m.set_deterministic(was)
