import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built libftk.so")
    config.addinivalue_line("markers", "slow: long-running CPU test")


import pytest  # noqa: E402


@pytest.fixture(scope="session", autouse=True)
def _built_library(request):
    """Build libftk.so (sm_100a) and the oracle once per session if stale."""
    from oracle import oracle
    from sparse_attention_indexer_ftk_b200 import build

    oracle.build()
    build.build()
