import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running case")


def pytest_sessionstart(session):
    # build the oracle (gcc) and the library (nvcc, sm_100a) in-tree if they are stale
    import oracle
    oracle.build()
    from vector_quantized_moe_b200 import build as libbuild
    libbuild.build()


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle.build()
    return oracle
