import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: longer CPU-side check")


def pytest_sessionstart(session):
    # Build (or refresh) the in-tree CUDA library and the oracle before any test
    # imports them; nvcc cross-compiles for sm_100a without a GPU.
    from bit_kv_cache_23_b200 import build as _b

    _b.build()
    import oracle

    oracle.build()
