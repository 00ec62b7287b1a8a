import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload check (minutes)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built C-ABI library, loaded through the Python binding.  Builds it
    in-tree first when the shared object is missing."""
    from compressed_sparse_long_hca_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from compressed_sparse_long_hca_b200 import build as _build
        _build.build()
    return _lib.load()
