import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # The CUDA library is built in-tree (nvcc, sm_100a); this is a no-op when
    # it is newer than its sources.  The binding itself never builds: without
    # the library it refuses to load.
    from kv_cache_injection_gather_b200 import build
    build.build()


@pytest.fixture(scope="session")
def cuda_available():
    import torch
    return torch.cuda.is_available()
