import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a); runs the CUDA library")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def pkv():
    """The CUDA library's binding (built in-tree if stale)."""
    import runpy
    runpy.run_path(os.path.join(ROOT, "paged_kv_cache_470_b200", "build.py"))["build"]()
    import paged_kv_cache_470_b200 as lib
    return lib


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device on this machine")
    major, minor = torch.cuda.get_device_capability(0)
    if (major, minor) < (10, 0):
        pytest.skip(f"needs sm_100 (found sm_{major}{minor})")
    return torch.device("cuda:0")
