import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload parity (GPU)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_sessionstart(session):
    # DUO_TEST_LIBRARY runs the GPU tests against another build of the library
    # (a variant under study); by default the in-tree libduoattn.so is used
    path = os.environ.get("DUO_TEST_LIBRARY")
    if path:
        import kv_cache_reduction_b200 as duo
        duo.load_library(path)
