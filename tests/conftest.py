import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_sessionstart(session):
    # a fresh checkout has no libqexpert.so (build output is not versioned):
    # cross-compile it once (nvcc needs no GPU) before any test imports it
    lib = os.path.join(ROOT, "quantized_expert_matvec_b200", "libqexpert.so")
    if not os.path.exists(lib):
        import __graft_entry__
        __graft_entry__._library_builder().build()


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
