import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session", autouse=True)
def _build_host_libs():
    import oracle
    import synth

    synth.build()
    oracle.build()
    yield


@pytest.fixture(scope="session")
def moba():
    """The package with libmoba.so built in-tree."""
    from block_sparse_long_gate_b200.build import build_library

    build_library()
    import block_sparse_long_gate_b200 as m

    m.lib()
    return m


@pytest.fixture(scope="session")
def cuda_dev():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda:0")
