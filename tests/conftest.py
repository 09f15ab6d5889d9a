import os
import sys

import pytest

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
for p in (ROOT, TESTS):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity on sampled rows")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def dsa_lib():
    """libdsa.so, rebuilt first when any source is newer than it."""
    from learned_sparse_attention_dsa_b200 import binding, build
    build.build()
    return binding.load_library()


@pytest.fixture(scope="session")
def cuda(dsa_lib):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    major, minor = torch.cuda.get_device_capability()
    assert major == 10, f"these kernels target sm_100a, found sm_{major}{minor}"
    return torch.device("cuda:0")
