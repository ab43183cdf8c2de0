import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


@pytest.fixture(scope="session")
def ora():
    import oracle
    oracle.build()
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def syn():
    import synth
    synth._build_host()
    return synth


@pytest.fixture(scope="session")
def coli():
    """The CUDA library's Python binding (needs a GPU to compute)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_weight_only_sigmoid_b200 as m
    m.load()
    return m
