import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU oracle run")


@pytest.fixture(scope="session")
def cuda_lib():
    """The product library on a GPU; loud failure when it is missing."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sampling_transform_lm_b200 as sts

    sts.load()  # raises if the shared library is absent
    return sts
