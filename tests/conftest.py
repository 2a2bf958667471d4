import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU oracle case")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="session")
def fs4():
    """The product package with its library built (GPU tests only)."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    from nvfp4_precision_optimizer_b200 import _lib, build
    if not os.path.exists(_lib.LIB_PATH):
        build.build()
    import nvfp4_precision_optimizer_b200 as F
    F._lib.lib()
    return F
