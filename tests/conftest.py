import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size layer checks (minutes)")


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library handle (loads the in-tree shared object)."""
    from post_weight_quantization_19_b200 import _abi
    return _abi.load()
