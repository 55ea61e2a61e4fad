import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Build the CUDA library (cross-compiles without a GPU) and the oracle before
# any test module imports them; both builds are skipped when up to date.
from paged_kv_cache_402_b200 import build as _pkg_build  # noqa: E402
from oracle import build as _oracle_build  # noqa: E402

_pkg_build.build()
_oracle_build.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    """The CUDA device for gpu-marked tests; a missing GPU is an error, not a skip."""
    import torch

    if not torch.cuda.is_available():
        pytest.fail("gpu-marked test run without a CUDA device")
    return torch.device("cuda:0")
