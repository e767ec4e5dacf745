import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU; runs the CUDA path through the C-ABI")
    config.addinivalue_line("markers", "slow: full-size workload checks (GPU)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built C-ABI library (fails loudly when it cannot be loaded)."""
    from moe_fp8_grouped_b200 import _binding
    return _binding.lib()
