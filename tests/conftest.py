import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The C-ABI library, loaded for GPU tests (fails loudly if it is missing)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp8_fp4_moe_b200 import binding
    return binding.lib()
