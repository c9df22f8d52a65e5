import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built librlscan.so")
    config.addinivalue_line("markers", "perf: one timed configuration per estimator (GPU)")
    config.addinivalue_line("markers", "slow: full-size or long-running case")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle._load()
    return oracle


@pytest.fixture(scope="session")
def rlscan_lib_path():
    """Path of the built C-ABI library (built on demand, no GPU needed)."""
    from linear_recurrence_scans_02_b200 import _build
    return _build.build_library()


def _cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_device():
    if not _cuda_ok():
        pytest.fail("a -m gpu test ran without a CUDA device")
    import torch
    return torch.device("cuda", 0)
