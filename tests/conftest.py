import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built libvsa.so")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes of host time)")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_terminal_summary(terminalreporter):
    try:
        import vsa_cases
    except ImportError:
        return
    n = vsa_cases.NEAR_TIE_ROWS[0]
    terminalreporter.write_line("near-tie query tiles checked on the GPU's own list: %d" % n)
