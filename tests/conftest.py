import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (seconds to minutes)")


def pytest_collection_modifyitems(config, items):
    # Keep the file that tests the allocation-free entry point last, so a run
    # that stops at the first failure has run everything else first.
    last = [it for it in items if os.path.basename(str(it.fspath)).startswith("test_zz_")]
    rest = [it for it in items if it not in last]
    items[:] = rest + last


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True
