import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(session, config, items):
    """The forward's and the decoding step's tests run before the backward's
    (which takes the forward's out and lse as inputs), and the no-allocation
    test runs last; the order inside each group is kept."""
    def group(item):
        name = item.nodeid
        if "test_zz_no_alloc" in name:
            return 2
        return 1 if "test_gpu_backward" in name else 0
    items.sort(key=group)


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def golden():
    import json
    with open(os.path.join(ROOT, "tests", "golden", "worked_examples.json")) as f:
        return json.load(f)
