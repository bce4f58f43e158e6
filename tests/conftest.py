import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")
    config.addinivalue_line(
        "markers", "late(rank): run after every unranked test, in increasing rank")


def pytest_collection_modifyitems(config, items):
    """Run order: every test without a `late` mark first, in collection order,
    then the `late(rank)` ones by rank (full-size and long-running suites,
    the canary sweep, the no-alloc entry point last).  A run that stops at
    its first failure has then run every test ranked before the failing one.
    The sort is stable, so tests of one rank keep their collection order."""
    def rank(item):
        m = item.get_closest_marker("late")
        return m.args[0] if m is not None else 0
    items[:] = sorted(items, key=rank)


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
