import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    # The oracle's mutation test points this at a deliberately altered copy.
    alt = os.environ.get("MUSE_ORACLE_SO")
    return oracle.Oracle(alt) if alt else oracle.default()


def pytest_collection_modifyitems(config, items):
    # GPU tests run only when a CUDA device is present; on CPU-only hosts they
    # are skipped rather than failing at device allocation.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
