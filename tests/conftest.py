import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_sessionstart(session):
    """Build the CUDA library and the oracle if they are missing or stale
    (both builders return at once when up to date), so that the suite runs
    from a fresh checkout."""
    from oracle import build as oracle_build
    from ssm_decode_step_b200 import build as cuda_build
    oracle_build.build()
    cuda_build.build()


@pytest.fixture(autouse=True)
def _oracle_unplanted():
    """Every test starts and ends with the oracle proper: a planted mistake
    (tests/test_oracle_mutations.py) never outlives its own test."""
    import sys as _sys
    O = _sys.modules.get("oracle.oracle")
    if O is not None:
        assert O.planted_fault() == "none", "a planted oracle mistake leaked into this test"
    yield
    O = _sys.modules.get("oracle.oracle")
    if O is not None and O.planted_fault() != "none":
        O._active, O._planted = None, "none"
        raise AssertionError("this test left a planted oracle mistake active")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU test")


def pytest_collection_modifyitems(config, items):
    """GPU tests are skipped (not failed) where no CUDA device is present."""
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
