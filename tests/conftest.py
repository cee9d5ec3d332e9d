import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


@pytest.fixture(scope="session")
def oracle_pool():
    """Threads for running the single-threaded C oracle on slices of large
    inputs in parallel (ctypes releases the interpreter lock during a call)."""
    from concurrent.futures import ThreadPoolExecutor
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    with ThreadPoolExecutor(max(1, min(64, n or 1))) as ex:
        yield ex


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a) and the built "
        "CUDA library")


def pytest_collection_modifyitems(config, items):
    # gpu tests need a device; skip them cleanly when there is none so that
    # `-m "not gpu"` and plain runs on CPU hosts stay green.
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
