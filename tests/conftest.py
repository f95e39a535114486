import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")


def pytest_collection_modifyitems(config, items):
    # Skip GPU tests cleanly on a host without CUDA only when they were not
    # selected explicitly with -m gpu (then a missing GPU must fail loudly).
    markexpr = config.getoption("-m") or ""
    if "gpu" in markexpr and "not gpu" not in markexpr:
        return
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if not has_gpu:
        skip = pytest.mark.skip(reason="no CUDA device")
        for item in items:
            if "gpu" in item.keywords:
                item.add_marker(skip)


@pytest.fixture(autouse=True)
def _device_error_word_stays_clear(request):
    """After every GPU test, the library's device error word must be clear:
    a bounded wait that ran out inside any kernel fails the test that ran it
    (the wait-timeout self-test clears the word itself)."""
    yield
    if "gpu" not in request.keywords:
        return
    import w4a4_int4_quantized_b200 as w4
    if w4._lib is None:
        return
    code = w4.w4a4_get_device_error()
    assert code == 0, f"device error word {code:#x} after {request.node.name}"
