import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: long host-side computation")


_FATAL_MARKERS = ("CUDA error", "illegal", "FA_ERR_CUDA", "misaligned address", "unspecified launch failure")


@pytest.hookimpl(hookwrapper=True)
def pytest_runtest_makereport(item, call):
    """Stop the whole session after a CUDA-level failure (a numerical mismatch does not stop it):
    nothing else runs on a device context that reported an error."""
    outcome = yield
    rep = outcome.get_result()
    if rep.failed and call.excinfo is not None:
        text = str(call.excinfo.value)
        if any(m in text for m in _FATAL_MARKERS):
            item.session.shouldstop = f"CUDA-level failure in {item.nodeid}: {text[:200]}"
