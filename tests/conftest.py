import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def _has_cuda():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if _has_cuda():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _guard_bands_intact(request):
    """With MUON_GUARD_BANDS=1 (the library lays out guard bands after every
    workspace region), every GPU test ends by checking that no launch wrote
    into them."""
    yield
    if os.environ.get("MUON_GUARD_BANDS") != "1" or "gpu" not in request.keywords or not _has_cuda():
        return
    import muon_newton_schulz_02_b200 as muon
    if muon._lib is None:
        return
    changed = muon.guard_check()
    assert changed == 0, f"{changed} guard-band bytes were overwritten"
