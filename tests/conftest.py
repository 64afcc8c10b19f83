import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
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


@pytest.fixture(autouse=True)
def _fresh_device_status(request):
    """A GPU test starts with the library's sticky device status cleared, so a
    failure earlier in the session cannot fail it."""
    if "gpu" in request.keywords:
        try:
            import torch
            if torch.cuda.is_available():
                import long_context_indexer_b200 as lci
                try:
                    lci.get_device_status()
                except lci.LciError:
                    pass
        except Exception:  # pragma: no cover
            pass
    yield
