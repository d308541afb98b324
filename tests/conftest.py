import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _debug_bounds_clean(request):
    """Under WAN_DEBUG_BOUNDS=1 (the package then loads the debug-bounds
    library), every GPU test must also leave no failed device-side index
    check behind."""
    yield
    if os.environ.get("WAN_DEBUG_BOUNDS") != "1" or request.node.get_closest_marker("gpu") is None:
        return
    import video_diffusion_transformer_packed_b200 as wan
    enabled, count, site, offset = wan.debug_bounds()
    assert enabled, "WAN_DEBUG_BOUNDS=1, but the loaded library is not the debug-bounds build"
    assert count == 0, f"{count} device-side index checks failed; the first at site {site}, element offset {offset}"
