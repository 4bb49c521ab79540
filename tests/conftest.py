import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built CUDA library")


@pytest.fixture(autouse=True)
def _no_internal_index_failure(request):
    """After every GPU test: no kernel reported a failed internal index check (a bit only the
    PA_DEBUG build can set).  When PA_B200_EXPECT_DEBUG is set, the loaded library must be that build."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import paged_kv_cache_457_b200 as pa
    if pa._lib is None:
        return
    if os.environ.get("PA_B200_EXPECT_DEBUG"):
        assert pa.build_flags() & pa.BUILD_DEBUG, "expected the PA_DEBUG build of the library"
    status = pa.device_status(clear=False)
    assert not status & pa.DEV_ERR_INTERNAL, f"a PA_DEBUG index check failed (status {status:#x})"
