import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU oracle runs")
    config.addinivalue_line("markers", "debug_trips: trips an index check of the debug build on purpose")


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _debug_check_word(request):
    """With the debug build loaded (KV_DEBUG_CHECKS=1), no GPU test may trip an
    index check unless it expects to (marker debug_trips)."""
    yield
    import kv_cache_compression_layer_b200 as kv

    if not (kv.DEBUG_CHECKS and request.node.get_closest_marker("gpu")):
        return
    word = kv.kv_debug_check_word(clear=True)
    if not request.node.get_closest_marker("debug_trips"):
        assert word == 0, f"index check tripped: {word:#x}"
