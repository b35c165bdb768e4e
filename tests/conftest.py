import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) and the built libqlora")
    config.addinivalue_line("markers", "slow: CPU test that takes tens of seconds")


@pytest.fixture(autouse=True)
def _restore_library_state(request):
    """The GEMM tile configuration and the persistent-grid cap are process-wide
    settings of the library; every GPU test starts with configuration 4 (the
    staged feed; a test that wants another, or the automatic setting, sets it)
    and no cap, and leaves both as it found them, whatever order the tests run
    in."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    from qlora_fine_tuning_nf4_b200 import ops
    prev_tiles = ops.qlora_set_tile_config(4)
    prev_cap = ops.qlora_test_set_grid_cap(0)
    try:
        yield
    finally:
        ops.qlora_set_tile_config(prev_tiles)
        ops.qlora_test_set_grid_cap(prev_cap)
