import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# CQ_TEST_DEBUG_LIB=1: the whole suite runs on the debug build of libcq (in-kernel index checks,
# cell_updates_b200/_build/libcq_debug.so), and after every GPU test the debug word must be 0,
# i.e. no index check fired anywhere in it.
DEBUG_LIB = os.environ.get("CQ_TEST_DEBUG_LIB") == "1"


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    if DEBUG_LIB:
        from cell_updates_b200 import build, cq
        build.build()
        cq.LIBCQ_PATH = build.test_variant_path("debug")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


@pytest.fixture(autouse=True)
def _no_index_check_fired(request):
    yield
    if DEBUG_LIB and request.node.get_closest_marker("gpu") is not None:
        from cell_updates_b200 import cq
        if os.path.basename(cq.LIBCQ_PATH) == "libcq_debug.so":
            assert cq.cq_debug_word() == 0, "an in-kernel index check fired during this test"
