import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")
    config.addinivalue_line("markers", "debug_failure_expected: the test makes an index check fail on purpose")


@pytest.fixture(autouse=True)
def _guard_bands(request):
    """For GPU tests: every buffer the binding allocates gets guard bands,
    checked after the test (see tests/gpu_util.py)."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import torch
    if not torch.cuda.is_available():
        yield
        return
    from tests import gpu_util
    from vision_language_model_b200 import vlm
    guard = gpu_util.Guard()
    old = vlm.set_allocator(guard)
    gpu_util._active_guard = guard
    try:
        yield
    finally:
        vlm.set_allocator(old)
        gpu_util._active_guard = None
    guard.check()
    # under the index-checked debug build (VLM_B200_LIBRARY=libvlm_b200_debug.so)
    # no check may have failed during the test
    if vlm._lib is not None and vlm.debug_build() and not request.node.get_closest_marker("debug_failure_expected"):
        code = vlm.debug_checks()
        assert code == 0, f"index check failed in file {code >> 16}, line {code & 0xFFFF}"
