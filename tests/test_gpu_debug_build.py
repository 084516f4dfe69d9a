"""The index-checked debug build (libvlm_b200_debug.so, compiled with
-DVLM_DEBUG) on the GPU.

In that build every index a kernel computes from tables or data before a
global access is checked; a failing check records a code (file id << 16 |
line) and skips the access instead of trapping. These tests

* make a check fail on purpose (vlm_debug_selftest_bounds: writes past n are
  caught and skipped, the code is recorded, reading it clears it), and
* rerun the kernel, model, front-end, FP8 and NVFP4 parity tests -- a
  tiny-shape run of every kernel of the path -- against the debug build in a
  child process, where the conftest fixture asserts after every test that no
  check failed.

Nothing here faults, traps or hangs a GPU: the failing accesses are exactly
the ones the checks skip.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

_SELFTEST = r"""
import torch
from vision_language_model_b200 import vlm
assert vlm.debug_build()
assert vlm.debug_checks() == 0
n = 300
buf = torch.zeros(2 * n, dtype=torch.int32, device="cuda")
vlm.debug_selftest_bounds(buf, n)
code = vlm.debug_checks()
assert code >> 16 == 1 and code & 0xFFFF > 0, code          # recorded by the small-kernel file
assert torch.equal(buf[:n].cpu(), torch.arange(1, n + 1, dtype=torch.int32))
assert int(buf[n:].abs().sum()) == 0                          # the checked writes were skipped
assert vlm.debug_checks() == 0                                # reading cleared the record
print("debug selftest ok", hex(code))
"""


def _debug_env():
    from vision_language_model_b200 import vlm
    path = vlm.DEBUG_LIB_PATH
    if not os.path.exists(path):
        from vision_language_model_b200 import build
        build.build(debug=True)
    env = dict(os.environ, VLM_B200_LIBRARY=path, PYTHONPATH=ROOT)
    return env


def test_debug_build_check_fails_into_record_and_skips_access():
    r = subprocess.run([sys.executable, "-c", _SELFTEST], cwd=ROOT, env=_debug_env(), capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug selftest ok" in r.stdout


def test_parity_suite_under_debug_build_trips_no_check():
    files = ["tests/test_gpu_kernels.py", "tests/test_gpu_model.py", "tests/test_gpu_frontend.py",
             "tests/test_gpu_fp8.py", "tests/test_gpu_nvfp4.py", "tests/test_gpu_nvfp4_tower.py",
             "tests/test_gpu_fused_scatter.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        "-k", "not full_size and not 1540"] + files,
                       cwd=ROOT, env=_debug_env(), capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-6000:] + r.stderr[-3000:]
    assert " passed" in r.stdout
