"""The checked build (FKM_CHECKED): its kernels verify every gather and
scatter index they use and record an out-of-range one in the status word
instead of touching memory.  The compute sanitizer is not available here,
so this build stands in for its out-of-bounds check: the main paths on odd
shapes (tests/checked_paths.py, run in a process that loads
libfkm_checked.so) must finish with a clean status and oracle parity."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_main_paths_are_clean_in_the_checked_build():
    from exact_means_clustering_b200 import build
    lib = build.build(checked=True)
    assert os.path.exists(lib)
    env = dict(os.environ, FKM_LIB_VARIANT="checked")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_paths.py")],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "all paths clean in the checked build" in r.stdout
