"""The debug build (libstd_b200_debug.so: the same kernels compiled with STD_DEBUG, every
index and cache row bounds-checked on the device, a failed check reported as
STD_DEVERR_DEBUG and the access skipped, never a trap) runs the canary-guarded parity
cases of test_gpu_canaries.py in a process of its own, and passes them: results match
the oracle, no guard byte changes and no device check fires."""
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def test_debug_build_passes_the_canary_cases():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    lib = os.path.join(ROOT, "sparse_top_kv_std_b200", "libstd_b200_debug.so")
    if not os.path.exists(lib):
        from sparse_top_kv_std_b200 import build
        build.build(debug=True)
    env = dict(os.environ, STD_B200_DEBUG="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_canaries.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout, r.stdout[-2000:]
