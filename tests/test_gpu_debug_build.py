"""The small parity cases under the debug build (GPU).

libdms_debug.so is compiled from the same sources with DMS_DEBUG defined: every
index the kernels derive by construction (page-table rows and columns, partial
slots, pool rows, free-stack positions) is checked against its buffer, and one
out of range latches DMS_ERR_INVALID and skips the access instead of faulting.
This is the bounds checker of a pool where no memory-checking tool runs. The
cases run in a child process that loads the debug library (DMS_LIBRARY=debug);
they must pass with no check firing (every case asserts DMS_OK).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_small_parity_cases_pass_under_the_debug_build():
    from learned_kv_cache_decode_b200 import build
    assert os.path.exists(build.DEBUG_LIB), "libdms_debug.so is not built"
    env = dict(os.environ, DMS_LIBRARY="debug")
    probe = subprocess.run([sys.executable, "-c", "from learned_kv_cache_decode_b200 import _native; "
                            "_native.load(); print(_native.LIB_PATH)"], cwd=ROOT, env=env, capture_output=True,
                           text=True, timeout=300)
    assert probe.returncode == 0 and probe.stdout.strip().endswith("libdms_debug.so"), probe.stderr
    sel = ("test_small_cases or test_small_cases_fused_step or test_fused_step_schedule_follows_every_change "
           "or test_window_sweep or test_fused_step_pool_exhaustion or test_sequence_reset or dominant "
           "or test_noalloc_permuted_subset")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-k", sel,
                        "tests/test_gpu_parity.py", "tests/test_gpu_dynamic_range.py", "tests/test_zz_no_alloc.py"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
