"""The debug build (librmt_debug.so: the library compiled with -DRMT_DEBUG) on the GPU.

compute-sanitizer cannot be used where this library is tested, so the debug build stands in
for it: every kernel reads its cells through a check of each index against the buffers the
host sized for that forward and reports a violation through the error word (RMT_EDEBUG at
rmt_sync) instead of making the access. These tests run parity cases of tests/test_forward.py
and tests/test_kernels.py against the debug build in a child process (the binding loads the
library named by RMT_LIBRARY): they must pass with no check firing, which shows that every
index those cases take stays inside its buffer. A self-check shows that the check does fire.
"""
import os
import subprocess
import sys

import pytest

from recurrent_memory_transformer_anti_b200 import rmt

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# small shapes that cover every kernel: fp32 and bf16 forwards (single-CTA and CTA-pair GEMMs,
# both attention kernels, the fused and separate memory reads), short segments, batches, the
# comparison model, and the kernel-level entry points
CASES = ("tests/test_forward.py::test_tiny_fp32_matches_oracle "
         "tests/test_forward.py::test_small_bf16_matches_oracle "
         "tests/test_forward.py::test_bf16_tile_paths_match_oracle "
         "tests/test_forward.py::test_short_last_segment_matches_oracle "
         "tests/test_forward.py::test_batch_matches_oracle_and_each_sequence_alone "
         "tests/test_forward.py::test_full_attention_matches_oracle "
         "tests/test_forward.py::test_random_bf16_shapes_match_oracle "
         "tests/test_kernels.py")


def _child(args, timeout=900):
    env = dict(os.environ, RMT_LIBRARY=rmt.DEBUG_LIB_PATH)
    return subprocess.run([sys.executable, *args], cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def test_parity_cases_pass_on_the_debug_build(cuda_ok):
    assert os.path.exists(rmt.DEBUG_LIB_PATH)
    r = _child(["-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *CASES.split()])
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]


def test_debug_build_bounds_check_fires(cuda_ok):
    code = ("from recurrent_memory_transformer_anti_b200 import rmt\n"
            "assert rmt.LIB_PATH == rmt.DEBUG_LIB_PATH\n"
            "rmt.rmt_bounds_selftest()\n"
            "try:\n"
            "    rmt.rmt_sync(None)\n"
            "    raise SystemExit('no error reported')\n"
            "except rmt.RmtError as e:\n"
            "    assert e.status == rmt.RMT_EDEBUG, e\n"
            "    assert 'error word 64)' in str(e), e\n"
            "rmt.rmt_sync(None)\n"  # the word was cleared; the context is still usable
            "print('bounds check ok')\n")
    r = _child(["-c", code], timeout=300)
    assert r.returncode == 0 and "bounds check ok" in r.stdout, r.stdout + r.stderr
