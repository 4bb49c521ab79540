"""The PA_DEBUG build of the library (every index the kernels derive is checked on the device before
use; a failed check skips the access and sets PA_DEV_ERR_INTERNAL) passes the small-shape parity cases
against the oracle and the error-path tests.  The tests run in a child process that loads
libpa_b200_debug.so through PA_B200_LIBRARY; the autouse fixture of conftest.py then checks, after
every test, that the loaded library is the debug build and that no index check failed."""
import os
import subprocess
import sys

import pytest

from paged_kv_cache_457_b200 import build_lib

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    "tests/test_gpu_parity.py::test_small_shapes",
    "tests/test_gpu_parity.py::test_small_batch_segment_path",
    "tests/test_gpu_parity.py::test_many_short_sequences",
    "tests/test_gpu_parity.py::test_shared_prefix_tables",
    "tests/test_gpu_parity.py::test_shared_prefix_bad_block_zeroes_only_its_sequence",
    "tests/test_gpu_cascade.py::test_cascade_planted_groups",
    "tests/test_gpu_cascade.py::test_cascade_device_checks",
    "tests/test_gpu_errors.py",
    "tests/test_gpu_properties.py",
    "tests/test_gpu_launch_config.py",
    "tests/test_gpu_prefill.py::test_prefill_matches_oracle",
    "tests/test_gpu_prefill.py::test_empty_sequences_and_larger_grid",
    "tests/test_gpu_prefill.py::test_bad_page_and_bad_context_zero_their_rows",
    "tests/test_gpu_prefill.py::test_max_query_len_too_small_is_flagged",
    "tests/test_gpu_blocks.py::test_copy_blocks_matches_oracle",
    "tests/test_gpu_blocks.py::test_copy_blocks_out_of_range_is_flagged_and_skipped",
]


def test_debug_build_passes_small_parity_and_error_cases():
    lib = build_lib.build(debug=True)
    env = dict(os.environ, PA_B200_LIBRARY=lib, PA_B200_EXPECT_DEBUG="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider"] + CASES
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = (r.stdout + r.stderr)[-4000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail
