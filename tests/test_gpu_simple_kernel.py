"""The one-CTA-per-query-block kernel (the library's path for calls beyond the
pipelined kernel's limits, also selected by LIBPREFILL_KERNEL=simple) against
the oracle: a selection of the parity tests re-run in a child process with
that variable set, so that this kernel is checked on the same cases."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SELECTION = [
    "tests/test_gpu_parity.py::test_single_sequence_lengths",
    "tests/test_gpu_parity.py::test_head_groupings",
    "tests/test_gpu_parity.py::test_varlen_with_empty_and_ragged_sequences",
    "tests/test_gpu_parity.py::test_chunked_matches_oracle",
    "tests/test_gpu_parity.py::test_first_row_is_v0_bit_exact",
    "tests/test_gpu_window.py::test_window_single_sequence",
    "tests/test_gpu_window.py::test_window_chunked",
    "tests/test_gpu_window.py::test_window_one_returns_own_value_bit_exact",
]


def test_simple_kernel_parity_selection():
    env = dict(os.environ, LIBPREFILL_KERNEL="simple")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        *SELECTION], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
