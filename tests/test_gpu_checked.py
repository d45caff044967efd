"""The checked build (SS_BOUNDS_CHECK) on the small and odd shapes.

In that build every global index a kernel forms is compared with its
tensor's extent before the access; a miss is skipped and recorded in the
device error word (no trap), and ss_last_device_error reports it as
SS_ERR_BOUNDS.  This runs the parity tests of small, ragged and unaligned
shapes -- the forward (plain, segmented, balanced, from a carried state, fused
convolution, exact zero-order hold) and the decode step -- against
libssscan_checked.so in a child process, with every test followed by a check
that the error word is clear.  It stands in for a memory checker.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SELECTION = [
    "tests/test_gpu_parity.py::test_small_shapes",
    "tests/test_gpu_parity.py::test_optional_inputs",
    "tests/test_gpu_parity.py::test_unaligned_fallback_path",
    "tests/test_gpu_parity.py::test_index_plumbing_distinct_values",
    "tests/test_gpu_segments.py",
    "tests/test_gpu_schedule.py::test_forced_split_parity",
    "tests/test_gpu_state.py",
    "tests/test_gpu_conv.py::test_conv_small_shapes",
    "tests/test_gpu_zoh.py::test_zoh_small_shapes",
]


def test_small_shapes_under_the_checked_build():
    from selective_state_space_ss_b200 import build as B

    lib = B.build_checked()
    env = dict(os.environ, SSSCAN_LIBRARY=lib, SS_CHECK_ERROR_WORD="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        *SELECTION], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
