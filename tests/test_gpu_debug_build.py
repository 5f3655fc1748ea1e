"""The debug build of the library (compiled with -DFS_DEBUG: device-side
bounds checks on the kernels' global, shared and tensor-memory indices that
record FS_ERR_DEVICE_BOUNDS in the status word instead of trapping) over
small and ragged shapes, B in {1, 3, 17}, V in {1, 7, 129, 4097}, d in
{8, 24}, and every kind of call, and over 250 and 256 rows (CTA pairs whose
partial tiles run transposed): no check fires and the tokens match the
oracle.  compute-sanitizer is closed on the test machines; these checks
stand in for it.  The cases run in a child process (tests/debug_build_cases.py)
because a process loads one build of the library."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_small_shapes_report_no_bounds_error():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_head_exact_fmms_b200 import build
    build.build(debug=True)
    env = dict(os.environ, FMMS_LIBRARY="debug")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_cases.py")],
                         env=env, capture_output=True, text=True, timeout=1800, cwd=ROOT)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-3000:]
    assert "34 shapes" in out.stdout
