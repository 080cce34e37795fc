"""The parity and corrupt-input tests once more under the checks build.

libdfw_checks.so is libdfw compiled with DFW_CHECKS: every copy range,
shared-memory extent and output index the kernels compute is checked against
its buffer before use, a failing access is skipped, and the first failing
site is recorded (dfw_checks_report).  This is the library's stand-in for a
memory checker.  The small-size GPU tests (the full-size ones are left out
for time) run in a child process with DFW_LIBRARY=checks; after each test the
conftest fixture fails it if any check fired.  The corrupt-input cases
matter most here: their damage must be caught by the kernels' own validation,
never by an access outside a buffer.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_decode.py", "tests/test_gpu_closed.py", "tests/test_gpu_seq.py", "tests/test_gpu_rans.py",
          "tests/test_gpu_encode.py", "tests/test_gpu_encode_multi.py", "tests/test_gpu_gemv.py",
          "tests/test_gpu_failure.py"]


def test_parity_and_corrupt_inputs_under_the_checks_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_entropy_coded_canonical_b200.build import build
    build(checks=True)
    env = dict(os.environ, DFW_LIBRARY="checks")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        "-k", "not full_size and not fullsize", *SUITES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=840)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-25:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
