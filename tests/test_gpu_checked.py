"""The range-checked build (libeta_checked.so, -DETA_CHECKED) on the GPU.

Every global load or store whose index a kernel computes from values it reads on
the device (lengths, block lists and counts, the share plan, partial-slot numbers,
key-tile ranges) is range-checked first in that build; an index outside its buffer
sets ETA_DEVSTAT_BOUNDS, skips the access and prints the file and line.  compute-
sanitizer is not relied on, so these tests stand in for its memcheck:
  * the check itself reports (and the release build compiles it away), on an index
    that is never dereferenced;
  * the parity, fused-step, prefill, robustness and no-allocation suites pass
    unchanged under the checked build, and no range report is printed."""
import os
import subprocess
import sys

import pytest
import torch

from long_context_decoding_eta_b200 import _lib as L

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REPORT = "eta checked build:"


def _checked_env():
    from long_context_decoding_eta_b200 import build
    build.build(checked=True)
    return dict(os.environ, ETA_CHECKED="1", PYTHONPATH=ROOT)


def test_release_build_compiles_the_check_away():
    assert not L.eta_build_checked()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.eta_selftest_bounds(10, 4, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_checked_build_reports_an_out_of_range_index():
    code = """
import torch
from long_context_decoding_eta_b200 import _lib as L
assert L.eta_build_checked()
st = torch.zeros(1, dtype=torch.int32, device="cuda")
for i, n in ((0, 4), (3, 4)):
    L.eta_selftest_bounds(i, n, st)
torch.cuda.synchronize()
print("inside", int(st.item()))
for i, n in ((4, 4), (-1, 4)):
    st.zero_()
    L.eta_selftest_bounds(i, n, st)
    torch.cuda.synchronize()
    print("outside", int(st.item()), L.eta_status_from_device(int(st.item())))
"""
    p = subprocess.run([sys.executable, "-c", code], env=_checked_env(), capture_output=True,
                       text=True, timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stdout + p.stderr
    assert "inside 0" in p.stdout
    assert p.stdout.count("outside %d 7" % L.DEVSTAT_BOUNDS) == 2, p.stdout
    # the first report of the source file is printed with its location
    assert p.stdout.count(REPORT) == 1 and "selftest.cu" in p.stdout, p.stdout


def test_suites_pass_under_the_checked_build():
    files = ["tests/test_gpu_parity.py", "tests/test_gpu_fused.py", "tests/test_gpu_prefill.py",
             "tests/test_gpu_robustness.py", "tests/test_gpu_sharded.py",
             "tests/test_zz_no_alloc.py"]
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-s", "-m", "gpu",
                        "-p", "no:cacheprovider", *files],
                       env=_checked_env(), capture_output=True, text=True, timeout=3000, cwd=ROOT)
    tail = "\n".join((p.stdout + p.stderr).splitlines()[-30:])
    assert p.returncode == 0, tail
    assert REPORT not in p.stdout and REPORT not in p.stderr, tail
    assert " passed" in p.stdout, tail
