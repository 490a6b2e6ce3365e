"""The index-checking build (libinvnum_debug.so, -DINV_DEBUG_BOUNDS).

* Its check itself: a kernel that stores past its declared extent has those
  stores skipped and reports INV_ERR_BOUNDS (the buffer beyond the extent,
  inside a canary band, stays untouched).
* The GPU parity, invariance and canary tests run again, in a child process,
  against the checking build: every index every kernel computes on those
  shapes lies inside its buffer (any that did not would record
  INV_ERR_BOUNDS, which every one of those tests asserts is absent), and the
  results still match the oracle.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _debug_lib():
    from invariant_numerics_b200 import build
    return build.build(debug_bounds=True)


def test_checking_build_skips_and_reports_an_out_of_extent_store():
    path = _debug_lib()
    code = f"""
import os, sys, torch
os.environ["INVNUM_LIBRARY"] = {path!r}
sys.path.insert(0, {ROOT!r})
from invariant_numerics_b200 import invnum as inv
assert inv.inv_debug_bounds_enabled()
assert inv.inv_get_device_status() == inv.INV_OK
band = torch.full((1024 + 64,), -1.0, device="cuda")   # 1000 declared floats, then a band
inv.inv_selftest_bounds(band[:1000], 1000, 1000)
assert inv.inv_get_device_status() == inv.INV_OK
assert torch.equal(band[:1000], torch.arange(1000, dtype=torch.float32, device="cuda"))
band.fill_(-1.0)
inv.inv_selftest_bounds(band[:1000], 1000, 1088)
assert inv.inv_get_device_status() == inv.INV_ERR_BOUNDS
assert torch.equal(band[:1000], torch.arange(1000, dtype=torch.float32, device="cuda"))
assert bool((band[1000:] == -1.0).all())
print("ok")
"""
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


def test_gpu_suite_passes_on_the_checking_build():
    path = _debug_lib()
    env = dict(os.environ, INVNUM_LIBRARY=path)
    files = ["tests/test_gpu_kernels.py", "tests/test_gpu_layer.py", "tests/test_gpu_lamp.py",
             "tests/test_gpu_canary.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *files],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and " skipped" not in r.stdout
