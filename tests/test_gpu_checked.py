"""GPU parity under the checked build (libcsa_checked.so, compiled with
-DCSA_CHECKED): every gather row of the attention and compression kernels is
bounds-checked on the device, a failed check is recorded in the device error
word that csa_check_device_error reports.  The parity tests run in a child
process that loads that library (CSA_LIBRARY); they must pass and leave no
error recorded."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch, pytest
from long_context_sparse_10_b200 import _lib
assert _lib.LIB_PATH.endswith("libcsa_checked.so"), _lib.LIB_PATH
rc = pytest.main(["-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", "tests/test_gpu_parity.py",
                  "tests/test_gpu_append_packed.py",
                  "-k", "compress or indexer_topk or sparse_mqa or dense_mqa or decode or pipeline or packed"])
lib = _lib.load()
st = lib.csa_check_device_error(torch.cuda.current_stream().cuda_stream)
print("device error status", st, lib.csa_last_error())
sys.exit(int(rc) if rc else (0 if st == 0 else 7))
"""


def test_parity_and_no_bounds_failure_under_the_checked_build():
    from long_context_sparse_10_b200 import build
    path = build.LIB_CHECKED
    if not os.path.exists(path):
        build.build(checked=True)
    env = dict(os.environ, CSA_LIBRARY=path)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
