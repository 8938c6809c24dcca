"""dla_decode_step_static refuses a cache whose scratch need exceeds its
static array, before it touches a device.

The call runs in a child process with no visible GPU and dummy pointers: the
size check must return DLA_ERR_WORKSPACE first.  If it ever regressed, the
call would reach the CUDA runtime, find no device and return DLA_ERR_CUDA;
nothing is launched on the dummy pointers either way.
"""
import os
import subprocess
import sys

from tests.test_zz_no_alloc import _REJECT

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_static_scratch_rejects_oversized_cache_without_a_device():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", _REJECT, ROOT], env=env, capture_output=True,
                       text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().splitlines()[-1] == "5"  # DLA_ERR_WORKSPACE
