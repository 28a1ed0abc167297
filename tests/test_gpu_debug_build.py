"""The debug build of the library (libthink_debug.so, compiled with
-DTHINK_DEBUG): index checks at the global stores set THINK_DEVICE_OOB in the
device status word instead of writing out of range.  The canary tests run on
it in a child process (the library is chosen when the package is imported);
their status checks require the OOB bit to stay clear and their canaries to
stay intact."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_canaries_on_the_debug_build():
    env = dict(os.environ, THINK_DEBUG_LIB="1")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join("tests", "test_gpu_canary.py"), "-q", "-x",
                        "-p", "no:cacheprovider", "-m", "gpu"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "passed" in r.stdout
