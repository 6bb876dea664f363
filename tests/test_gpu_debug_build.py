"""The bounds-checked build (libsfc_debug.so, -DSFC_DEBUG: every scratch
access tested against its protocol region on the device) runs the parity
matrix without recording an out-of-region access. It runs in a subprocess
because the library is chosen when the binding first loads it."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
DEBUG_LIB = os.path.join(ROOT, "latency_self_synchronizing_b200", "libsfc_debug.so")


def test_debug_build_parity_without_scratch_violations():
    if not os.path.exists(DEBUG_LIB):
        from latency_self_synchronizing_b200 import build
        build.build(debug=True)
    env = dict(os.environ, SFC_LIB=DEBUG_LIB, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    res = subprocess.run([sys.executable, os.path.join(HERE, "_debug_parity_body.py")], env=env, cwd=ROOT,
                         capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    assert "no out-of-region scratch access" in res.stdout
