"""The bounds-checked build (libbitsmoe_checked.so, compiled with
-DBITSMOE_CHECKED): every computed shared-memory and global index of the
expert kernels is checked against its extent, and a violation sets the status
bit BITSMOE_ST_BOUNDS instead of faulting.  The small parity cases run through
it in a process of their own (the library is chosen when it is first loaded),
at one token and at every token, with status 0 and oracle parity."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_checked_build_small_cases():
    from mixed_precision_decode_b200 import build
    build.build(checked=True)
    env = dict(os.environ, BITSMOE_CHECKED="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_cases.py")], capture_output=True, text=True,
                       timeout=600, env=env)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "checked ok" in r.stdout
    assert r.stdout.count("ok ") >= 6
