"""The bounds-checking build (-DBSQ_DEBUG, libbsq_debug.so) runs every entry
point on tiny and ragged shapes without a single failed index check, and its
results equal the oracle's.  It runs in a child process so that the debug
library, not the normal one, is the one loaded."""
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT

pytestmark = pytest.mark.gpu


def test_debug_build_no_failed_index_checks():
    from fp8_microscaling_quantization_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, BSQ_LIBRARY=lib)
    child = os.path.join(ROOT, "tests", "debug_build_child.py")
    r = subprocess.run([sys.executable, child], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("{")][-1]
    res = json.loads(line)
    assert res["failed_checks"] == 0, res
