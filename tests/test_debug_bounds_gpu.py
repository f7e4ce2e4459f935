"""The bounds-checking debug build (libcpattn_debug.so, -DCP_DEBUG): every global index a
kernel computes is checked against its buffer.  Run over a workload that touches every
kernel path, it must record no violation (CP_ERR_BOUNDS) and give the same bytes as the
release build, since the checks change no arithmetic.  This stands in for a memory
checker, which is not available here."""

import json
import os
import subprocess
import sys

import pytest

from context_attention_dit_b200 import binding
from context_attention_dit_b200 import build as libbuild
from tests import bounds_workload

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_no_violations_and_same_results():
    assert os.path.exists(libbuild.LIB_DEBUG), "libcpattn_debug.so not built (build_debug)"
    env = dict(os.environ, CPATTN_LIB="debug", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "tests.bounds_workload"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    debug = json.loads(r.stdout.strip().splitlines()[-1])
    release = bounds_workload.run()
    assert set(debug) == set(release)
    for name in release:
        assert debug[name]["status"] == 0, f"{name}: debug build reported status {debug[name]['status']}"
        assert release[name]["status"] == 0, name
        assert debug[name]["digest"] == release[name]["digest"], f"{name}: debug and release outputs differ"
    assert binding.CP_ERR_BOUNDS == -7
