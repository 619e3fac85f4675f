"""The MOE_DEBUG build on the GPU: tests/debug_build_case.py runs in a
process of its own with MOE_DEBUG=1 (the binding then loads
libmoe_debug.so): layer parity, and corrupt caller indices flagged with
MOE_DEV_BAD_INDEX instead of being read or written out of bounds."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_checks_caller_indices():
    from mixture_experts_layer_33_b200 import build
    build.build(debug=True)
    env = dict(os.environ, MOE_DEBUG="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_case.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("DEBUG_BUILD_CASE ")][-1]
    res = json.loads(line.split(" ", 1)[1])
    assert res["lib"] == "libmoe_debug.so"
    assert res["parity_mmoe"] <= 2e-2 and res["parity_ecdit"] <= 2e-2
    assert res["offsets_flag"] & 16 and res["rows_flag"] & 16
    assert all(f & 16 for f in res["token_list_flags"])
