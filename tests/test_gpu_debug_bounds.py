"""The bounds-checked build on the GPU: on valid inputs it reports no error and
computes exactly what the release build computes (every layer call, bit for
bit); on a corrupted index it reports FLIDE_ERR_BOUNDS with the failing site
instead of making the access.  Each build runs in a child process of its own
(a process loads one library)."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

from tree_forked_decision_b200 import flide

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _child(mode, out_dir, debug):
    env = dict(os.environ, FLIDE_DEBUG_BOUNDS="1" if debug else "0")
    out = subprocess.run([sys.executable, os.path.join(HERE, "_debug_bounds_cases.py"), mode, out_dir],
                         env=env, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-3000:]


def test_debug_build_matches_release_build(tmp_path):
    rel, dbg = tmp_path / "release", tmp_path / "debug"
    rel.mkdir()
    dbg.mkdir()
    _child("run", str(rel), debug=False)
    _child("run", str(dbg), debug=True)
    r_rel = json.loads((rel / "result.json").read_text())
    r_dbg = json.loads((dbg / "result.json").read_text())
    assert r_rel.pop("debug_bounds") == 0 and r_dbg.pop("debug_bounds") == 1
    assert all(v == 0 for v in r_dbg.values()), r_dbg
    assert r_rel == r_dbg
    a_rel, a_dbg = np.load(rel / "arrays.npz"), np.load(dbg / "arrays.npz")
    assert sorted(a_rel.files) == sorted(a_dbg.files)
    for k in a_rel.files:
        assert np.array_equal(a_rel[k], a_dbg[k], equal_nan=True), k


def test_debug_build_reports_a_corrupted_node_id(tmp_path):
    _child("corrupt", str(tmp_path), debug=True)
    res = json.loads((tmp_path / "corrupt.json").read_text())
    assert res["tc"][0] == flide.ERR_BOUNDS and res["tc"][1] == 205, res
    assert res["portable"][0] == flide.ERR_BOUNDS and res["portable"][1] == 301, res
    assert res["tc"][2] == res["portable"][2] == 2 + 2 * 7, res  # the planted id: N + 2
