"""The bounds-checked build (libflide_dbg.so) on the CPU: it exists (built by
__graft_entry__.build(), or here), loads when FLIDE_DEBUG_BOUNDS=1 selects it,
exports every symbol of include/flide.h and says it is the checked build."""
import os
import subprocess
import sys

from tree_forked_decision_b200 import build as flide_build
from tree_forked_decision_b200 import flide

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_library_loads_and_reports_itself():
    if not os.path.exists(flide_build.LIB_DBG):
        flide_build.build(debug_bounds=True)
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from tree_forked_decision_b200 import flide\n"
            "lib = flide.load()\n"
            "assert flide.LIB_PATH.endswith('libflide_dbg.so'), flide.LIB_PATH\n"
            "assert lib.flide_debug_bounds() == 1\n"
            "assert lib.flide_strerror(flide.ERR_BOUNDS) != b'unknown status'\n"
            "print('ok')\n") % ROOT
    env = dict(os.environ, FLIDE_DEBUG_BOUNDS="1")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip().endswith("ok")


def test_release_library_is_unchecked():
    assert flide.load().flide_debug_bounds() == 0
