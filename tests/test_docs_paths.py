"""Every repository path the documents cite exists (the design doc's file map,
README.md, the profile index), so a renamed or removed file cannot leave a
stale reference behind.  Bare kernel file names resolve under the package's
csrc/ directory; the one path that belongs to the pages' own project is
listed separately."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "tree_forked_decision_b200")
NOT_HERE = {"flide/kernels/gdn.py"}  # the pages' GDN kernel, prior art named in the design doc


@pytest.mark.parametrize("doc", ["DESIGN.md", "README.md", "profiles/README.md"])
def test_cited_paths_exist(doc):
    text = open(os.path.join(ROOT, doc)).read()
    paths = set(re.findall(r"`([A-Za-z0-9_./-]+\.(?:py|cu|cuh|h|md|json|c))`", text))
    assert paths
    missing = [p for p in sorted(paths - NOT_HERE)
               if not any(os.path.exists(os.path.join(base, p))
                          for base in (ROOT, PKG, os.path.join(PKG, "csrc"), os.path.join(ROOT, "profiles")))]
    assert not missing, missing
