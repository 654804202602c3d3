"""CPU checks of the C-ABI library: it loads without a GPU and exports every
function include/flide.h declares; the binding mirrors the header's structs."""
import ctypes
import os
import re
import subprocess


from tree_forked_decision_b200 import flide

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flide.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(flide_[a-z0-9_]+)\s*\(", src)))


def test_library_exists_and_loads():
    assert os.path.exists(flide.LIB_PATH), "run tree_forked_decision_b200.build first"
    flide.load()


def test_exports_every_declared_symbol():
    declared = _declared()
    assert declared, "no declarations parsed"
    out = subprocess.run(["nm", "-D", "--defined-only", flide.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(flide_\w+)", out))
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    assert sorted(flide.SYMBOLS) == declared


def test_struct_layouts_match_header():
    src = open(HEADER).read()
    structs = dict((name, body) for body, name in re.findall(r"typedef struct \{([^}]*)\} (\w+);", src))
    body = structs["flide_tree_index"]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\*(\w+)", body)
    assert names == flide.INDEX_ARRAYS
    assert ctypes.sizeof(flide.TreeIndexC) == 16 + 8 * len(flide.INDEX_ARRAYS) + 8
    assert ctypes.sizeof(flide.TreeDesc) == 16 + 8 * 4


def test_host_only_entry_points():
    lib = flide.load()
    n = lib.flide_tree_index_bytes(4, 30, 1000, 3)
    assert n > 0 and n % 256 == 0
    assert lib.flide_tree_index_bytes(-1, 3, 3, 1) == 0
    # arrays past int32 indexing are refused (ancestor lists: N * (max_depth + 1))
    assert lib.flide_tree_index_bytes(1, 2 ** 31 - 1, 10, 2 ** 31 - 1) == 0
    assert lib.flide_tree_index_bytes(1, 2 ** 20, 10, 2 ** 11) == 0
    assert lib.flide_tree_index_bytes(1, 2 ** 20, 10, 2 ** 11 - 2) > 0
    assert lib.flide_tree_index_init(ctypes.byref(flide.TreeIndexC()), ctypes.c_void_p(1 << 20),
                                     1 << 40, 1, 2 ** 20, 10, 2 ** 11) == flide.ERR_SHAPE
    idx = flide.TreeIndexC()
    # host-only layout over a fake, aligned address: no device access happens
    base = 1 << 20
    assert lib.flide_tree_index_init(ctypes.byref(idx), ctypes.c_void_p(base), n, 4, 30, 1000, 3) == 0
    ptrs = [getattr(idx, a) for a in flide.INDEX_ARRAYS]
    assert all(p % 256 == 0 for p in ptrs) and ptrs == sorted(ptrs) and ptrs[0] == base
    assert ptrs[-1] < base + n
    assert lib.flide_tree_index_init(ctypes.byref(idx), ctypes.c_void_p(base), n - 1, 4, 30, 1000, 3) == flide.ERR_CAPACITY
    assert lib.flide_tree_index_init(ctypes.byref(idx), ctypes.c_void_p(base + 4), n, 4, 30, 1000, 3) == flide.ERR_SHAPE
    for code in range(7):
        assert lib.flide_strerror(code) and lib.flide_strerror(code) != b"unknown status"
    assert lib.flide_strerror(7) == b"unknown status"
    assert lib.flide_debug_bounds() == 0  # the release build
