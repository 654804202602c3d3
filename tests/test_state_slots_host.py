"""Host query of the node-state slots (flide_tree_state_slots) on the CPU.

The count must equal what flide_tree_build writes to counts["SLOTS"] (the GPU
side of that is test_gpu_slots.py).  Here it is checked against a brute-force
walk written in the test: depth by following parents, inner nodes (nodes with
children) counted per depth, one slot per non-empty request's root plus the
widest odd and the widest even depth >= 2 (techfi24.com, "Limites et
perspectives": memory for cloned states bounds the number of options)."""
import ctypes

import numpy as np
import pytest

from tree_forked_decision_b200 import flide, inputs


def _walk_slots(rp, parent):
    R = len(rp) - 1
    roots, per_depth = 0, {}
    for r in range(R):
        n0, n1 = int(rp[r]), int(rp[r + 1])
        if n1 > n0:
            roots += 1
        depth = {}
        inner = set()
        for n in range(n0, n1):
            d, cur = 0, n
            while parent[cur] >= 0:
                cur = n0 + int(parent[cur])
                d += 1
            depth[n] = d
            if parent[n] >= 0:
                inner.add(n0 + int(parent[n]))
        for n in inner:
            if depth[n] >= 1:
                per_depth[depth[n]] = per_depth.get(depth[n], 0) + 1
    odd = max([c for d, c in per_depth.items() if d % 2 == 1], default=0)
    even = max([c for d, c in per_depth.items() if d % 2 == 0], default=0)
    return roots + odd + even


@pytest.mark.parametrize("seed", range(12))
def test_host_query_equals_walk_on_random_trees(seed):
    rng = np.random.default_rng(seed)
    tree = inputs.leveled_tree(rng, int(rng.integers(1, 7)), depth_range=(1, 6),
                               options_range=(2, 40), prefix_range=(1, 9), n_resume=0)
    rp, parent, _seg, _past = tree.arrays()
    assert flide.state_slots(tree) == _walk_slots(rp, parent)


def test_host_query_special_cases():
    # empty requests count no root; a depth-8 chain reuses two regions
    chain = inputs._tree([(0, [(-1, 3)] + [(i, 2) for i in range(8)])], 8)
    assert flide.state_slots(chain) == 1 + 1 + 1
    empty = inputs._tree([(0, []), (0, [(-1, 4), (0, 2)]), (0, [])], 1)
    assert flide.state_slots(empty) == 1
    fan = inputs.fanout_tree(3, 16, 9, 2)
    assert flide.state_slots(fan) == 3


def _call(R, rp, parent, with_out=True):
    out = ctypes.c_int32(-7)
    rpa = None if rp is None else np.ascontiguousarray(rp, np.int32)
    pa = None if parent is None else np.ascontiguousarray(parent, np.int32)
    ptr = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
    code = flide._lib().flide_tree_state_slots(R, ptr(rpa), ptr(pa),
                                               ctypes.byref(out) if with_out else None)
    return code, out.value


def test_host_query_refusals():
    assert _call(1, [0, 2], [-1, 0])[0] == flide.OK
    assert _call(-1, [0], [])[0] == flide.ERR_SHAPE
    assert _call(1, None, [-1])[0] == flide.ERR_SHAPE
    assert _call(1, [0, 2], None)[0] == flide.ERR_SHAPE
    assert _call(1, [0, 2], [-1, 0], with_out=False)[0] == flide.ERR_SHAPE
    assert _call(1, [1, 2], [-1, 0])[0] == flide.ERR_INVALID     # does not start at 0
    assert _call(2, [0, 2, 1], [-1, 0])[0] == flide.ERR_INVALID  # not monotone
    assert _call(1, [0, 2], [0, 0])[0] == flide.ERR_INVALID      # root with a parent
    assert _call(1, [0, 3], [-1, 0, 2])[0] == flide.ERR_INVALID  # parent not before the node
    assert _call(1, [0, 2], [-1, -1])[0] == flide.ERR_INVALID    # second root
