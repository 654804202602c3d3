"""The native planner of the memory-bounded GDN schedule
(flide_plan_state_groups), host only: every non-root node gets the group of
its level-1 ancestor, groups follow stream order, each group's batch (per
request a zero-token root plus the group's subtrees) needs at most the budget
of node-state slots by the slot rule flide_tree_build applies, packing is
greedy (the next group's first subtree would not have fitted), and a subtree
that alone exceeds the budget, or a malformed tree, is refused; the Python
side's batches cover every token row once."""
import numpy as np
import pytest

from tree_forked_decision_b200 import flide, inputs
from tree_forked_decision_b200.schedule import plan_state_groups


def _level1(tree):
    rp, parent, _, _ = tree.arrays()
    top = {}
    for r in range(tree.R):
        for n in range(rp[r] + 1, rp[r + 1]):
            p = int(rp[r] + parent[n])
            top[n] = n if p == rp[r] else top[p]
    return top


def _group_tree(tree, members):
    """Sub-batch of the given non-root nodes (whole subtrees, stream order)."""
    rp, parent, seg, _ = tree.arrays()
    reqs, cur, local = [], -1, {}
    for n in members:
        r = int(np.searchsorted(rp, n, side="right") - 1)
        if r != cur:
            reqs.append((0, [(-1, 0)]))
            cur, local = r, {int(rp[r]): 0}
        local[n] = len(reqs[-1][1])
        reqs[-1][1].append((local[int(rp[r] + parent[n])], int(seg[n])))
    return inputs._tree(reqs, 8)


TREES = {
    "leveled": lambda rng: inputs.leveled_tree(rng, 6, depth_range=(1, 3), options_range=(2, 60),
                                               prefix_range=(10, 50), branch_range=(1, 9)),
    "random": lambda rng: inputs.random_tree(rng, R=7, max_nodes=14, prefix_range=(0, 20),
                                             branch_range=(1, 9)),
    "deep_chains": lambda rng: inputs._tree([(0, [(-1, 3)] + [(i, 2) for i in range(6)]),
                                             (0, [(-1, 1), (0, 1), (0, 1), (1, 1), (2, 1)])], 6),
}


@pytest.mark.parametrize("case", sorted(TREES))
@pytest.mark.parametrize("seed", range(4))
def test_groups_fit_the_budget_and_are_greedy(case, seed):
    rng = np.random.default_rng(seed)
    tree = TREES[case](rng)
    top = _level1(tree)
    rp = tree.req_node_ptr
    for budget in sorted({2, 3, 5, 9, 40, flide.state_slots(tree) + 1}):
        try:
            grp, ng = plan_state_groups(tree, budget)
        except flide.FlideError as e:
            assert e.code == flide.ERR_CAPACITY
            # some single subtree needs more than the budget
            assert any(flide.state_slots(_group_tree(tree, [m for m in top if top[m] == n])) > budget
                       for n in set(top.values()))
            continue
        roots = {int(rp[r]) for r in range(tree.R) if rp[r + 1] > rp[r]}
        assert all(grp[n] == -1 for n in roots)
        assert all(grp[n] == grp[top[n]] for n in top)           # whole subtrees
        order = [int(grp[n]) for n in sorted(top) if top[n] == n]
        assert order == sorted(order)                            # stream order
        assert set(order) == set(range(ng))
        members = [[n for n in sorted(top) if grp[n] == g] for g in range(ng)]
        for g in range(ng):
            assert flide.state_slots(_group_tree(tree, members[g])) <= budget
            if g + 1 < ng:
                first_next = [n for n in members[g + 1] if top[n] == members[g + 1][0]]
                assert flide.state_slots(_group_tree(tree, members[g] + first_next)) > budget


def test_one_group_when_the_budget_allows():
    tree = inputs.leveled_tree(np.random.default_rng(1), 3, depth_range=(2, 3), options_range=(4, 30),
                               prefix_range=(5, 9), branch_range=(1, 3))
    grp, ng = plan_state_groups(tree, 10 ** 6)
    assert ng == (1 if tree.N > tree.R else 0)


def test_refuses_malformed_trees_and_bad_budgets():
    lib = flide._lib()
    import ctypes
    rp = np.array([0, 3], np.int32)
    bad_parent = np.array([-1, 2, 0], np.int32)  # parent after the child
    out = np.zeros(3, np.int32)
    ng = ctypes.c_int32(0)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    assert lib.flide_plan_state_groups(1, p(rp), p(bad_parent), 4, p(out), ctypes.byref(ng)) == flide.ERR_INVALID
    good = np.array([-1, 0, 0], np.int32)
    assert lib.flide_plan_state_groups(1, p(rp), p(good), 0, p(out), ctypes.byref(ng)) == flide.ERR_SHAPE
    assert lib.flide_plan_state_groups(1, p(rp), p(good), 1, p(out), ctypes.byref(ng)) == flide.OK
    assert ng.value == 1 and out.tolist() == [-1, 0, 0]
    # request tables that are not monotone are refused before anything is sized
    for bad_rp in ([0, -5], [0, 3, 2], [0, 2, -1]):
        t = np.array(bad_rp, np.int32)
        assert lib.flide_plan_state_groups(len(t) - 1, p(t), p(good), 4, p(out), ctypes.byref(ng)) \
            == flide.ERR_INVALID


@pytest.mark.parametrize("case", sorted(TREES))
def test_batches_cover_every_token_row_once(case):
    """schedule._batches (host): root batches hold every request's root rows,
    group batches every other node's rows, each row exactly once; a group's
    batch rebuilds the subtrees with request-local parents (zero-token roots),
    and every batch fits the budget by the index builder's slot rule."""
    from tree_forked_decision_b200.schedule import _batches
    rng = np.random.default_rng(11)
    tree = TREES[case](rng)
    rp, _parent, seg, _ = tree.arrays()
    for budget in (3, 7, 50):
        try:
            batches = _batches(tree, budget)
        except flide.FlideError:
            continue
        seen = np.zeros(tree.T, int)
        for kind, batch, req_ids in batches:
            assert flide.state_slots(batch) <= budget
            brp, bpar, bseg, _ = batch.arrays()
            assert len(req_ids) == len(brp) - 1 and int(bseg.sum()) == len(batch.rows)
            seen[batch.rows] += 1
            if kind == "roots":
                assert all(p == -1 for p in bpar) and len(bpar) == len(req_ids)
                assert list(bseg) == [int(seg[rp[r]]) for r in req_ids]
            else:
                for bi, r in enumerate(req_ids):
                    nodes = range(brp[bi], brp[bi + 1])
                    assert bpar[brp[bi]] == -1 and bseg[brp[bi]] == 0   # zero-token root
                    for n in nodes:
                        if n > brp[bi]:
                            assert 0 <= bpar[n] < n - brp[bi]            # parent precedes
        assert (seen == 1).all()


def test_host_entry_points_survive_random_arguments():
    """Random request tables (monotone or not, negative entries), parents and
    budgets for the planner, and random slots and counts for the history
    pool's appends, in a child process: every call returns a status code and
    the process never aborts (no exception crosses the C ABI)."""
    import subprocess
    import sys
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = r'''
import ctypes, numpy as np
from tree_forked_decision_b200 import flide
lib = flide._lib()
p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
rng = np.random.default_rng(77)
codes = {flide.OK, flide.ERR_INVALID, flide.ERR_SHAPE, flide.ERR_CAPACITY}
for _ in range(3000):
    R = int(rng.integers(0, 6))
    rp = np.cumsum(np.concatenate([[0], rng.integers(-2, 5, R)])).astype(np.int32)
    if rng.random() < 0.2:
        rp[0] = int(rng.integers(-3, 3))
    N = max(int(rp.max()), 0)
    parent = rng.integers(-2, 6, max(N, 1)).astype(np.int32)
    out = np.zeros(max(N, 1), np.int32)
    ng = ctypes.c_int32(0)
    st = lib.flide_plan_state_groups(R, p(rp), p(parent), int(rng.integers(-1, 8)), p(out),
                                     ctypes.byref(ng))
    assert st in codes, st
pool = lib.flide_pool_create(12, 4, 5, 3)
for _ in range(3000):
    k = int(rng.integers(0, 6))
    sl = rng.integers(-2, 7, k).astype(np.int32)
    ct = rng.integers(-3, 20, k).astype(np.int32)
    starts = np.zeros(max(k, 1), np.int32)
    st = lib.flide_pool_append_batch(pool, k, p(sl), p(ct), p(starts))
    assert st in codes, st
    if rng.random() < 0.3:
        lib.flide_pool_release(pool, int(rng.integers(-1, 6)))
    assert 0 <= lib.flide_pool_free_blocks(pool) <= 12
lib.flide_pool_destroy(pool)
print("ok")
'''
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout[-2000:] + r.stderr[-2000:]
