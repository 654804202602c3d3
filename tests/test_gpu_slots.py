"""Node-state slots reused across tree levels: an inner node's state is read
only by the next level's launch, so inner nodes of depths L and L+2 share a
region.  The device count equals the host formula (flide.state_slots), and the
GDN fork scan with node_state sized to exactly that count matches the oracle
on deep trees (fewer slots than one per inner node)."""
import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import assert_close, build, oracle_gdn, run_gdn

pytestmark = pytest.mark.gpu


def _deep_chain(depth, seg=5):
    # each inner node has a leaf child and an inner child, down to `depth`
    nodes = [(-1, 40)]
    cur = 0
    for _ in range(depth):
        nodes.append((cur, seg))      # leaf option at this depth
        nodes.append((cur, seg + 2))  # continuing node
        cur = len(nodes) - 1
    return nodes


TREES = {
    "chains_depth6": lambda: inputs._tree([(0, _deep_chain(6)), (7, _deep_chain(5, 3))], 6),
    "leveled_depth4_5": lambda: inputs.leveled_tree(np.random.default_rng(6), 3, depth_range=(4, 5),
                                                    options_range=(3, 6), prefix_range=(60, 200),
                                                    branch_range=(3, 20), n_resume=1),
    "depth8_chain": lambda: inputs._tree([(3, [(-1, 17)] + [(i, 5 + i) for i in range(8)])], 8),
}


def _inner_count(tree):
    rp = tree.req_node_ptr
    inner = set()
    for r in range(tree.R):
        for n in range(rp[r] + 1, rp[r + 1]):
            inner.add(rp[r] + tree.parent[n])
    roots = {int(rp[r]) for r in range(tree.R) if rp[r + 1] > rp[r]}
    return len(inner | roots)


@pytest.mark.parametrize("flags", [0, flide.FLAG_PORTABLE], ids=["tc", "portable"])
@pytest.mark.parametrize("case", sorted(TREES))
def test_compact_slots_match_oracle(case, flags):
    tree = TREES[case]()
    _, idx = build(tree)
    torch.cuda.synchronize()
    slots = idx.counts()["SLOTS"]
    assert slots == flide.state_slots(tree)
    assert slots < _inner_count(tree)  # levels really share slots
    g = inputs.gdn_inputs(tree, 2, 128, 128, torch.bfloat16, np.random.default_rng(2), gate_scale=0.1)
    got, _, _ = run_gdn(tree, g, n_slots=slots, flags=flags)
    assert_close(got, oracle_gdn(tree, g), torch.bfloat16)
