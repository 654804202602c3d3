"""Memory-bounded GDN schedule (schedule.fork_gdn_bounded): roots first, then
groups of whole level-1 subtrees resumed from the roots' kept states, each
group within a node-state slot budget.  Fork = isolation makes every output
row and every root end state equal to the one-shot flide_fork_gdn's.  The
roots run exactly as in the one-shot call, so their end states must match bit
for bit; a group may pack sibling leaves into one chunk differently (leaves
that were not adjacent in the full stream can be adjacent in a group's), which
moves the rounding, so the outputs are held to the bf16 bar against both the
oracle and the one-shot result."""
import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import flide, inputs
from tree_forked_decision_b200.schedule import fork_gdn_bounded, plan_state_groups

from gpu_helpers import assert_close, oracle_gdn, run_gdn

pytestmark = pytest.mark.gpu

CASES = {
    "leveled_depth3": lambda rng: inputs.leveled_tree(rng, 4, depth_range=(2, 3), options_range=(6, 40),
                                                      prefix_range=(60, 300), branch_range=(2, 30),
                                                      n_resume=2),
    "deep_chains": lambda rng: inputs._tree([(0, [(-1, 70)] + [(i, 9) for i in range(6)]),
                                             (5, [(-1, 20), (0, 3), (0, 66), (1, 4), (2, 8), (2, 1)])], 6),
    "wide_depth2": lambda rng: inputs._tree([(0, [(-1, 130)] + [(0, 5)] * 12 +
                                                  [(1 + (i % 12), 3 + i % 7) for i in range(48)])], 2),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_bounded_equals_one_shot(case):
    rng = np.random.default_rng(17)
    tree = CASES[case](rng)
    g = inputs.gdn_inputs(tree, 2, 128, 128, torch.bfloat16, rng, gate_scale=0.1)
    want, node_state, _ = run_gdn(tree, g)
    has_state = bool(np.any(tree.past_len > 0))
    dev = {k: v.cuda() for k, v in g.items() if isinstance(v, torch.Tensor)}
    roots = [r for r in range(tree.R) if tree.req_node_ptr[r + 1] > tree.req_node_ptr[r]]
    full = flide.state_slots(tree)
    budgets = sorted({full, max(3, full // 2), 4})
    want_oracle = oracle_gdn(tree, g)
    for budget in budgets:
        try:
            _, ng = plan_state_groups(tree, budget)
        except flide.FlideError:
            continue  # a single subtree needs more than this budget
        out, root_state = fork_gdn_bounded(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], tree,
                                           budget, state_in=dev["state_in"] if has_state else None)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert_close(got, want, torch.bfloat16)
        for i, r in enumerate(roots):
            assert torch.equal(root_state[r], node_state[i]), (case, budget, r)
        assert_close(got, want_oracle, torch.bfloat16)


def test_bounded_runs_where_the_budget_is_far_below_one_shot():
    rng = np.random.default_rng(5)
    tree = inputs.leveled_tree(rng, 6, depth_range=(2, 2), options_range=(100, 200), prefix_range=(30, 90),
                               branch_range=(2, 12))
    full = flide.state_slots(tree)
    budget = 4
    _, ng = plan_state_groups(tree, budget)
    assert full > 4 * budget and ng > 3
    g = inputs.gdn_inputs(tree, 2, 128, 128, torch.bfloat16, rng, gate_scale=0.1)
    dev = {k: v.cuda() for k, v in g.items() if isinstance(v, torch.Tensor)}
    out, _ = fork_gdn_bounded(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], tree, budget)
    torch.cuda.synchronize()
    assert_close(out.float().cpu().numpy(), oracle_gdn(tree, g), torch.bfloat16)
