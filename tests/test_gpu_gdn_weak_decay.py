"""GDN precision under weak decay.

With gate_scale 0.01 the gates are alpha = exp(-0.01 softplus(x)), about
0.993: the state forgets slowly, so its magnitude and the rounding of its bf16
operand copies accumulate over the longest stretch.  The chunked tensor-core
scan must still match the token-by-token fp64 oracle at the bf16 bar on every
token of the sampled (request, head) pairs, over a 32K-token prefix and over a
two-level tree, and its saved end states must match the oracle's (kongchang.com
article on Flide, "ForkAttention" section: forked execution equals isolated
execution in exact arithmetic; Gated DeltaNet box)."""
import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import inputs

from gpu_helpers import assert_close, oracle_gdn, run_gdn

pytestmark = pytest.mark.gpu


def _tree(case):
    if case == "prefix_32k":
        return inputs.fanout_tree(2, 32768, 16, 8)
    rng = np.random.default_rng(31)
    return inputs.leveled_tree(rng, 3, depth_range=(2, 2), options_range=(8, 40),
                               prefix_range=(4000, 8000), n_resume=1)


@pytest.mark.parametrize("case", ["prefix_32k", "two_level"])
def test_gdn_weak_decay_matches_oracle(case):
    tree = _tree(case)
    H = 4
    rng = np.random.default_rng(41)
    g = inputs.gdn_inputs(tree, H, 128, 128, torch.bfloat16, rng, gate_scale=0.01)
    got, node_state, idx = run_gdn(tree, g)
    sel = np.random.default_rng(43).choice(tree.R * H, size=4, replace=False)
    pairs = [(int(i // H), int(i % H)) for i in sel]
    want, states = oracle_gdn(tree, g, pairs=pairs, want_states=True)
    starts = np.concatenate([[0], np.cumsum(tree.seg_len)])
    rp = tree.req_node_ptr
    slot = idx.array("state_slot", tree.N).cpu().numpy()
    ns = node_state.cpu().numpy()
    for r, h in pairs:
        toks = np.arange(starts[rp[r]], starts[rp[r + 1]])
        assert_close(got[toks, h], want[toks, h], torch.bfloat16)
        for n in range(rp[r], rp[r + 1]):
            if slot[n] >= 0:  # roots and depth-1 inner nodes: not reused at depth <= 2
                err = float(np.abs(ns[slot[n], h] - states[n, h]).max())
                assert err <= 2e-2, (n, h, err)
