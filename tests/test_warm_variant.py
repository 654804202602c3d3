"""The resumed-prefix (warm) form of a batch that bench.py times: the tree
transform keeps exactly the branch rows, and, run through the oracle with the
root's checkpoint (past + root K/V rows, the root's end state) as past and
state_in, it reproduces the from-scratch outputs of those rows (resume equals
scratch, the exact-state-forking reading)."""
import math

import numpy as np
import torch

import oracle
from tree_forked_decision_b200 import inputs


def _cold_tree():
    # two requests with past rows, a depth-2 tree and an empty request
    return inputs._tree([(5, [(-1, 23), (0, 4), (0, 6), (1, 3)]),
                         (0, []),
                         (9, [(-1, 17), (0, 5), (1, 2), (1, 7)])], 2)


def test_warm_variant_structure():
    t = _cold_tree()
    w, rows = inputs.warm_variant(t)
    assert w.R == t.R and w.N == t.N
    assert w.past_len.tolist() == [5 + 23, 0, 9 + 17]
    assert w.seg_len.tolist() == [0, 4, 6, 3, 0, 5, 2, 7]
    assert w.parent.tolist() == t.parent.tolist()
    assert w.branch_tokens == t.branch_tokens == w.T == len(rows)
    starts = np.concatenate([[0], np.cumsum(t.seg_len)])
    expect = np.concatenate([np.arange(starts[1], starts[4]), np.arange(starts[5], starts[8])])
    assert np.array_equal(rows, expect)


def test_warm_equals_cold_through_the_oracle():
    t = _cold_tree()
    rng = np.random.default_rng(5)
    Hq, Hkv, d, H, dk, dv = 4, 2, 32, 2, 16, 16
    a = inputs.attn_inputs(t, Hq, Hkv, d, torch.float32, rng)
    g = inputs.gdn_inputs(t, H, dk, dv, torch.float32, rng, gate_scale=0.5)
    f = lambda x: x.float().numpy().astype(np.float64)
    scale = 1.0 / math.sqrt(d)
    cold_a = oracle.attention_all(t.arrays(), f(a["q"]), f(a["k"]), f(a["v"]), f(a["past_k"]),
                                  f(a["past_v"]), scale)
    cold_g, states = oracle.gdn(t.arrays(), f(g["q"]), f(g["k"]), f(g["v"]), f(g["g"]),
                                f(g["beta"]), state_in=f(g["state_in"]), want_states=True)
    w, rows = inputs.warm_variant(t)
    # checkpoint: per request its past rows then its root rows; roots' end states
    starts = np.concatenate([[0], np.cumsum(t.seg_len)])
    rp, p0 = t.req_node_ptr, np.concatenate([[0], np.cumsum(t.past_len)])
    ck_k, ck_v, st = [], [], np.zeros((t.R, H, dv, dk))
    for r in range(t.R):
        ck_k.append(f(a["past_k"])[p0[r]:p0[r + 1]])
        ck_v.append(f(a["past_v"])[p0[r]:p0[r + 1]])
        if rp[r + 1] > rp[r]:
            root = rp[r]
            ck_k.append(f(a["k"])[starts[root]:starts[root + 1]])
            ck_v.append(f(a["v"])[starts[root]:starts[root + 1]])
            st[r] = states[root]
    warm_a = oracle.attention_all(w.arrays(), f(a["q"])[rows], f(a["k"])[rows], f(a["v"])[rows],
                                  np.concatenate(ck_k), np.concatenate(ck_v), scale)
    warm_g = oracle.gdn(w.arrays(), f(g["q"])[rows], f(g["k"])[rows], f(g["v"])[rows],
                        f(g["g"])[rows], f(g["beta"])[rows], state_in=st)
    assert np.max(np.abs(warm_a - cold_a[rows])) < 1e-12
    assert np.max(np.abs(warm_g - cold_g[rows])) < 1e-12
