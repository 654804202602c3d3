"""Pins for the decision-scoring oracle (oracle/decision.py) against things other
than itself: a pure-Python brute force, closed forms and symmetries, and the
total-variation definition's own special cases (kongchang.com article on
Flide, "total variation distance" box)."""
import math

import numpy as np

import oracle
from tree_forked_decision_b200 import inputs


def _tiny():
    # request 0: root 3 tokens, options: a leaf of 2 tokens, and a node of 1
    # token with two leaf children (2 and 1 tokens); request 1: root only;
    # request 2: root 2 tokens, one leaf of 3 tokens
    return inputs._tree([(0, [(-1, 3), (0, 2), (0, 1), (2, 2), (2, 1)]),
                         (4, [(-1, 5)]),
                         (0, [(-1, 2), (0, 3)])], 2)


def test_branch_logprob_matches_brute_force_loops():
    t = _tiny()
    rng = np.random.default_rng(0)
    V, D = 5, 3
    h = rng.standard_normal((t.T, D))
    w = rng.standard_normal((V, D))
    y = rng.integers(0, V, t.T)
    got = oracle.branch_logprob(t.arrays(), h, w, y)
    starts = np.concatenate([[0], np.cumsum(t.seg_len)])
    rp = t.req_node_ptr
    branch_tokens = set()
    for r in range(t.R):
        for n in range(rp[r] + 1, rp[r + 1]):
            branch_tokens.update(range(starts[n], starts[n + 1]))
    for tok in range(t.T):
        if tok not in branch_tokens:
            assert math.isnan(got[tok])
            continue
        logits = [sum(h[tok][d] * w[v][d] for d in range(D)) for v in range(V)]
        lse = math.log(sum(math.exp(z) for z in logits))
        assert abs(got[tok] - (logits[y[tok]] - lse)) < 1e-12


def test_zero_head_gives_length_closed_form():
    # W = 0: every branch token has log p = -log V, so an option of L tokens
    # scores -L log V and the leaves' softmax is a closed form in the lengths
    t = _tiny()
    V = 7
    logp = oracle.branch_logprob(t.arrays(), np.ones((t.T, 4)), np.zeros((V, 4)), np.zeros(t.T, int))
    path, prob = oracle.option_probs(t.arrays(), logp)
    # request 0 leaves: node 1 (2 tokens), node 3 (1 + 2), node 4 (1 + 1)
    lens = np.array([2, 3, 2])
    e = np.exp(-lens * math.log(V))
    assert np.allclose(prob[[1, 3, 4]], e / e.sum(), rtol=0, atol=1e-15)
    assert np.allclose(path[[1, 2, 3, 4]], -np.array([2, 1, 3, 2]) * math.log(V), atol=1e-12)
    assert prob[0] == prob[2] == 0.0  # root and inner node carry no mass
    assert prob[5] == 0.0             # request with a root only
    assert prob[7] == 1.0             # request with a single option


def test_path_sums_by_hand():
    t = _tiny()
    logp = np.full(t.T, np.nan)
    starts = np.concatenate([[0], np.cumsum(t.seg_len)])
    vals = {1: [-0.5, -1.0], 2: [-0.25], 3: [-2.0, -0.125], 4: [-3.0], 7: [-1.0, -1.0, -1.0]}
    for n, v in vals.items():
        logp[starts[n]:starts[n + 1]] = v
    path, prob = oracle.option_probs(t.arrays(), logp)
    assert path[1] == -1.5 and path[2] == -0.25
    assert path[3] == -0.25 - 2.125 and path[4] == -0.25 - 3.0 and path[7] == -3.0
    s = np.array([-1.5, -2.375, -3.25])
    e = np.exp(s - s.max())
    assert np.allclose(prob[[1, 3, 4]], e / e.sum(), atol=1e-15)


def test_identical_options_split_evenly():
    t = inputs.fanout_tree(1, 4, 2, 3)
    rng = np.random.default_rng(1)
    h = rng.standard_normal((t.T, 6))
    h[7:10] = h[4:7]  # second option repeats the first one's hidden states
    y = rng.integers(0, 11, t.T)
    y[7:10] = y[4:7]
    logp = oracle.branch_logprob(t.arrays(), h, rng.standard_normal((11, 6)), y)
    _, prob = oracle.option_probs(t.arrays(), logp)
    assert abs(prob[1] - 0.5) < 1e-15 and abs(prob[2] - 0.5) < 1e-15


def test_tvd_special_cases():
    t = inputs.fanout_tree(2, 1, 3, 1)
    p = np.zeros(t.N)
    q = np.zeros(t.N)
    p[[1, 5]] = 1.0        # request 0: all mass on option 1; request 1: on its option 1
    q[[2, 6]] = 1.0        # disjoint supports
    assert np.allclose(oracle.tvd(t.arrays(), p, q), [1.0, 1.0])
    assert np.allclose(oracle.tvd(t.arrays(), p, p), [0.0, 0.0])
    q = np.zeros(t.N)
    q[[1, 2]] = 0.5
    q[[5, 6, 7]] = 1.0 / 3
    assert np.allclose(oracle.tvd(t.arrays(), p, q), [0.5, 2.0 / 3])


def test_tvd_equals_largest_event_difference():
    """TVD is also the largest |P(A) - Q(A)| over events A: checked by
    enumerating every subset of a request's leaves."""
    import itertools
    t = inputs._tree([(0, [(-1, 2), (0, 1), (0, 1), (0, 1), (0, 1)])], 1)
    rng = np.random.default_rng(5)
    for _ in range(20):
        p, q = np.zeros(t.N), np.zeros(t.N)
        p[1:], q[1:] = rng.dirichlet(np.ones(4)), rng.dirichlet(np.ones(4))
        sup = max(abs(p[list(A)].sum() - q[list(A)].sum())
                  for k in range(5) for A in itertools.combinations(range(1, 5), k))
        assert math.isclose(oracle.tvd(t.arrays(), p, q)[0], sup, rel_tol=1e-12, abs_tol=1e-15)
