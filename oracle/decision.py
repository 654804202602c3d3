"""Decision scoring oracle (fp64, numpy) -- TEST INFRASTRUCTURE ONLY.

Decision models answer with probabilities over a small set of candidate
options rather than with generated text (openai-hub.com news article on the
Flide release, paragraphs on Jev-like decision models), and the engines are compared by the total variation
distance of those probabilities to a high-precision reference (kongchang.com
article on Flide, "total variation distance" box: half the sum of absolute
differences over the outcomes, in [0, 1]).

Reading used here (the pages do not spell the scoring head out): every leaf of
a request's tree is one option; its score is the log-likelihood of the
option's tokens, the sum over the branch tokens on its path (non-root nodes
from the root's child to the leaf) of log p(target | hidden state) under an LM
head W (vocabulary x hidden); the decision distribution is the softmax of the
scores over the request's leaves.  Root tokens are the shared context and are
not scored.

Every function here is the plain definition in double precision; pins in
``tests/test_decision_oracle.py``.
"""
from __future__ import annotations

import numpy as np


def _structure(tree):
    """Per node: request, parent (global id or -1), token range; per request
    the node range (from the tree's four arrays)."""
    rp, parent, seg, _past = (np.asarray(a) for a in tree)
    R, N = len(rp) - 1, len(parent)
    starts = np.concatenate([[0], np.cumsum(seg)]).astype(np.int64)
    req = np.zeros(N, np.int64)
    gpar = np.full(N, -1, np.int64)
    for r in range(R):
        for n in range(rp[r], rp[r + 1]):
            req[n] = r
            gpar[n] = -1 if parent[n] < 0 else rp[r] + parent[n]
    has_child = np.zeros(N, bool)
    has_child[gpar[gpar >= 0]] = True
    return rp, gpar, starts, req, has_child


def branch_logprob(tree, h, w, targets):
    """log p(targets[t] | h[t]) = logit[t, y] - logsumexp_v logit[t, v] with
    logit = h W^T, for every branch token t (tokens of non-root nodes); root
    tokens get NaN.  h [T, D], w [V, D], targets [T] (int)."""
    rp, gpar, starts, _req, _hc = _structure(tree)
    h = np.asarray(h, np.float64)
    w = np.asarray(w, np.float64)
    T = h.shape[0]
    out = np.full(T, np.nan)
    branch = np.zeros(T, bool)
    for n in range(len(gpar)):
        if gpar[n] >= 0:
            branch[starts[n]:starts[n + 1]] = True
    rows = np.nonzero(branch)[0]
    if len(rows):
        logits = h[rows] @ w.T
        m = logits.max(axis=1, keepdims=True)
        lse = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
        out[rows] = logits[np.arange(len(rows)), np.asarray(targets)[rows]] - lse
    return out


def option_probs(tree, logp):
    """Per node: path log-likelihood (sum of branch-token log-probs from the
    root's child down to the node; 0 for roots) and, for leaves, the softmax of
    the leaves' path scores within their request (0 for other nodes)."""
    rp, gpar, starts, req, has_child = _structure(tree)
    N = len(gpar)
    path = np.zeros(N)
    for n in range(N):  # parents precede children inside a request
        if gpar[n] >= 0:
            path[n] = path[gpar[n]] + float(np.sum(logp[starts[n]:starts[n + 1]]))
    prob = np.zeros(N)
    for r in range(len(rp) - 1):
        leaves = [n for n in range(rp[r], rp[r + 1]) if gpar[n] >= 0 and not has_child[n]]
        if not leaves:
            continue
        s = path[leaves]
        e = np.exp(s - s.max())
        prob[leaves] = e / e.sum()
    return path, prob


def tvd(tree, p, q):
    """Total variation distance per request between two leaf distributions
    given per node (only leaves carry mass): 0.5 * sum |p - q|."""
    rp = np.asarray(tree[0])
    return np.array([0.5 * float(np.sum(np.abs(np.asarray(p)[rp[r]:rp[r + 1]]
                                                - np.asarray(q)[rp[r]:rp[r + 1]])))
                     for r in range(len(rp) - 1)])
