"""Full-size workloads through the C ABI in the launch configuration bench.py
times, checked against the oracle on sampled outputs: attention on a seeded
sample of query rows (first and last root rows of every request, every branch
row of query head 0, every branch row of the last request for all G query
heads of the last kv group -- so the in-group positions 1..G-1 of the 128-row
tile packing are all covered at full size -- plus random rows), GDN on every
token of sampled (request, head) pairs."""
import numpy as np
import pytest

import oracle
from tree_forked_decision_b200 import inputs

from gpu_helpers import assert_close, run_attn, run_gdn

pytestmark = pytest.mark.gpu


def _rows(tree, Hq, Hkv, n_random, rng):
    starts = np.concatenate([[0], np.cumsum(tree.seg_len)])
    rp = tree.req_node_ptr
    rows = []
    G = Hq // Hkv
    last = max(r for r in range(tree.R) if rp[r + 1] > rp[r])
    for t in range(starts[rp[last] + 1], starts[rp[last + 1]]):  # all heads of kv group Hkv - 1
        rows += [(t, h) for h in range(Hq - G, Hq)]
    for r in range(tree.R):
        if rp[r + 1] == rp[r]:
            continue
        rs, re, end = starts[rp[r]], starts[rp[r] + 1], starts[rp[r + 1]]
        for t in list(range(rs, min(rs + 4, re))) + list(range(max(rs, re - 4), re)):
            rows.append((t, int(rng.integers(0, Hq))))
        rows += [(t, 0) for t in range(re, end)]  # every branch row of head 0
    pick = rng.integers(0, tree.T * Hq, size=n_random)
    rows += [(int(i // Hq), int(i % Hq)) for i in pick]
    return np.unique(np.asarray(rows, np.int32), axis=0)


@pytest.mark.parametrize("name", ["attn_fanout_bf16", "mixed_hybrid_bf16", "large_fanout_bf16"])
def test_fullsize_attention_sampled(name):
    tree, a, _, dtype = inputs.make_inputs(name)
    got, scale = run_attn(tree, a)
    rng = np.random.default_rng(1)
    rows = _rows(tree, a["Hq"], a["Hkv"], 1500, rng)
    f = lambda t: t.float().numpy()
    want = oracle.attention_rows(tree.arrays(), f(a["q"]), f(a["k"]), f(a["v"]),
                                 f(a["past_k"]), f(a["past_v"]), scale, rows)
    assert np.all(np.isfinite(got))
    assert_close(got[rows[:, 0], rows[:, 1]], want, dtype)


@pytest.mark.parametrize("name,n_pairs", [("gdn_fanout_bf16", 6), ("mixed_hybrid_bf16", 6),
                                          ("large_fanout_bf16", 4)])
def test_fullsize_gdn_sampled(name, n_pairs):
    tree, _, g, dtype = inputs.make_inputs(name)
    got, _, _ = run_gdn(tree, g)
    rng = np.random.default_rng(2)
    H = g["H"]
    sel = rng.choice(tree.R * H, size=n_pairs, replace=False)
    heads = sorted({int(i % H) for i in sel})
    pairs = [(int(i // H), heads.index(int(i % H))) for i in sel]
    hs = lambda t: np.ascontiguousarray(t.float().numpy()[:, heads])
    has_state = bool(np.any(tree.past_len > 0))
    want = oracle.gdn(tree.arrays(), hs(g["q"]), hs(g["k"]), hs(g["v"]), hs(g["g"]),
                      hs(g["beta"]), state_in=hs(g["state_in"]) if has_state else None,
                      pairs=pairs)
    starts = np.concatenate([[0], np.cumsum(tree.seg_len)])
    rp = tree.req_node_ptr
    for (r, hi) in pairs:
        toks = np.arange(starts[rp[r]], starts[rp[r + 1]])
        assert_close(got[toks, heads[hi]], want[toks, hi], dtype)
