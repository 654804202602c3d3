"""The named synthetic workloads have the shapes their descriptions state
(requests, prefix, options, branch lengths, heads, dtype), the mixed batch
follows its level recipe (depth 1-3, 2-256 leaves, prefix 256-8192, branches
4-64, 16 of 32 requests resumed with the checkpointed prefix as past), and
the same seed gives the same batch."""
import math

import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import inputs

FANOUT = {
    # name: (R, prefix, branches, branch_len, attention heads (Hq, Hkv, d) or None,
    #        GDN heads (H, dk, dv) or None, dtype)
    "tiny_fp32": (1, 64, 4, 8, (4, 4, 64), (4, 64, 64), torch.float32),
    "attn_fanout_bf16": (8, 2048, 16, 32, (16, 4, 128), None, torch.bfloat16),
    "gdn_fanout_bf16": (8, 4096, 64, 16, None, (16, 128, 128), torch.bfloat16),
    "large_fanout_bf16": (4, 32768, 256, 8, (32, 8, 128), (32, 128, 128), torch.bfloat16),
    "attn_longprefix_bf16": (1, 32768, 256, 8, (4, 1, 128), None, torch.bfloat16),
    "large_fanout_req_bf16": (1, 32768, 256, 8, (32, 8, 128), (32, 128, 128), torch.bfloat16),
}


@pytest.mark.parametrize("name", sorted(FANOUT))
def test_fanout_workloads_match_their_description(name):
    R, prefix, B, L, attn, gdn, dtype = FANOUT[name]
    tree, a, g, dt, _ = inputs.workload(name)
    assert dt == dtype and tree.R == R and tree.levels == 1
    assert tree.N == R * (1 + B) and tree.T == R * (prefix + B * L) and tree.P_past == 0
    rp, parent, seg, past = tree.arrays()
    for r in range(R):
        nodes = range(rp[r], rp[r + 1])
        assert [int(parent[n]) for n in nodes] == [-1] + [0] * B
        assert [int(seg[n]) for n in nodes] == [prefix] + [L] * B
    assert tree.branch_tokens == R * B * L
    assert (a is None) == (attn is None) and (g is None) == (gdn is None)
    if attn:
        assert (a["Hq"], a["Hkv"], a["d"]) == attn
    if gdn:
        assert (g["H"], g["dk"], g["dv"]) == gdn
    assert inputs.WORKLOADS[name]["desc"]


def test_mixed_hybrid_follows_its_recipe():
    tree, a, g, dt, _ = inputs.workload("mixed_hybrid_bf16")
    assert tree.R == 32 and dt == torch.bfloat16 and 1 <= tree.levels <= 3
    assert (a["Hq"], a["Hkv"], a["d"]) == (16, 4, 128) and (g["H"], g["dk"], g["dv"]) == (16, 128, 128)
    rp, parent, seg, past = tree.arrays()
    resumed = 0
    for r in range(tree.R):
        nodes = list(range(rp[r], rp[r + 1]))
        depth = {nodes[0]: 0}
        for n in nodes[1:]:
            depth[n] = depth[rp[r] + parent[n]] + 1
        D = max(depth.values())
        assert 1 <= D <= 3
        sizes = [sum(1 for n in nodes if depth[n] == k) for k in range(D + 1)]
        O = sizes[-1]
        assert 2 <= O <= 256
        assert sizes == [1] + [math.ceil(O ** (k / D)) for k in range(1, D)] + [O]
        leaves = [n for n in nodes if depth[n] == D]
        assert all(not any(rp[r] + parent[m] == n for m in nodes[1:]) for n in leaves)
        assert all(4 <= seg[n] <= 64 for n in nodes[1:])
        P = int(past[r]) + int(seg[nodes[0]])                # the whole prefix
        assert 256 <= P <= 8192
        if past[r] > 0:
            resumed += 1
            assert 4 <= seg[nodes[0]] <= 64                  # the root keeps delta tokens
    assert resumed == 16


def test_same_seed_same_batch():
    t1, *_ = inputs.workload("mixed_hybrid_bf16")
    t2, *_ = inputs.workload("mixed_hybrid_bf16")
    t3, *_ = inputs.workload("mixed_hybrid_bf16", seed=99)
    assert all(np.array_equal(x, y) for x, y in zip(t1.arrays(), t2.arrays()))
    assert t1.T != t3.T or not all(np.array_equal(x, y) for x, y in zip(t1.arrays(), t3.arrays()))
    (_, a1, g1, _), (_, a2, g2, _) = inputs.make_inputs("tiny_fp32"), inputs.make_inputs("tiny_fp32")
    for key in ("q", "k", "v"):
        assert torch.equal(a1[key], a2[key]) and torch.equal(g1[key], g2[key])
    assert torch.equal(g1["g"], g2["g"]) and torch.equal(g1["beta"], g2["beta"])
