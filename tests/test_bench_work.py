"""The algorithmic work bench.py divides by (host only): the visible-key count
behind the attention FLOPs, the attention bytes, and the GDN bytes (inputs and
outputs once, one fp32 state write per saved node, one state read per node
whose children continue from it and per resumed root).  Pinned by closed forms
on fan-out trees and by walking every token's isolated sequence on random
trees."""
import numpy as np
import pytest
import torch

import bench
from tree_forked_decision_b200 import inputs


def _spec_attn(d, Hq, Hkv, dtype):
    return dict(d=d, Hq=Hq, Hkv=Hkv, q=torch.empty(0, dtype=dtype))


def _spec_gdn(H, dk, dv, dtype):
    return dict(H=H, dk=dk, dv=dv, q=torch.empty(0, dtype=dtype))


@pytest.mark.parametrize("R,prefix,B,L,past", [(1, 5, 3, 2, 0), (4, 64, 16, 8, 7), (3, 1, 1, 1, 100)])
def test_fanout_closed_forms(R, prefix, B, L, past):
    tree = inputs.fanout_tree(R, prefix, B, L, past=past)
    # token i of the root sees past + i + 1 keys; token j of a branch sees
    # past + prefix + j + 1
    vis = R * (prefix * past + prefix * (prefix + 1) // 2
               + B * (L * (past + prefix) + L * (L + 1) // 2))
    assert int((bench.isolated_positions(tree) + 1).sum()) == vis
    d, Hq, Hkv = 16, 8, 2
    flops, byts = bench.attn_work(tree, _spec_attn(d, Hq, Hkv, torch.bfloat16))
    T = R * (prefix + B * L)
    assert flops == 4.0 * d * Hq * vis
    assert byts == 2 * d * (2 * T * Hq + 2 * T * Hkv + 2 * R * past * Hkv)
    assert bench.attn_work(tree, _spec_attn(d, Hq, Hkv, torch.float32))[1] == 2 * byts
    H, dk, dv = 4, 16, 32
    state = 4 * H * dk * dv
    # every root has children: R writes, R reads by the branches, R more
    # reads of the resumed states when past > 0
    n_state = R + R + (R if past else 0)
    g16 = _spec_gdn(H, dk, dv, torch.bfloat16)
    assert bench.gdn_work(tree, g16) == T * H * ((2 * dk + 2 * dv) * 2 + 8) + n_state * state
    # e4m3 q, k, v (1 byte) with a bf16 output
    assert bench.gdn_work(tree, g16, esize=1) == T * H * ((2 * dk + dv) + 2 * dv + 8) + n_state * state
    g32 = _spec_gdn(H, dk, dv, torch.float32)
    assert bench.gdn_work(tree, g32) == T * H * ((2 * dk + 2 * dv) * 4 + 8) + n_state * state


def test_roots_without_branches():
    """A request that is only a root still writes its end state (the next
    step resumes from it) and reads nothing unless it was resumed."""
    tree = inputs._tree([(0, [(-1, 9)]), (3, [(-1, 4)]), (0, [])], 0)
    H, dk, dv = 2, 8, 8
    state = 4 * H * dk * dv
    io = tree.T * H * ((2 * dk + 2 * dv) * 4 + 8)
    assert bench.gdn_work(tree, _spec_gdn(H, dk, dv, torch.float32)) == io + (2 + 1) * state


def _walk_visible(tree):
    """Keys visible to each stream token, from its explicit key list: the
    request's past rows, every token of every proper ancestor (walking parent
    links), and its own node's tokens up to and including itself."""
    rp, pa, sl, pl = tree.arrays()
    starts = np.concatenate([[0], np.cumsum(sl)])
    out = np.zeros(tree.T, np.int64)
    for r in range(tree.R):
        for n in range(rp[r], rp[r + 1]):
            anc = []
            a = int(pa[n])
            while a >= 0:
                anc.append(int(rp[r]) + a)
                a = int(pa[rp[r] + a])
            keys = int(pl[r]) + sum(int(sl[m]) for m in anc)
            for j in range(int(sl[n])):
                out[starts[n] + j] = keys + j + 1
    return out


def _brute_gdn_states(tree):
    """(writes, reads) counted per node from its child list."""
    rp, pa, sl, pl = tree.arrays()
    writes = reads = 0
    for r in range(tree.R):
        nodes = range(rp[r], rp[r + 1])
        for n in nodes:
            kids = [m for m in nodes if pa[m] >= 0 and rp[r] + pa[m] == n]
            root = pa[n] < 0
            writes += 1 if (root or kids) else 0
            reads += 1 if kids else 0
            reads += 1 if (root and pl[r] > 0) else 0
    return writes, reads


@pytest.mark.parametrize("seed", range(6))
def test_random_trees_against_walks(seed):
    rng = np.random.default_rng(100 + seed)
    tree = inputs.random_tree(rng, R=5, max_nodes=9, prefix_range=(0, 30), branch_range=(1, 7))
    vis = _walk_visible(tree)
    assert np.array_equal(bench.isolated_positions(tree) + 1, vis)
    flops, _ = bench.attn_work(tree, _spec_attn(32, 4, 1, torch.bfloat16))
    assert flops == 4.0 * 32 * 4 * vis.sum()
    w, r = _brute_gdn_states(tree)
    H, dk, dv = 3, 8, 16
    got = bench.gdn_work(tree, _spec_gdn(H, dk, dv, torch.bfloat16))
    assert got == tree.T * H * ((2 * dk + 2 * dv) * 2 + 8) + (w + r) * 4 * H * dk * dv
