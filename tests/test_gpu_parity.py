"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Indices bit-exact; fp32 outputs within 1e-4 max-abs;
bf16 outputs within 2e-2 max-abs and 1e-2 relative L2."""
import json
import os
import zlib

import numpy as np
import pytest
import torch

import oracle
from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import (assert_close, build, oracle_attn, oracle_gdn, run_attn,
                         run_gdn)

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden")
INDEX_KEYS = ["node_start", "token_node", "token_pos", "depth", "anc_ptr", "anc_node", "ctx_len"]


def _gpu_index(tree, idx):
    N, T = tree.N, tree.T
    c = idx.counts()
    anc_len = int(idx.array("anc_ptr", N + 1)[-1].item())
    sizes = dict(node_start=N + 1, token_node=T, token_pos=T, depth=N, anc_ptr=N + 1,
                 anc_node=anc_len, ctx_len=N)
    return {k: idx.array(k, n).cpu().numpy() for k, n in sizes.items()}, c


def _check_index(tree):
    _, idx = build(tree)
    assert idx.status() == 0
    got, counts = _gpu_index(tree, idx)
    want = oracle.tree_index(*tree.arrays())
    for k in INDEX_KEYS:
        assert np.array_equal(got[k], want[k]), k
    assert counts["N"] == tree.N and counts["T"] == tree.T
    assert counts["BRANCH_TOK"] == tree.branch_tokens
    return idx


# ---------------------------------------------------------------------------
# tree index
# ---------------------------------------------------------------------------

def test_tree_build_golden():
    g = json.load(open(os.path.join(GOLD, "tree_index_small.json")))
    tree = inputs._tree([(g["past_len"][0], list(zip(g["parent"][:4], g["seg_len"][:4]))),
                         (g["past_len"][1], list(zip(g["parent"][4:], g["seg_len"][4:])))], 2)
    _, idx = build(tree)
    got, _ = _gpu_index(tree, idx)
    for k, want in g["expect"].items():
        assert got[k].tolist() == want, k


@pytest.mark.parametrize("seed", range(5))
def test_tree_build_random(seed):
    rng = np.random.default_rng(500 + seed)
    _check_index(inputs.random_tree(rng, R=7, max_nodes=12, prefix_range=(0, 30),
                                    branch_range=(1, 9), past_range=(0, 20)))


def test_tree_build_leveled_full_size():
    # the mixed-batch generator at full size (32 requests, depth 1-3, 2-256 options)
    tree, *_ = inputs.workload("mixed_hybrid_bf16")
    idx = _check_index(tree)
    lv = idx.array("level_ptr", tree.levels + 2).cpu().numpy()
    depth = idx.array("depth", tree.N).cpu().numpy()
    nodes = idx.array("level_node", tree.N).cpu().numpy()
    for lvl in range(tree.levels + 1):
        sel = nodes[lv[lvl]:lv[lvl + 1]]
        assert np.array_equal(sel, np.flatnonzero(depth == lvl))


@pytest.mark.parametrize("bad", ["parent_ge_self", "root_parent", "empty_branch"])
def test_tree_build_rejects_malformed(bad):
    rp, pa, sl, pl = [0, 3], [-1, 0, 1], [2, 1, 1], [0]
    if bad == "parent_ge_self":
        pa = [-1, 1, 1]
    elif bad == "root_parent":
        pa = [0, 0, 1]
    elif bad == "empty_branch":
        sl = [2, 0, 1]
    dt = flide.DeviceTree(rp, pa, sl, pl, max_depth=2)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, dt.max_depth)
    flide.tree_build(dt, idx)
    torch.cuda.synchronize()
    assert idx.status() == flide.ERR_INVALID


def test_tree_build_depth_capacity():
    tree = inputs._tree([(0, [(-1, 3), (0, 2), (1, 2), (2, 2)])], 3)
    dt = flide.DeviceTree(*tree.arrays(), max_depth=2)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, 2)
    flide.tree_build(dt, idx)
    torch.cuda.synchronize()
    assert idx.status() == flide.ERR_CAPACITY


def test_tree_build_padding_requests():
    # empty trailing requests act as padding inside larger capacities
    tree = inputs.fanout_tree(2, 5, 3, 2)
    rp = np.concatenate([tree.req_node_ptr, [tree.N, tree.N]]).astype(np.int32)
    pl = np.concatenate([tree.past_len, [0, 0]]).astype(np.int32)
    dt = flide.DeviceTree(rp, tree.parent, tree.seg_len, pl, max_depth=3, N=tree.N + 10,
                          T=tree.T + 50)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, 3)
    flide.tree_build(dt, idx)
    torch.cuda.synchronize()
    assert idx.status() == 0
    got, counts = _gpu_index(tree, idx)
    want = oracle.tree_index(*tree.arrays())
    for k in INDEX_KEYS:
        assert np.array_equal(got[k], want[k]), k


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def test_attn_tiny_fp32_all_rows():
    tree, a, _, dtype = inputs.make_inputs("tiny_fp32")
    got, scale = run_attn(tree, a)
    assert_close(got, oracle_attn(tree, a, scale), dtype)


@pytest.mark.parametrize("seed", range(3))
def test_attn_portable_fp32_random_trees(seed):
    rng = np.random.default_rng(600 + seed)
    tree = inputs.random_tree(rng, R=4, max_nodes=9, prefix_range=(0, 70), branch_range=(1, 40),
                              past_range=(0, 50))
    a = inputs.attn_inputs(tree, 6, 2, 64, torch.float32, rng)
    got, scale = run_attn(tree, a)
    assert_close(got, oracle_attn(tree, a, scale), torch.float32)


BF16_CASES = {
    # name: (tree builder, Hq, Hkv)
    "fanout_g4_ragged": (lambda rng: inputs.fanout_tree(2, 300, 6, 13), 8, 2),
    "fanout_g4_past": (lambda rng: inputs.fanout_tree(2, 170, 5, 29, past=77), 8, 2),
    "fanout_g1": (lambda rng: inputs.fanout_tree(1, 260, 3, 50), 2, 2),
    "fanout_g8": (lambda rng: inputs.fanout_tree(2, 140, 9, 5), 16, 2),
    "leveled_depth3_resume": (lambda rng: inputs.leveled_tree(rng, 3, depth_range=(2, 3),
                                                              options_range=(5, 40),
                                                              prefix_range=(100, 400),
                                                              n_resume=2), 8, 2),
    "random_irregular": (lambda rng: inputs.random_tree(rng, R=4, max_nodes=12,
                                                        prefix_range=(0, 200),
                                                        branch_range=(1, 70),
                                                        past_range=(0, 90)), 4, 1),
}


@pytest.mark.parametrize("case", sorted(BF16_CASES))
@pytest.mark.parametrize("flags", [0, flide.FLAG_PORTABLE], ids=["tc", "portable"])
def test_attn_bf16_vs_oracle(case, flags):
    rng = np.random.default_rng(zlib.crc32(case.encode()) % 1000)
    build_tree, Hq, Hkv = BF16_CASES[case]
    tree = build_tree(rng)
    a = inputs.attn_inputs(tree, Hq, Hkv, 128, torch.bfloat16, rng)
    got, scale = run_attn(tree, a, flags=flags)
    assert np.all(np.isfinite(got))
    assert_close(got, oracle_attn(tree, a, scale), torch.bfloat16)


# ---------------------------------------------------------------------------
# Gated DeltaNet
# ---------------------------------------------------------------------------

def test_gdn_tiny_fp32_all_outputs_and_states():
    tree, _, g, dtype = inputs.make_inputs("tiny_fp32")
    got, node_state, idx = run_gdn(tree, g)
    want, states = oracle_gdn(tree, g, want_states=True)
    assert_close(got, want, dtype)
    slot = idx.array("state_slot", tree.N).cpu().numpy()
    ns = node_state.cpu().numpy()
    for n in range(tree.N):
        if slot[n] >= 0:
            np.testing.assert_allclose(ns[slot[n]], states[n], atol=1e-4, rtol=0)


@pytest.mark.parametrize("seed", range(3))
def test_gdn_fp32_random_trees(seed):
    rng = np.random.default_rng(700 + seed)
    tree = inputs.random_tree(rng, R=3, max_nodes=10, prefix_range=(0, 50), branch_range=(1, 30),
                              past_range=(0, 5))
    g = inputs.gdn_inputs(tree, 3, 64, 32, torch.float32, rng)
    got, _, _ = run_gdn(tree, g)
    assert_close(got, oracle_gdn(tree, g), torch.float32)


@pytest.mark.parametrize("flags", [0, flide.FLAG_PORTABLE], ids=["tc", "portable"])
@pytest.mark.parametrize("seed", range(3))
def test_gdn_bf16_leveled(seed, flags):
    rng = np.random.default_rng(800 + seed)
    tree = inputs.leveled_tree(rng, 3, depth_range=(1, 3), options_range=(3, 30),
                               prefix_range=(60, 300), n_resume=1)
    g = inputs.gdn_inputs(tree, 4, 128, 128, torch.bfloat16, rng, gate_scale=0.1)
    got, node_state, idx = run_gdn(tree, g, flags=flags)
    want, states = oracle_gdn(tree, g, want_states=True)
    assert_close(got, want, torch.bfloat16)
    # saved end states of roots and inner nodes
    slot = idx.array("state_slot", tree.N).cpu().numpy()
    ns = node_state.cpu().numpy()
    for n in range(tree.N):
        if slot[n] >= 0:
            err = np.abs(ns[slot[n]] - states[n]).max()
            assert err <= 2e-2, (n, err)


@pytest.mark.parametrize("flags", [0, flide.FLAG_PORTABLE], ids=["tc", "portable"])
def test_gdn_bf16_strong_gates_long_prefix(flags):
    # gate scale 1 (alpha ~ 0.45 per token) over a prefix of many chunks
    tree = inputs.fanout_tree(2, 700, 9, 13, past=5)
    g = inputs.gdn_inputs(tree, 2, 128, 128, torch.bfloat16, np.random.default_rng(9), gate_scale=1.0)
    got, _, _ = run_gdn(tree, g, flags=flags)
    assert_close(got, oracle_gdn(tree, g), torch.bfloat16)


def test_gdn_state_capacity_error():
    tree = inputs.fanout_tree(2, 5, 3, 2)
    g = inputs.gdn_inputs(tree, 2, 64, 32, torch.float32, np.random.default_rng(1))
    _, idx = build(tree)
    node_state = torch.zeros((1, 2, 32, 64), device="cuda")
    flide.fork_gdn(g["q"].cuda(), g["k"].cuda(), g["v"].cuda(), g["g"].cuda(), g["beta"].cuda(),
                   idx, node_state)
    torch.cuda.synchronize()
    assert idx.status() == flide.ERR_CAPACITY
