"""Parity at the boundaries of the tensor-core kernels' tilings.

Attention packs G = Hq/Hkv query heads of one kv head with the tokens into the
128 MMA rows of a tile half, so a half holds 128/G tokens: the large groups
(G = 16, 32, 128; 8, 4 and 1 tokens per half) are the cases where a tile is a
handful of tokens and ragged tails and node boundaries fall inside almost
every tile.  The GDN scan cuts nodes into 64-token chunks and packs runs of
sibling leaves that fit one chunk into one block-diagonal item: segments of
exactly 63, 64, 65, 127, 128 and 129 tokens, one-token leaves and two leaves
that fill a chunk exactly sit on those cuts.  Both are compared with the
oracle (kongchang.com article on Flide, "ForkAttention" section: every branch
equals its isolated sequence; its Gated DeltaNet box for the recurrent layer),
the GDN's saved node states too."""
import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import assert_close, oracle_attn, oracle_gdn, run_attn, run_gdn

pytestmark = pytest.mark.gpu


def _boundary_tree():
    # request 0: root 64; children 63, [inner 64 -> leaves 64, 1 + 31], 65,
    # 32 + 32 (packed: exactly one chunk), 1, 64.  request 1: 5 past rows;
    # root 129; leaves 127, 128, 31 + 33 (exactly one chunk).  Nodes in level
    # order, siblings consecutive.
    r0 = [(-1, 64), (0, 63), (0, 64), (0, 65), (0, 32), (0, 32), (0, 1), (0, 64),
          (2, 64), (2, 1), (2, 31)]
    r1 = [(-1, 129), (0, 127), (0, 128), (0, 31), (0, 33)]
    return inputs._tree([(0, r0), (5, r1)], 2)


@pytest.mark.parametrize("Hq,Hkv", [(32, 2), (32, 1), (128, 1)], ids=["g16", "g32", "g128"])
def test_attn_large_head_groups(Hq, Hkv):
    rng = np.random.default_rng(Hq * 7 + Hkv)
    for tree in (inputs.fanout_tree(2, 37, 5, 3, past=9), _boundary_tree()):
        a = inputs.attn_inputs(tree, Hq, Hkv, 128, torch.bfloat16, rng)
        got, scale = run_attn(tree, a)
        simt, _ = run_attn(tree, a, flags=flide.FLAG_PORTABLE)
        assert not np.array_equal(got, simt)  # the tensor-core kernel ran
        assert np.all(np.isfinite(got))
        assert_close(got, oracle_attn(tree, a, scale), torch.bfloat16)


def test_gdn_chunk_boundaries_outputs_and_states():
    tree = _boundary_tree()
    rng = np.random.default_rng(64)
    g = inputs.gdn_inputs(tree, 2, 128, 128, torch.bfloat16, rng, gate_scale=0.1)
    got, node_state, idx = run_gdn(tree, g)
    want, states = oracle_gdn(tree, g, want_states=True)
    assert np.all(np.isfinite(got))
    assert_close(got, want, torch.bfloat16)
    slot = idx.array("state_slot", tree.N).cpu().numpy()
    ns = node_state.cpu().numpy()
    saved = [n for n in range(tree.N) if slot[n] >= 0]
    assert len(saved) == 3  # the two roots and the inner node
    for n in saved:
        err = np.abs(ns[slot[n]] - states[n]).max()
        assert err <= 2e-2, (n, err)
