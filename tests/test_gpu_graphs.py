"""CUDA-graph shape buckets: one captured graph replays any tree that fits,
bit for bit equal to the eager call sequence, and matches the oracle."""
import math

import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import flide, inputs
from tree_forked_decision_b200.graphs import BucketShape, GraphBuckets

from gpu_helpers import assert_close, oracle_attn, oracle_gdn, run_attn, run_gdn

pytestmark = pytest.mark.gpu

ATTN = dict(Hq=8, Hkv=2, d=128)
GDN = dict(H=2, dk=128, dv=128)


def _trees():
    rng = np.random.default_rng(42)
    return [
        inputs.fanout_tree(2, 180, 6, 11, past=30),
        inputs.leveled_tree(rng, 3, depth_range=(1, 3), options_range=(3, 12),
                            prefix_range=(40, 200), n_resume=1),
        inputs.random_tree(rng, R=4, max_nodes=10, prefix_range=(0, 90), branch_range=(1, 40),
                           past_range=(0, 40)),
    ]


def test_graph_bucket_replay_matches_eager_and_oracle():
    buckets = GraphBuckets([BucketShape(R=4, N=64, T=1200, P=200, D=8),
                            BucketShape(R=8, N=256, T=4096, P=512, D=8)], ATTN, GDN).capture()
    for i, tree in enumerate(_trees()):
        rng = np.random.default_rng(100 + i)
        a = inputs.attn_inputs(tree, ATTN["Hq"], ATTN["Hkv"], ATTN["d"], torch.bfloat16, rng)
        g = inputs.gdn_inputs(tree, GDN["H"], GDN["dk"], GDN["dv"], torch.bfloat16, rng,
                              gate_scale=0.1)
        b = buckets.run(tree, a, g)
        torch.cuda.synchronize()
        assert b.idx.status() == 0
        out = {k: v.float().cpu().numpy() for k, v in b.outputs().items()}
        eager_a, scale = run_attn(tree, a)
        eager_g, _, _ = run_gdn(tree, g)
        assert np.array_equal(out["attn"], eager_a)
        assert np.array_equal(out["gdn"], eager_g)
        assert_close(out["attn"], oracle_attn(tree, a, scale), torch.bfloat16)
        assert_close(out["gdn"], oracle_gdn(tree, g), torch.bfloat16)


def test_graph_bucket_rejects_oversize_tree():
    buckets = GraphBuckets([BucketShape(R=2, N=8, T=100, P=0, D=1)], ATTN, None)
    with pytest.raises(ValueError):
        buckets.pick(inputs.fanout_tree(1, 200, 2, 4))
