"""Host logic of the CUDA-graph shape buckets, on the CPU: a batch goes to the
smallest bucket it fits (or is refused), and loading a tree writes the
request table padded with empty requests, zero past lengths for the padding,
the tree's rows at the front of every static buffer and zero initial states
for padded requests, also when a smaller tree follows a larger one in the
same bucket.  Buffers are allocated on the CPU; nothing is captured."""
import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import inputs
from tree_forked_decision_b200.graphs import BucketShape, GraphBucket, GraphBuckets

ATTN = dict(Hq=4, Hkv=2, d=16)
GDN = dict(H=2, dk=16, dv=16)


def _bucket(shape):
    b = object.__new__(GraphBucket)
    b.shape, b.attn_spec, b.gdn_spec, b.device, b.graph = shape, ATTN, GDN, "cpu", None
    b._alloc(torch.float32)
    return b


def _tensors(tree, seed):
    rng = np.random.default_rng(seed)
    a = inputs.attn_inputs(tree, ATTN["Hq"], ATTN["Hkv"], ATTN["d"], torch.float32, rng)
    g = inputs.gdn_inputs(tree, GDN["H"], GDN["dk"], GDN["dv"], torch.float32, rng)
    return a, g


def test_fits_and_pick_smallest():
    tree = inputs.fanout_tree(2, 30, 4, 5, past=3)            # R 2, N 10, T 100, P 6, D 1
    shapes = [BucketShape(8, 64, 4096, 512, 3), BucketShape(2, 10, 100, 6, 1),
              BucketShape(4, 32, 512, 64, 2)]
    assert [s.fits(tree) for s in shapes] == [True, True, True]
    assert not BucketShape(2, 10, 99, 6, 1).fits(tree)
    assert not BucketShape(2, 10, 100, 5, 1).fits(tree)
    assert not BucketShape(1, 10, 100, 6, 1).fits(tree)
    assert not BucketShape(2, 9, 100, 6, 1).fits(tree)
    deep = inputs._tree([(0, [(-1, 4), (0, 2), (1, 2)])], 2)
    assert not BucketShape(2, 10, 100, 6, 1).fits(deep)
    bs = object.__new__(GraphBuckets)
    bs.buckets = [_bucket(s) for s in sorted(shapes, key=lambda s: (s.T, s.N, s.R, s.P, s.D))]
    assert bs.pick(tree).shape == BucketShape(2, 10, 100, 6, 1)
    big = inputs.fanout_tree(3, 100, 8, 20, past=10)
    assert bs.pick(big).shape == BucketShape(8, 64, 4096, 512, 3)
    with pytest.raises(ValueError):
        bs.pick(inputs.fanout_tree(9, 10, 1, 1))


def _check_loaded(b, tree, a, g):
    s, R, N, T, P = b.shape, tree.R, tree.N, tree.T, tree.P_past
    rp = b.req_node_ptr.numpy()
    assert rp[:R + 1].tolist() == list(tree.req_node_ptr) and (rp[R + 1:] == N).all()
    pl = b.past_len.numpy()
    assert pl[:R].tolist() == list(tree.past_len) and (pl[R:] == 0).all()
    assert b.parent[:N].tolist() == list(tree.parent) and b.seg_len[:N].tolist() == list(tree.seg_len)
    for buf, src in ((b.q, a["q"]), (b.k, a["k"]), (b.v, a["v"]), (b.gq, g["q"]), (b.gk, g["k"]),
                     (b.gv, g["v"]), (b.gg, g["g"]), (b.gb, g["beta"])):
        assert torch.equal(buf[:T], src)
    if P:
        assert torch.equal(b.past_k[:P], a["past_k"]) and torch.equal(b.past_v[:P], a["past_v"])
    assert torch.equal(b.state_in[:R], g["state_in"])
    assert not b.state_in[R:].any()                            # padded requests start from zero
    assert b.loaded is tree


def test_load_pads_with_empty_requests_and_reloads_smaller():
    b = _bucket(BucketShape(6, 40, 800, 200, 8))
    rng = np.random.default_rng(4)
    big = inputs.random_tree(rng, R=5, max_nodes=7, prefix_range=(5, 40), branch_range=(1, 9),
                             past_range=(1, 30))
    assert b.shape.fits(big)
    a, g = _tensors(big, 1)
    g["state_in"] = torch.randn_like(g["state_in"])            # every request resumed
    _check_loaded(b.load(big, a, g), big, a, g)
    small = inputs.fanout_tree(2, 12, 3, 4, past=5)
    a2, g2 = _tensors(small, 2)
    _check_loaded(b.load(small, a2, g2), small, a2, g2)
    with pytest.raises(ValueError):
        b.load(inputs.fanout_tree(7, 4, 1, 1), None, None)
