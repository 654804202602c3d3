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


def test_e4m3_and_paged_calls_replay_in_a_graph():
    """The e4m3 quantisation (amax, codes), the e4m3 attention and the paged
    attention are asynchronous, allocation-free calls: captured once in a CUDA
    graph with the tree build, a replay on new input values equals the same
    calls run eagerly, bit for bit."""
    tree = inputs.fanout_tree(2, 150, 5, 9, past=200)
    Hq, Hkv, d, rows_per_block = 8, 2, 128, 128
    dt = flide.DeviceTree(*tree.arrays(), max_depth=1)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, dt.max_depth)
    scale = 1.0 / math.sqrt(d)
    dev = lambda t: t.cuda()
    a = inputs.attn_inputs(tree, Hq, Hkv, d, torch.bfloat16, np.random.default_rng(0))
    q, k, v, pk, pv = (dev(a[n]) for n in ("q", "k", "v", "past_k", "past_v"))
    u8 = lambda t: torch.empty(t.shape, dtype=torch.uint8, device="cuda")
    q8, k8, v8, pk8, pv8 = u8(q), u8(k), u8(v), u8(pk), u8(pv)
    am = torch.zeros(3, device="cuda")
    ds = torch.empty(3, device="cuda")
    o8 = torch.empty_like(q)
    op = torch.empty_like(q)
    # pool: request r's past rows in blocks 2r+1, 2r (reversed order), slots 1, 0
    P = int(tree.past_len[0])
    nb = -(-P // rows_per_block)
    pool_k = torch.zeros((2 * tree.R * nb * rows_per_block, Hkv, d), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.zeros_like(pool_k)
    table = torch.zeros((tree.R, nb), dtype=torch.int32)
    slots = torch.tensor(list(range(tree.R))[::-1], dtype=torch.int32)
    for r in range(tree.R):
        for b in range(nb):
            table[slots[r], b] = tree.R * nb + r * nb + (nb - 1 - b)
    table_d, slots_d = table.view(-1).cuda(), slots.cuda()

    def fill_pool():
        for r in range(tree.R):
            for b in range(nb):
                blk = int(table[slots[r], b])
                n = min(rows_per_block, P - b * rows_per_block)
                src = slice(r * P + b * rows_per_block, r * P + b * rows_per_block + n)
                pool_k[blk * rows_per_block: blk * rows_per_block + n] = pk[src]
                pool_v[blk * rows_per_block: blk * rows_per_block + n] = pv[src]

    def calls():
        flide.tree_build(dt, idx)
        for i, (x, px) in enumerate(((q, None), (k, pk), (v, pv))):
            flide.amax(x, out=am[i:i + 1])
            if px is not None:
                flide.amax(px, out=am[i:i + 1], accumulate=True)
        for i, (x, x8, px, px8) in enumerate(((q, q8, None, None), (k, k8, pk, pk8), (v, v8, pv, pv8))):
            flide.quantize_e4m3(x, am[i:i + 1], out=x8, descale=ds[i:i + 1])
            if px is not None:
                flide.quantize_e4m3(px, am[i:i + 1], out=px8, descale=None)
        flide.fork_attn_fp8(q8, k8, v8, idx, scale, ds, past_k=pk8, past_v=pv8, out=o8)
        flide.fork_attn_paged(q, k, v, idx, scale, pool_k, pool_v, table_d, slots_d, rows_per_block, nb,
                              out=op)

    fill_pool()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        calls()  # first calls outside the capture (per-device set-up)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        calls()
    # new values in the same buffers, then replay
    b = inputs.attn_inputs(tree, Hq, Hkv, d, torch.bfloat16, np.random.default_rng(1))
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (pk, "past_k"), (pv, "past_v")):
        t.copy_(b[n])
    fill_pool()
    graph.replay()
    torch.cuda.synchronize()
    assert idx.status() == 0
    got = [t.clone() for t in (o8, op, q8, k8, pk8, ds)]
    calls()
    torch.cuda.synchronize()
    assert idx.status() == 0
    for g_, e_ in zip(got, (o8, op, q8, k8, pk8, ds)):
        assert torch.equal(g_, e_)
    # and the replayed paged output equals the packed-past attention on the new values
    assert torch.equal(got[1], flide.fork_attn(q, k, v, idx, scale, past_k=pk, past_v=pv))
