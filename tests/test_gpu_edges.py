"""Edge cases and checkpoint resume on the GPU path."""
import math

import numpy as np
import pytest
import torch

import oracle
from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import (assert_close, build, oracle_attn, oracle_gdn, run_attn, run_gdn, to_dev)

pytestmark = pytest.mark.gpu

EDGE_TREES = {
    "root_only_and_branches": lambda: inputs._tree([(0, [(-1, 70)]), (0, [(-1, 33), (0, 9), (0, 4)])], 1),
    "zero_token_root_with_past": lambda: inputs._tree([(50, [(-1, 0), (0, 5), (0, 7)]),
                                                       (0, [(-1, 20), (0, 3)])], 1),
    "single_token_branches": lambda: inputs.fanout_tree(2, 100, 40, 1),
    "depth8_chain": lambda: inputs._tree([(3, [(-1, 17)] + [(i, 5 + i) for i in range(8)])], 8),
    "depth9_chain_portable": lambda: inputs._tree([(0, [(-1, 9)] + [(i, 3) for i in range(9)])], 9),
    "wide_257_leaves": lambda: inputs.fanout_tree(1, 129, 257, 2),
}


@pytest.mark.parametrize("flags", [0, flide.FLAG_PORTABLE], ids=["tc", "portable"])
@pytest.mark.parametrize("case", sorted(EDGE_TREES))
def test_edge_attention_and_gdn(case, flags):
    tree = EDGE_TREES[case]()
    rng = np.random.default_rng(3)
    a = inputs.attn_inputs(tree, 8, 2, 128, torch.bfloat16, rng)
    got, scale = run_attn(tree, a, flags=flags)
    assert np.all(np.isfinite(got))
    assert_close(got, oracle_attn(tree, a, scale), torch.bfloat16)
    g = inputs.gdn_inputs(tree, 2, 128, 128, torch.bfloat16, rng, gate_scale=0.1)
    gg, _, _ = run_gdn(tree, g, flags=flags)
    assert_close(gg, oracle_gdn(tree, g), torch.bfloat16)


def test_edge_gdn_small_head_dims():
    tree = EDGE_TREES["zero_token_root_with_past"]()
    rng = np.random.default_rng(4)
    g = inputs.gdn_inputs(tree, 2, 64, 64, torch.bfloat16, rng, gate_scale=0.1)
    gg, _, _ = run_gdn(tree, g)
    assert_close(gg, oracle_gdn(tree, g), torch.bfloat16)


def test_empty_batch_runs_clean():
    tree = inputs._tree([(0, []), (0, [])], 0)
    dt = flide.DeviceTree(*tree.arrays(), max_depth=1, N=1, T=1)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, 1)
    flide.tree_build(dt, idx)
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device="cuda")
    flide.fork_attn(q, kv, kv, idx, 0.1)
    gq = torch.zeros((1, 2, 64), dtype=torch.bfloat16, device="cuda")
    gf = torch.zeros((1, 2), dtype=torch.float32, device="cuda")
    ns = torch.zeros((1, 2, 64, 64), device="cuda")
    flide.fork_gdn(gq, gq, gq, gf, gf, idx, ns)
    torch.cuda.synchronize()
    assert idx.status() == 0
    assert idx.counts()["N"] == 0 and idx.counts()["T"] == 0


def test_checkpoint_save_resume_equals_scratch():
    """Pass 1 runs requests whose roots are histories and saves checkpoints;
    pass 2 resumes them with a new observation as root and new options.  Its
    outputs must equal one pass over history + observation from scratch."""
    Hq, Hkv, d, H, dk, dv = 8, 2, 128, 2, 128, 128
    rng = np.random.default_rng(11)
    hist = [(7, 150), (0, 97), (20, 260)]   # (past, root tokens) of pass 1
    new = [(12, [9, 14, 3]), (5, [6]), (31, [4, 4, 8, 2])]  # (root tokens, option lengths)
    pass1 = inputs._tree([(p, [(-1, h), (0, 5)]) for p, h in hist], 1)
    scratch = inputs._tree([(p, [(-1, h + n)] + [(0, o) for o in opts])
                            for (p, h), (n, opts) in zip(hist, new)], 1)
    # one set of token tensors laid out for the scratch tree; pass 1 and
    # pass 2 take their rows from it
    a = inputs.attn_inputs(scratch, Hq, Hkv, d, torch.bfloat16, rng)
    g = inputs.gdn_inputs(scratch, H, dk, dv, torch.bfloat16, rng, gate_scale=0.1)
    g["state_in"] = g["state_in"] * 0 + torch.from_numpy(
        inputs.normals(rng, tuple(g["state_in"].shape)) * np.float32(0.1))
    s_starts = np.concatenate([[0], np.cumsum(scratch.seg_len)])
    rp = scratch.req_node_ptr
    rows1, rows2 = [], []
    for r, ((p, h), (n, opts)) in enumerate(zip(hist, new)):
        r0 = s_starts[rp[r]]
        rows1 += list(range(r0, r0 + h)) + list(range(r0, r0 + 5))  # root + a dummy option
        rows2 += list(range(r0 + h, s_starts[rp[r + 1]]))
    rows1, rows2 = np.asarray(rows1), np.asarray(rows2)
    sel = lambda t, rows: t[torch.from_numpy(rows)].contiguous()

    # pass 1 on the GPU, then save
    _, idx1 = build(pass1)
    dev = lambda t: t.cuda()
    k1, v1 = dev(sel(a["k"], rows1)), dev(sel(a["v"], rows1))
    flide.fork_attn(dev(sel(a["q"], rows1)), k1, v1, idx1, 1 / math.sqrt(d),
                    past_k=dev(a["past_k"]), past_v=dev(a["past_v"]))
    ns1 = torch.zeros((pass1.N, H, dv, dk), device="cuda")
    flide.fork_gdn(dev(sel(g["q"], rows1)), dev(sel(g["k"], rows1)), dev(sel(g["v"], rows1)),
                   dev(sel(g["g"], rows1)), dev(sel(g["beta"], rows1)), idx1, ns1,
                   state_in=dev(g["state_in"]))
    ck_rows = pass1.P_past + pass1.root_tokens
    ck = torch.empty((ck_rows, Hkv, d), dtype=torch.bfloat16, device="cuda")
    cv = torch.empty_like(ck)
    cS = torch.empty((pass1.R, H, dv, dk), device="cuda")
    flide.state_save(idx1, k1, v1, ck, cv, cS, past_k=dev(a["past_k"]), past_v=dev(a["past_v"]),
                     node_state=ns1)
    torch.cuda.synchronize()
    assert idx1.status() == 0

    # resume into pass 2 (request order permuted on purpose)
    perm = [2, 0, 1]
    pass2 = inputs._tree([(hist[s][0] + hist[s][1], [(-1, new[s][0])] + [(0, o) for o in new[s][1]])
                          for s in perm], 1)
    src_req = torch.tensor(perm, dtype=torch.int32, device="cuda")
    past_len = torch.zeros(3, dtype=torch.int32, device="cuda")
    pk = torch.empty((pass2.P_past, Hkv, d), dtype=torch.bfloat16, device="cuda")
    pv = torch.empty_like(pk)
    state_in2 = torch.empty((3, H, dv, dk), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flide.state_resume(src_req, idx1.array("ckpt_start", 4), ck, cv, cS, past_len, pk, pv,
                       state_in2, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert past_len.cpu().tolist() == pass2.past_len.tolist()
    dt2 = flide.DeviceTree(pass2.req_node_ptr, pass2.parent, pass2.seg_len, pass2.past_len,
                           max_depth=1)
    dt2.past_len = past_len  # the resumed lengths, written on the device
    idx2 = flide.TreeIndex(dt2.R, dt2.N, dt2.T, 1)
    flide.tree_build(dt2, idx2)
    p_rows = np.concatenate([rows2[np.isin(rows2, np.arange(s_starts[rp[s]], s_starts[rp[s + 1]]))]
                             for s in perm])
    o2 = flide.fork_attn(dev(sel(a["q"], p_rows)), dev(sel(a["k"], p_rows)), dev(sel(a["v"], p_rows)),
                         idx2, 1 / math.sqrt(d), past_k=pk, past_v=pv)
    ns2 = torch.zeros((pass2.N, H, dv, dk), device="cuda")
    go2 = flide.fork_gdn(dev(sel(g["q"], p_rows)), dev(sel(g["k"], p_rows)),
                         dev(sel(g["v"], p_rows)), dev(sel(g["g"], p_rows)),
                         dev(sel(g["beta"], p_rows)), idx2, ns2, state_in=state_in2)
    torch.cuda.synchronize()
    assert idx2.status() == 0

    # the oracle over the scratch tree, rows of pass 2 in pass-2 order
    f = lambda t: t.float().numpy()
    heads = np.repeat(np.arange(Hq)[None], len(p_rows), 0)
    rows = np.stack([np.repeat(p_rows, Hq), heads.ravel()], 1)
    want_a = oracle.attention_rows(scratch.arrays(), f(a["q"]), f(a["k"]), f(a["v"]),
                                   f(a["past_k"]), f(a["past_v"]), 1 / math.sqrt(d), rows)
    assert_close(o2.float().cpu().numpy().reshape(-1, d), want_a, torch.bfloat16)
    want_g = oracle.gdn(scratch.arrays(), f(g["q"]), f(g["k"]), f(g["v"]), f(g["g"]),
                        f(g["beta"]), state_in=f(g["state_in"]))
    assert_close(go2.float().cpu().numpy(), want_g[p_rows], torch.bfloat16)


def test_resume_fresh_request_and_bad_source():
    Hkv, d = 2, 128
    src_start = torch.tensor([0, 5, 9], dtype=torch.int32, device="cuda")
    sk = torch.randn((9, Hkv, d), device="cuda").to(torch.bfloat16)
    sS = torch.randn((2, 1, 32, 32), device="cuda")
    past_len = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    pk = torch.zeros((9, Hkv, d), dtype=torch.bfloat16, device="cuda")
    st = torch.full((3, 1, 32, 32), 7.0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flide.state_resume(torch.tensor([1, -1, 0], dtype=torch.int32, device="cuda"), src_start,
                       sk, sk, sS, past_len, pk, pk.clone(), st, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert past_len.cpu().tolist() == [4, 0, 5]
    assert torch.equal(pk[:4], sk[5:9]) and torch.equal(pk[4:9], sk[0:5])
    assert torch.equal(st[0], sS[1]) and bool((st[1] == 0).all()) and torch.equal(st[2], sS[0])
    flide.state_resume(torch.tensor([2, 0, 0], dtype=torch.int32, device="cuda"), src_start,
                       sk, sk, sS, past_len, pk, pk.clone(), st, status)
    torch.cuda.synchronize()
    assert int(status.item()) == flide.ERR_INVALID


@pytest.mark.parametrize("path", ["tc", "portable", "noalloc"])
def test_past_buffers_shorter_than_tree_past_are_refused(path):
    """The tree asks for 80 past rows but the caller passes buffers of 60: the
    kernels must report FLIDE_ERR_CAPACITY instead of reading rows beyond the
    buffers (the tensor-core path would otherwise attend to zero rows).  The
    60-row buffers are views of longer tensors, so no read can leave device
    memory whatever the kernels do."""
    tree = inputs._tree([(50, [(-1, 10), (0, 5)]), (30, [(-1, 8), (0, 3)])], 1)
    rng = np.random.default_rng(9)
    a = inputs.attn_inputs(tree, 8, 2, 128, torch.bfloat16, rng)
    assert a["past_k"].shape[0] == 80
    pk, pv = to_dev(a["past_k"]), to_dev(a["past_v"])
    _, idx = build(tree)
    q, k, v = to_dev(a["q"]), to_dev(a["k"]), to_dev(a["v"])
    if path == "noalloc":
        flide.fork_attn_noalloc(q, k, v, idx, 0.1, past_k=pk[:60], past_v=pv[:60])
    else:
        flags = flide.FLAG_PORTABLE if path == "portable" else 0
        flide.fork_attn(q, k, v, idx, 0.1, past_k=pk[:60], past_v=pv[:60], flags=flags)
    torch.cuda.synchronize()
    assert idx.status() == flide.ERR_CAPACITY
    # the same call with every row present runs clean
    _, idx2 = build(tree)
    flide.fork_attn(q, k, v, idx2, 0.1, past_k=pk, past_v=pv)
    torch.cuda.synchronize()
    assert idx2.status() == 0


def test_tree_token_total_beyond_int32_is_refused():
    """Per-node lengths that pass every single check but add up past 2^31 - 1
    (tokens plus past rows) must give FLIDE_ERR_CAPACITY before the int32
    prefix sums can wrap.  The descriptor's token capacity is set high so
    that only the 64-bit total check can catch it; no layer kernel runs."""
    rp = np.array([0, 3, 5], np.int32)
    parent = np.array([-1, 0, 0, -1, 0], np.int32)
    seg = np.array([1, 1, 1, 1, 1], np.int32)
    past = np.array([0x7ffffff0, 0x20], np.int32)
    dt = flide.DeviceTree(rp, parent, seg, past, max_depth=1, N=5, T=16)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, 1)
    flide.tree_build(dt, idx)
    torch.cuda.synchronize()
    assert idx.status() == flide.ERR_CAPACITY
