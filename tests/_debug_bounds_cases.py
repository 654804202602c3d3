"""Small cases of every layer call, run once with each build of the library.

test_debug_bounds*.py run these in a child process with FLIDE_DEBUG_BOUNDS=1
(the bounds-checked libflide_dbg.so) and in a child with the release build,
and compare what both wrote.  Not collected by pytest (no test_ prefix)."""
import json
import math
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tree_forked_decision_b200 import flide, inputs  # noqa: E402


def run(out_dir):
    torch.cuda.set_device(0)
    res = {"debug_bounds": int(flide._lib().flide_debug_bounds())}
    arrays = {}
    rng = np.random.default_rng(21)
    tree = inputs.leveled_tree(rng, 3, depth_range=(1, 3), options_range=(3, 12),
                               prefix_range=(90, 260), n_resume=1)
    dt = flide.DeviceTree(*tree.arrays(), max_depth=tree.levels)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, dt.max_depth)
    flide.tree_build(dt, idx)
    torch.cuda.synchronize()
    res["status_tree"] = idx.status()
    for name in flide.INDEX_ARRAYS[2:-1]:  # every index array but status, counts and scratch
        n = {"node_start": tree.N + 1, "anc_ptr": tree.N + 1, "token_node": tree.T, "token_pos": tree.T,
             "past_start": tree.R + 1, "req_node": tree.R + 1, "ckpt_start": tree.R + 1,
             "level_ptr": tree.levels + 2}.get(name, tree.N)
        arrays["idx_" + name] = idx.array(name, n).cpu().numpy()
    a = inputs.attn_inputs(tree, 8, 2, 128, torch.bfloat16, rng)
    ad = {k: v.cuda() for k, v in a.items()}
    scale = 1.0 / math.sqrt(128)
    for tag, flags in (("tc", 0), ("portable", flide.FLAG_PORTABLE)):
        o = flide.fork_attn(ad["q"], ad["k"], ad["v"], idx, scale, past_k=ad["past_k"],
                            past_v=ad["past_v"], flags=flags)
        torch.cuda.synchronize()
        res["status_attn_" + tag] = idx.status()
        arrays["attn_" + tag] = o.float().cpu().numpy()
    g = inputs.gdn_inputs(tree, 2, 128, 128, torch.bfloat16, rng, gate_scale=0.1)
    gd = {k: v.cuda() for k, v in g.items()}
    slots = max(flide.state_slots(tree), 1)
    for tag, flags in (("tc", 0), ("portable", flide.FLAG_PORTABLE)):
        ns = torch.zeros((slots, 2, 128, 128), device="cuda")
        go = flide.fork_gdn(gd["q"], gd["k"], gd["v"], gd["g"], gd["beta"], idx, ns,
                            state_in=gd["state_in"], flags=flags)
        torch.cuda.synchronize()
        res["status_gdn_" + tag] = idx.status()
        arrays["gdn_" + tag] = go.float().cpu().numpy()
        arrays["gdn_states_" + tag] = ns.cpu().numpy()
    ck = torch.empty((tree.P_past + tree.root_tokens, 2, 128), dtype=torch.bfloat16, device="cuda")
    cv = torch.empty_like(ck)
    cS = torch.empty((tree.R, 2, 128, 128), device="cuda")
    flide.state_save(idx, ad["k"], ad["v"], ck, cv, cS, past_k=ad["past_k"], past_v=ad["past_v"],
                     node_state=ns)
    torch.cuda.synchronize()
    res["status_save"] = idx.status()
    arrays["ckpt_k"] = ck.float().cpu().numpy()
    arrays["ckpt_S"] = cS.cpu().numpy()
    o = flide.fork_attn(ad["q"], ad["k"], ad["v"], idx, scale, past_k=ad["past_k"], past_v=ad["past_v"])
    D, V = 8 * 128, 512
    grng = torch.Generator(device="cpu").manual_seed(5)
    w = (torch.randn((V, D), generator=grng) / math.sqrt(D)).to(torch.bfloat16).cuda()
    y = torch.randint(0, V, (tree.T,), generator=grng, dtype=torch.int32).cuda()
    lp = flide.branch_logprob(o.view(tree.T, D), w, y, idx)
    path, prob = flide.option_probs(idx, lp)
    torch.cuda.synchronize()
    res["status_decision"] = idx.status()
    arrays["logp"] = lp.cpu().numpy()
    arrays["prob"] = prob.cpu().numpy()
    np.savez(os.path.join(out_dir, "arrays.npz"), **arrays)
    with open(os.path.join(out_dir, "result.json"), "w") as f:
        json.dump(res, f)


def run_corrupt(out_dir):
    """Debug build only: a branch token's node id is overwritten with one past
    the tree's nodes after the build.  The tensor-core attention's item decode
    and the CUDA-core attention must report FLIDE_ERR_BOUNDS (their checks on
    token_node) instead of indexing with it.  Without the checks the reads would
    still stay inside the index buffer (the id is only two past the node
    count), so no access leaves device memory either way."""
    torch.cuda.set_device(0)
    assert flide._lib().flide_debug_bounds() == 1
    res = {}
    tree = inputs.fanout_tree(2, 100, 6, 9)
    a = inputs.attn_inputs(tree, 8, 2, 128, torch.bfloat16, np.random.default_rng(3))
    ad = {k: v.cuda() for k, v in a.items()}
    for tag, flags in (("tc", 0), ("portable", flide.FLAG_PORTABLE)):
        dt = flide.DeviceTree(*tree.arrays(), max_depth=1)
        idx = flide.TreeIndex(dt.R, dt.N, dt.T, dt.max_depth)
        flide.tree_build(dt, idx)
        torch.cuda.synchronize()
        tn = idx.array("token_node", tree.T)
        tn[150] = tree.N + 2  # a branch token of the first request
        flide.fork_attn(ad["q"], ad["k"], ad["v"], idx, 0.1, flags=flags)
        torch.cuda.synchronize()
        c = idx.counts()
        res[tag] = [idx.status(), c["CHECK_SITE"], c["CHECK_VALUE"]]
    with open(os.path.join(out_dir, "corrupt.json"), "w") as f:
        json.dump(res, f)


if __name__ == "__main__":
    if sys.argv[1] == "corrupt":
        run_corrupt(sys.argv[2])
    else:
        run(sys.argv[2])
