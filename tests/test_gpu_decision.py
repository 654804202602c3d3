"""Decision scoring on the GPU (flide_branch_logprob, flide_option_probs)
against the fp64 oracle (oracle/decision.py): per-token log-probabilities,
path sums and leaf softmax, and the total variation distance of the decision
distributions (kongchang.com article on Flide, "total variation distance" box).

Bars: log p max-abs 1e-3 (bf16 inputs shared with the oracle, fp32
accumulation over D, so the difference is accumulation order and exp2
rounding); path sums rel. 1e-5 and probabilities abs. 1e-6 when both sides
start from the same log p; end-to-end TVD <= 1e-3 per request.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import build, run_attn

pytestmark = pytest.mark.gpu


def _inputs(tree, D, V, seed):
    rng = np.random.default_rng(seed)
    h = torch.from_numpy(inputs.normals(rng, (tree.T, D))).to(torch.bfloat16)
    w = torch.from_numpy(inputs.normals(rng, (V, D)) / np.float32(math.sqrt(D))).to(torch.bfloat16)
    y = torch.from_numpy(rng.integers(0, V, tree.T).astype(np.int32))
    return h, w, y


def _gpu(tree, h, w, y):
    _, idx = build(tree)
    logp = flide.branch_logprob(h.cuda(), w.cuda(), y.cuda(), idx)
    path, prob = flide.option_probs(idx, logp)
    torch.cuda.synchronize()
    assert idx.status() == 0
    return logp.cpu().numpy().astype(np.float64), path.cpu().numpy()[:tree.N], prob.cpu().numpy()[:tree.N]


CASES = {
    "fanout_one_vocab_tile": (lambda: inputs.fanout_tree(2, 100, 5, 7), 64, 128),
    "ragged_tiles_vocab_split": (lambda: inputs.fanout_tree(3, 40, 37, 9), 128, 4096),
    "leveled_depth3": (lambda: inputs.leveled_tree(np.random.default_rng(4), 4, depth_range=(2, 3),
                                                   options_range=(3, 9), prefix_range=(64, 300),
                                                   branch_range=(4, 40)), 512, 1024),
    "root_only_requests_mixed": (lambda: inputs._tree([(0, [(-1, 30)]), (3, [(-1, 10), (0, 5), (0, 2)]),
                                                       (0, []), (0, [(-1, 1), (0, 130)])], 1), 64, 256),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_branch_logprob_and_probs_vs_oracle(case):
    make, D, V = CASES[case]
    tree = make()
    h, w, y = _inputs(tree, D, V, 7)
    logp, path, prob = _gpu(tree, h, w, y)
    want = oracle.branch_logprob(tree.arrays(), h.double().numpy(), w.double().numpy(), y.numpy())
    root = np.isnan(want)
    assert np.all(np.isnan(logp[root]))
    assert np.max(np.abs(logp[~root] - want[~root]), initial=0.0) <= 1e-3
    wpath, wprob = oracle.option_probs(tree.arrays(), want)
    tv = oracle.tvd(tree.arrays(), prob, wprob)
    assert np.max(tv, initial=0.0) <= 1e-3, tv
    assert np.max(np.abs(path - wpath), initial=0.0) <= 1e-3 * max(1.0, np.max(np.abs(wpath), initial=0.0))


def test_option_probs_from_the_same_logp():
    tree = CASES["leveled_depth3"][0]()
    rng = np.random.default_rng(3)
    lp = -rng.random(tree.T) * 3.0
    _, idx = build(tree)
    path, prob = flide.option_probs(idx, torch.from_numpy(lp.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    wpath, wprob = oracle.option_probs(tree.arrays(), lp.astype(np.float32).astype(np.float64))
    path, prob = path.cpu().numpy()[:tree.N], prob.cpu().numpy()[:tree.N]
    assert np.allclose(path, wpath, rtol=1e-5, atol=1e-5)
    assert np.max(np.abs(prob - wprob)) <= 1e-6
    # every request with options sums to one
    rp = tree.req_node_ptr
    for r in range(tree.R):
        if rp[r + 1] - rp[r] > 1:
            assert abs(prob[rp[r]:rp[r + 1]].sum() - 1.0) < 1e-5


def test_decision_tvd_on_attention_output():
    """The hot path's own attention output as the hidden states."""
    tree = inputs.leveled_tree(np.random.default_rng(9), 3, depth_range=(1, 2), options_range=(4, 12),
                               prefix_range=(150, 400), branch_range=(4, 30))
    rng = np.random.default_rng(9)
    a = inputs.attn_inputs(tree, 8, 2, 128, torch.bfloat16, rng)
    o, _ = run_attn(tree, a)
    h = torch.from_numpy(o.reshape(tree.T, -1)).to(torch.bfloat16)  # [T, Hq * d]
    D, V = h.shape[1], 2048
    w = torch.from_numpy(inputs.normals(rng, (V, D)) / np.float32(math.sqrt(D) / 8)).to(torch.bfloat16)
    y = torch.from_numpy(rng.integers(0, V, tree.T).astype(np.int32))
    logp, _, prob = _gpu(tree, h, w, y)
    want = oracle.branch_logprob(tree.arrays(), h.double().numpy(), w.double().numpy(), y.numpy())
    _, wprob = oracle.option_probs(tree.arrays(), want)
    tv = oracle.tvd(tree.arrays(), prob, wprob)
    print(f"decision TVD per request vs fp64 oracle: {tv}")
    assert np.max(tv) <= 1e-3


def test_decision_fullsize_large_fanout():
    """4 requests x 256 options x 8 tokens (8192 branch tokens), D = 4096
    (Hq x d of the large fan-out attention), V = 8192."""
    tree = inputs.fanout_tree(4, 32768, 256, 8)
    D, V = 4096, 8192
    h, w, y = _inputs(tree, D, V, 11)
    _, idx = build(tree)
    logp = flide.branch_logprob(h.cuda(), w.cuda(), y.cuda(), idx)
    _, prob = flide.option_probs(idx, logp)
    torch.cuda.synchronize()
    assert idx.status() == 0
    logp, prob = logp.cpu().numpy().astype(np.float64), prob.cpu().numpy()[:tree.N]
    # oracle on the branch rows only: a tree with the roots' tokens moved to past
    wtree, rows = inputs.warm_variant(tree)
    want = oracle.branch_logprob(wtree.arrays(), h[torch.from_numpy(rows)].double().numpy(),
                                 w.double().numpy(), y.numpy()[rows])
    assert np.max(np.abs(logp[rows] - want)) <= 1e-3
    _, wprob = oracle.option_probs(wtree.arrays(), want)
    tv = oracle.tvd(tree.arrays(), prob, wprob)
    print(f"full-size decision TVD per request: {tv}")
    assert np.max(tv) <= 1e-3


def test_decision_rejects_unsupported_shapes():
    tree = inputs.fanout_tree(1, 10, 2, 3)
    _, idx = build(tree)
    h = torch.zeros((tree.T, 100), dtype=torch.bfloat16, device="cuda")  # D not a multiple of 64
    w = torch.zeros((128, 100), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(tree.T, dtype=torch.int32, device="cuda")
    with pytest.raises(flide.FlideError):
        flide.branch_logprob(h, w, y, idx)
