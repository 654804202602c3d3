"""flide_fork_attn_noalloc against flide_fork_attn and the oracle.

The scratch-free entry point exists for callers that cannot reserve scratch
memory next to the tree index -- because they only have read access to an
index built by another component, or because their framework's device memory
pool accepts no new allocations.  It runs the same kernels as the regular
entry point on the same inputs; only the place of the per-call work table
differs, so its output must be bit for bit the same.  These tests call both
through the C ABI, three scratch-free calls in a row on different trees (the
fixed device array keeps the previous call's contents; the third tree has
fewer requests than the second, so stale entries past its end would show),
compare each result with the fp64 oracle at the bf16 bar, check that the
tensor-core kernel ran (its rounding differs from the CUDA-core kernel's) and
that the caller's idx->work is never touched.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from tree_forked_decision_b200 import flide, inputs

from gpu_helpers import assert_close, build, oracle_attn

pytestmark = pytest.mark.gpu


def _run_three(tree, Hq, Hkv, seed):
    a_host = inputs.attn_inputs(tree, Hq, Hkv, 128, torch.bfloat16, np.random.default_rng(seed))
    a = {k: v.cuda() for k, v in a_host.items()}
    pk = a["past_k"] if a["past_k"].shape[0] else None
    pv = a["past_v"] if a["past_v"].shape[0] else None
    _, idx = build(tree)
    scale = 1.0 / math.sqrt(128)
    ref = flide.fork_attn(a["q"], a["k"], a["v"], idx, scale, past_k=pk, past_v=pv)
    simt = flide.fork_attn(a["q"], a["k"], a["v"], idx, scale, past_k=pk, past_v=pv,
                           flags=flide.FLAG_PORTABLE)
    torch.cuda.synchronize()
    work = idx.array("work", tree.R + 1)
    work.fill_(-7)  # sentinel: the scratch-free call must leave it alone
    got = flide.fork_attn_noalloc(a["q"], a["k"], a["v"], idx, scale, past_k=pk, past_v=pv)
    torch.cuda.synchronize()
    assert idx.status() == 0
    assert bool(torch.all(work == -7))
    return got, ref, simt, a_host, scale


def test_noalloc_matches_regular_entry_point_three_calls():
    rng = np.random.default_rng(5)
    cases = [
        (inputs.fanout_tree(3, 300, 7, 13, past=40), 8, 2, 11),
        (inputs.leveled_tree(rng, 5, depth_range=(1, 3), options_range=(3, 25),
                             prefix_range=(50, 300), n_resume=2), 16, 4, 12),
        (inputs.leveled_tree(rng, 2, depth_range=(2, 3), options_range=(2, 9),
                             prefix_range=(130, 260), n_resume=1), 8, 1, 13),
    ]
    assert cases[2][0].R < cases[1][0].R
    for tree, Hq, Hkv, seed in cases:
        got, ref, simt, a_host, scale = _run_three(tree, Hq, Hkv, seed)
        assert torch.equal(got, ref)
        assert not torch.equal(got, simt)  # the tensor-core kernel ran, not the CUDA-core one
        out = got.float().cpu().numpy()
        assert np.all(np.isfinite(out))
        assert_close(out, oracle_attn(tree, a_host, scale), torch.bfloat16)


def test_noalloc_rejects_too_many_requests():
    lib = flide.load()
    R = 16385
    idx = flide.TreeIndexC()
    nbytes = lib.flide_tree_index_bytes(R, R, R, 1)
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    assert lib.flide_tree_index_init(ctypes.byref(idx), buf.data_ptr(), nbytes, R, R, R, 1) == flide.OK
    q = torch.zeros((R, 8, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((R, 2, 128), dtype=torch.bfloat16, device="cuda")
    code = lib.flide_fork_attn_noalloc(q.data_ptr(), kv.data_ptr(), kv.data_ptr(), None, None, 0,
                                       ctypes.byref(idx), 8, 2, 128, flide.BF16, 0.1, q.data_ptr(), 0,
                                       torch.cuda.current_stream().cuda_stream)
    assert code == flide.ERR_CAPACITY
