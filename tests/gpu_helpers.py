"""Shared helpers for the GPU tests: run the CUDA path through the C ABI on a
seeded tree and compare with the oracle."""
import math

import numpy as np
import torch

import oracle
from tree_forked_decision_b200 import flide

FP32_MAX_ABS = 1e-4   # fp32 inputs: max-abs error bound vs the fp64 oracle
BF16_MAX_ABS = 2e-2   # bf16 inputs: max-abs error bound ...
BF16_REL_L2 = 1e-2    # ... and relative L2 error bound


def device_tree(tree, max_depth=None, N=None, T=None):
    md = tree.levels if max_depth is None else max_depth
    dt = flide.DeviceTree(*tree.arrays(), max_depth=md, N=N, T=T)
    idx = flide.TreeIndex(dt.R, dt.N, dt.T, dt.max_depth)
    return dt, idx


def build(tree, **kw):
    dt, idx = device_tree(tree, **kw)
    flide.tree_build(dt, idx)
    torch.cuda.synchronize()
    return dt, idx


def to_dev(x):
    return None if x is None else x.cuda()


def run_attn(tree, a, flags=0, idx=None):
    if idx is None:
        _, idx = build(tree)
    q, k, v = to_dev(a["q"]), to_dev(a["k"]), to_dev(a["v"])
    pk = to_dev(a["past_k"]) if a["past_k"].shape[0] else None
    pv = to_dev(a["past_v"]) if a["past_v"].shape[0] else None
    scale = 1.0 / math.sqrt(q.shape[2])
    out = flide.fork_attn(q, k, v, idx, scale, past_k=pk, past_v=pv, flags=flags)
    torch.cuda.synchronize()
    assert idx.status() == 0, idx.status()
    return out.float().cpu().numpy(), scale


def oracle_attn(tree, a, scale, rows=None):
    f = lambda t: t.float().numpy()
    if rows is None:
        return oracle.attention_all(tree.arrays(), f(a["q"]), f(a["k"]), f(a["v"]),
                                    f(a["past_k"]), f(a["past_v"]), scale)
    return oracle.attention_rows(tree.arrays(), f(a["q"]), f(a["k"]), f(a["v"]),
                                 f(a["past_k"]), f(a["past_v"]), scale, rows)


def run_gdn(tree, g, idx=None, n_slots=None, flags=0):
    if idx is None:
        _, idx = build(tree)
    q, k, v = to_dev(g["q"]), to_dev(g["k"]), to_dev(g["v"])
    H, dk, dv = q.shape[1], q.shape[2], v.shape[2]
    slots = n_slots if n_slots is not None else max(tree.N, 1)
    node_state = torch.zeros((slots, H, dv, dk), dtype=torch.float32, device="cuda")
    has_state = bool(np.any(tree.past_len > 0))
    state_in = to_dev(g["state_in"]) if has_state else None
    out = flide.fork_gdn(q, k, v, to_dev(g["g"]), to_dev(g["beta"]), idx, node_state,
                         state_in=state_in, flags=flags)
    torch.cuda.synchronize()
    assert idx.status() == 0, idx.status()
    return out.float().cpu().numpy(), node_state, idx


def oracle_gdn(tree, g, pairs=None, want_states=False):
    f = lambda t: t.float().numpy()
    has_state = bool(np.any(tree.past_len > 0))
    return oracle.gdn(tree.arrays(), f(g["q"]), f(g["k"]), f(g["v"]), f(g["g"]), f(g["beta"]),
                      state_in=f(g["state_in"]) if has_state else None, pairs=pairs,
                      want_states=want_states)


def errors(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    max_abs = float(np.max(np.abs(got - want))) if got.size else 0.0
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    return max_abs, rel


def assert_close(got, want, dtype):
    max_abs, rel = errors(got, want)
    if dtype == torch.float32:
        assert max_abs <= FP32_MAX_ABS, (max_abs, rel)
    else:
        assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_L2, (max_abs, rel)
    return max_abs, rel
